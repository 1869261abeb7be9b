"""One decode step (nosa_step) captured in a CUDA graph over static buffers.

Host orchestration only: the graph holds the same kernels that NosaCache.step launches (fused
append + score + selection, the page copies with host pools, split-K attention with its
combine), with their arguments frozen to the buffers below. Everything that carries over from
one step to the next lives on the device: the cache state, and the per-group "selection
published" / "pages in place" flags and tickets in the workspace, which the last consumer of
a group clears. One captured graph therefore serves every step of a cache, as long as each
step's inputs are first copied into the graph's input buffers (`stage`).
"""
from __future__ import annotations

from typing import Optional

import torch


class StepGraph:
    """nosa_step of `cache` captured once and replayed per decode step.

    Inputs (`q`, `k_new`, `v_new`, `evict` and, with one forecast row per group, `rows`) and
    outputs (`sel`, `out`, `miss`) are the graph's own device buffers, flat, in the layouts
    nosa_step documents. `run` stages a step's inputs and replays the graph on the current
    stream; results are in `sel`, `out` and `miss[:B*Hkv]` once that stream reaches them.
    Capture after the cache has taken at least one step with direct launches (the usual
    warm-up before a capture), so that the kernels are loaded before their launches are
    recorded.
    """

    def __init__(self, cache, forecast_rows: bool = False):
        c = cache.cfg
        dev = cache.device
        G = c.Hq // c.Hkv
        ng = c.B * c.Hkv
        if not forecast_rows and c.n_score_rows != G:
            raise ValueError("the configuration scores with forecast rows: pass forecast_rows=True")
        self.n_groups = ng
        self.q = torch.empty(c.B * c.Hq * c.d, dtype=torch.int16, device=dev)
        self.k_new = torch.empty(ng * c.d, dtype=torch.int16, device=dev)
        self.v_new = torch.empty(ng * c.d, dtype=torch.int16, device=dev)
        self.evict = torch.empty(ng * c.max_blocks, dtype=torch.float32, device=dev)
        self.rows = (torch.empty(ng * c.n_score_rows * c.d, dtype=torch.int16, device=dev)
                     if forecast_rows else None)
        self.sel = torch.empty(ng * (c.k_q + c.k_e), dtype=torch.int32, device=dev)
        self.out = torch.empty(c.B * c.Hq * c.d, dtype=torch.float32, device=dev)
        self.miss = torch.empty(-(-ng // 4) * 4, dtype=torch.int32, device=dev)
        self.graph = torch.cuda.CUDAGraph()
        torch.cuda.synchronize(dev)
        # capture records the launches; nothing runs (the cache state is not touched)
        with torch.cuda.graph(self.graph, capture_error_mode="relaxed"):
            cache.step(self.q, self.k_new, self.v_new, self.evict, self.sel, self.out,
                       self.miss[:ng], score_rows=self.rows)

    def stage(self, q, k_new, v_new, evict, rows: Optional[torch.Tensor] = None):
        """Copies one step's inputs (device tensors of the documented sizes) into the graph's
        buffers, on the current stream."""
        self.q.copy_(q.reshape(-1), non_blocking=True)
        self.k_new.copy_(k_new.reshape(-1), non_blocking=True)
        self.v_new.copy_(v_new.reshape(-1), non_blocking=True)
        self.evict.copy_(evict.reshape(-1), non_blocking=True)
        if self.rows is not None:
            if rows is None:
                raise ValueError("this graph scores with forecast rows: pass rows")
            self.rows.copy_(rows.reshape(-1), non_blocking=True)

    def replay(self):
        """One decode step on the staged inputs, on the current stream."""
        self.graph.replay()

    def run(self, q, k_new, v_new, evict, rows: Optional[torch.Tensor] = None):
        self.stage(q, k_new, v_new, evict, rows)
        self.replay()
