"""Allocation helper: owns the decode-state buffers of one NOSA layer.

Memory comes from PyTorch (device tensors, and pinned host tensors for the
offloaded backing copy); all computation goes through the C ABI.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import (nosa_config, nosa_state, STATE_FIELDS, state_sizes, workspace_size, workspace_init,
               state_init, append, score_blocks, select, gather, decode_attn, step, check_device,
               plan_ahead, prefetch, attend, stop_counts, NosaError, NOSA_EINVAL)

_DTYPE = {"seq_len": torch.int32, "kc": torch.float32, "prev_sel": torch.int32,
          "alive": torch.int32, "last_used": torch.int32, "block_table": torch.int32,
          "slot_owner": torch.int32, "k_pool": torch.int16, "v_pool": torch.int16,
          "host_k": torch.int16, "host_v": torch.int16, "err": torch.int32}


def buffer_bytes(cfg: nosa_config) -> dict:
    """Bytes of each per-call buffer in the layouts include/nosa.h documents."""
    ng = cfg.B * cfg.Hkv
    k = cfg.k_q + cfg.k_e
    return {"q": cfg.B * cfg.Hq * cfg.d * 2, "out": cfg.B * cfg.Hq * cfg.d * 4,
            "k_new": ng * cfg.d * 2, "v_new": ng * cfg.d * 2,
            "score_rows": ng * cfg.n_score_rows * cfg.d * 2,
            "block_scores": ng * cfg.max_blocks * 4, "evict": ng * cfg.max_blocks * 4,
            "sel": ng * k * 4, "miss_count": ng * 4, "used": cfg.B * cfg.Hq * 4,
            "prefill_len": cfg.B * 4, "resident": ng * cfg.max_blocks}


def check_buffer(name: str, t, nbytes: int, device: Optional[torch.device] = None):
    """Refuses (NosaError, NOSA_EINVAL) a tensor that is not a contiguous CUDA tensor of at
    least `nbytes` bytes on `device` (the GPU that holds the state): the kernels read and write
    the documented extent through its data pointer, and a pointer into another GPU's memory
    would fault there instead of failing here. Integer addresses pass unchecked, as at the C
    ABI."""
    if t is None or isinstance(t, int):
        return
    if not t.is_cuda:
        raise NosaError(NOSA_EINVAL, f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise NosaError(NOSA_EINVAL, f"{name} is on {t.device}, the state is on {device}")
    if not t.is_contiguous():
        raise NosaError(NOSA_EINVAL, f"{name} must be contiguous")
    have = t.numel() * t.element_size()
    if have < nbytes:
        raise NosaError(NOSA_EINVAL, f"{name} holds {have} bytes, the call needs {nbytes}")


class NosaCache:
    """Decode state + workspace for one configuration.

    offload=True keeps the full K/V backing copy in pinned host memory and
    `cfg.slots` pages per group in HBM; otherwise every block is in HBM.
    Every call checks the sizes of the buffers it is given (check_buffer) before
    the library launches anything.
    """

    def __init__(self, cfg: nosa_config, offload: bool = False, device: str = "cuda"):
        self.cfg = cfg
        self.offload = offload
        self.device = torch.device(device)
        sz = state_sizes(cfg)
        self.t = {}
        for name in STATE_FIELDS:
            nbytes = getattr(sz, name)
            dt = _DTYPE[name]
            n = max(1, nbytes // torch.tensor([], dtype=dt).element_size())
            if name in ("host_k", "host_v"):
                self.t[name] = (torch.empty(n, dtype=dt, pin_memory=True) if offload else None)
            else:
                self.t[name] = torch.empty(n, dtype=dt, device=self.device)
        # the state's own device, with its index (the buffers of every call must be there)
        self.device = self.t["seq_len"].device
        self.ws_bytes = workspace_size(cfg)
        self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device=self.device)
        workspace_init(self.ws, self.ws_bytes)
        self.state = nosa_state(*[(self.t[n].data_ptr() if self.t[n] is not None else None)
                                  for n in STATE_FIELDS])
        self._bytes = buffer_bytes(cfg)

    def _check(self, **bufs):
        for name, t in bufs.items():
            check_buffer(name, t, self._bytes[name], self.device)

    # views in the documented layouts
    def pool_view(self, name: str) -> torch.Tensor:
        c = self.cfg
        G = c.B * c.Hkv
        pages = c.max_blocks if name.startswith("host") else c.slots
        return self.t[name].view(G, pages, c.block_size, c.d)

    def init(self, prefill_len: torch.Tensor, resident: Optional[torch.Tensor] = None, stream=None):
        self._check(prefill_len=prefill_len, resident=resident)
        state_init(self.cfg, self.state, prefill_len, resident, self.ws, self.ws_bytes, stream)

    def append(self, k_new, v_new, stream=None):
        self._check(k_new=k_new, v_new=v_new)
        append(self.cfg, self.state, k_new, v_new, stream)

    def score_blocks(self, rows, block_scores, stream=None):
        self._check(score_rows=rows, block_scores=block_scores)
        score_blocks(self.cfg, self.state, rows, block_scores, stream)

    def select(self, block_scores, evict, sel, stream=None):
        self._check(block_scores=block_scores, evict=evict, sel=sel)
        select(self.cfg, self.state, block_scores, evict, sel, stream)

    def gather(self, sel, miss_count, stream=None):
        self._check(sel=sel, miss_count=miss_count)
        gather(self.cfg, self.state, sel, miss_count, self.ws, self.ws_bytes, stream)

    def decode_attn(self, q, sel, out, stream=None):
        self._check(q=q, sel=sel, out=out)
        decode_attn(self.cfg, self.state, q, sel, out, self.ws, self.ws_bytes, stream)

    def step(self, q, k_new, v_new, evict, sel, out, miss_count, score_rows=None, stream=None,
             events=None):
        self._check(q=q, k_new=k_new, v_new=v_new, evict=evict, sel=sel, out=out,
                    miss_count=miss_count, score_rows=score_rows)
        step(self.cfg, self.state, q, score_rows, k_new, v_new, evict, sel, out, miss_count, self.ws,
             self.ws_bytes, stream, events)

    def plan_ahead(self, score_rows, evict, sel, miss_count, stream=None):
        self._check(score_rows=score_rows, evict=evict, sel=sel, miss_count=miss_count)
        plan_ahead(self.cfg, self.state, score_rows, evict, sel, miss_count, self.ws, self.ws_bytes,
                   stream)

    def prefetch(self, stream=None):
        prefetch(self.cfg, self.state, self.ws, self.ws_bytes, stream)

    def attend(self, q, k_new, v_new, sel, out, stream=None):
        self._check(q=q, k_new=k_new, v_new=v_new, sel=sel, out=out)
        attend(self.cfg, self.state, q, k_new, v_new, sel, out, self.ws, self.ws_bytes, stream)

    def stop_counts(self, used, stream=None):
        self._check(used=used)
        stop_counts(self.cfg, self.ws, self.ws_bytes, used, stream)

    def check(self, stream=None):
        return check_device(self.state, stream)
