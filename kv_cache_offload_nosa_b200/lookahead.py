"""SparDA lookahead pipeline across the attention layers of one decode token.

Host orchestration over the C ABI only: every step of the path runs in libnosa's kernels.
SparDA (gist.science/de/paper/2606.04511, section 2) selects the blocks layer l+1 will attend
from a forecast row produced one layer earlier, so that their host -> HBM copies overlap the
computation of the current layer ("Asynchrones Prefetching mit persistentem UVA-Kernel").

Per layer l of a token the pipeline issues, on three CUDA streams:
  plan stream     nosa_plan_ahead(l)   forecast scoring, dual selection, residency plan
  copy stream     nosa_prefetch(l)     the planned pages over UVA, after plan(l)
  compute stream  nosa_attend(l)       append + attention, after prefetch(l)
The order follows the data the forecast needs. Layer l's forecast row for layer l+1 comes
from layer l's input, which exists once layer l-1 has attended; so plan(l+1) waits for
attend(l-1) (the first two plans only for the token's inputs). Copies run layer after layer,
so PCIe does not idle between layers, and layer l attends while layer l+1's pages cross PCIe.
Every wait is on work that has already been issued, so no kernel occupies SMs spinning on a
kernel that cannot start.

The forecast rows are inputs here (no model weights): in a model, layer l's forecast
projection would produce layer l+1's rows from layer l's input.
"""
from __future__ import annotations

from typing import Sequence

import torch


class LookaheadPipeline:
    """Schedules nosa_plan_ahead / nosa_prefetch / nosa_attend of several layers' caches."""

    def __init__(self, caches: Sequence):
        self.caches = list(caches)
        self.plan_stream = torch.cuda.Stream()
        self.copy_stream = torch.cuda.Stream()
        n = len(self.caches)
        self.planned = [torch.cuda.Event() for _ in range(n)]
        self.copied = [torch.cuda.Event() for _ in range(n)]
        self.attended = [torch.cuda.Event() for _ in range(n)]

    def token(self, score_rows, evict, q, k_new, v_new, sel, miss, out, stream=None):
        """One decode token through every layer (per-layer sequences of device tensors).

        Asynchronous: the compute stream (`stream`, default the current one) holds every
        layer's `out`, `sel` and `miss` once it reaches the end of this call's work.
        """
        comp = stream if stream is not None else torch.cuda.current_stream()
        n = len(self.caches)
        # inputs are ready on the compute stream, and so is the previous token's attend of
        # every layer, which a layer's plan must follow (it reads the appended state)
        self.plan_stream.wait_stream(comp)

        def plan_and_copy(l):
            c = self.caches[l]
            c.plan_ahead(score_rows[l], evict[l], sel[l], miss[l], stream=self.plan_stream)
            self.planned[l].record(self.plan_stream)
            self.copy_stream.wait_event(self.planned[l])
            c.prefetch(stream=self.copy_stream)
            self.copied[l].record(self.copy_stream)

        # layer 0's and layer 1's forecast rows come from the token's input (layer 0's input)
        for l in range(min(2, n)):
            plan_and_copy(l)
        for l, c in enumerate(self.caches):
            comp.wait_event(self.copied[l])
            c.attend(q[l], k_new[l], v_new[l], sel[l], out[l], stream=comp)
            self.attended[l].record(comp)
            if l + 2 < n:
                # layer l+1's input (so its forecast row for layer l+2) exists after attend(l)
                self.plan_stream.wait_event(self.attended[l])
                plan_and_copy(l + 2)
