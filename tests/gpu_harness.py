"""Runs oracle-generated cases through the CUDA library and compares the results.

Everything here marshals arrays; the arithmetic under test is in libnosa.so
and the expected values come from the fp64 oracle on the same seeded inputs.
"""
from __future__ import annotations

import numpy as np
import torch

import kv_cache_offload_nosa_b200 as nosa
import nosa_synth as syn

ATOL = 2e-3      # max-abs error of the attention output vs fp64
RTOL_L2 = 1e-3   # relative L2 error of the attention output vs fp64


def c_config(cfg: syn.NosaConfig, attn_split: int = 0) -> nosa.nosa_config:
    return nosa.make_config(cfg.B, cfg.Hq, cfg.Hkv, cfg.d, cfg.block, cfg.sub_block, cfg.k_q, cfg.k_e,
                            cfg.max_blocks, slots=cfg.n_slots, n_score_rows=cfg.rows,
                            attn_split=attn_split, scale=cfg.scale, score_mode=cfg.score_mode,
                            stop_tau=cfg.stop_tau, kc_bf16=cfg.kc_bf16)


def dev(a: np.ndarray) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a))
    if t.dtype == torch.uint16:
        t = t.view(torch.int16)
    if t.dtype == torch.uint8:
        pass
    return t.cuda()


def setup(cfg: syn.NosaConfig, inputs: syn.Inputs, attn_split: int = 0) -> nosa.NosaCache:
    cc = c_config(cfg, attn_split)
    cache = nosa.NosaCache(cc, offload=cfg.offload)
    NG = cfg.B * cfg.Hkv
    pk = torch.from_numpy(inputs.pool_k.reshape(NG, cfg.max_blocks, cfg.block, cfg.d)).view(torch.int16)
    pv = torch.from_numpy(inputs.pool_v.reshape(NG, cfg.max_blocks, cfg.block, cfg.d)).view(torch.int16)
    names = ("host_k", "host_v") if cfg.offload else ("k_pool", "v_pool")
    for name, src in zip(names, (pk, pv)):
        dst = cache.pool_view(name)
        dst.copy_(src)
        # rows past each prefill are zeroed (the oracle may have appended into the source)
        flat = dst.view(cfg.B, cfg.Hkv, cfg.max_blocks * cfg.block, cfg.d)
        for b in range(cfg.B):
            flat[b, :, cfg.T[b]:] = 0
    resident = dev(inputs.resident.reshape(NG, cfg.max_blocks)) if cfg.offload else None
    plen = dev(np.array(cfg.T, np.int32))
    cache.init(plen, resident)
    torch.cuda.synchronize()
    cache._plen, cache._res = plen, resident
    return cache


class StepIO:
    """Device buffers of one step's inputs and outputs."""

    def __init__(self, cfg: syn.NosaConfig):
        NG = cfg.B * cfg.Hkv
        self.sel = torch.empty(NG * cfg.k, dtype=torch.int32, device="cuda")
        self.out = torch.empty(cfg.B * cfg.Hq * cfg.d, dtype=torch.float32, device="cuda")
        self.miss = torch.empty(NG, dtype=torch.int32, device="cuda")
        self.scores = torch.empty(NG * cfg.max_blocks, dtype=torch.float32, device="cuda")


def run_step(cache, cfg, inputs, rec, t, io: StepIO, mode: str = "fused"):
    q = dev(rec.q)
    rows = dev(rec.rows) if cfg.n_score_rows == 1 else None
    kn, vn = dev(inputs.k_new[t]), dev(inputs.v_new[t])
    ev = dev(inputs.evict[t])
    if mode == "fused":
        cache.step(q, kn, vn, ev, io.sel, io.out, io.miss, score_rows=rows)
    elif mode == "events":
        # the profiling form of the step: events between its kernels, each kernel waiting for
        # the previous grid as a whole instead of per-group flags
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        for e in evs:
            e.record()  # torch creates the CUDA events when first recorded
        cache.step(q, kn, vn, ev, io.sel, io.out, io.miss, score_rows=rows, events=evs)
    elif mode == "lookahead":
        # SparDA order on one stream: select and plan from the forecast row, copy, then
        # append and attend
        cache.plan_ahead(rows if rows is not None else q, ev, io.sel, io.miss)
        cache.prefetch()
        cache.attend(q, kn, vn, io.sel, io.out)
    else:
        cache.append(kn, vn)
        cache.score_blocks(rows if rows is not None else q, io.scores)
        cache.select(io.scores, ev, io.sel)
        cache.gather(io.sel, io.miss)
        cache.decode_attn(q, io.sel, io.out)
    torch.cuda.synchronize()


def bits_to_flags(words: torch.Tensor, NG: int, nb: int) -> np.ndarray:
    w = words.cpu().numpy().view(np.uint32).reshape(NG, -1)
    bits = ((w[:, :, None] >> np.arange(32, dtype=np.uint32)) & 1).reshape(NG, -1)
    return bits[:, :nb].astype(np.uint8)


def out_errors(got: np.ndarray, want: np.ndarray):
    d = got.astype(np.float64) - want
    return float(np.abs(d).max()), float(np.linalg.norm(d) / max(np.linalg.norm(want), 1e-300))


def compare_step(cache, cfg, rec, io: StepIO, t: int, check_state: bool = True):
    NG = cfg.B * cfg.Hkv
    sel = io.sel.cpu().numpy().reshape(NG, cfg.k)
    assert np.array_equal(sel, rec.sel), f"{cfg.name} step {t}: sel differs\n{sel}\n{rec.sel}"
    out = io.out.cpu().numpy().reshape(cfg.B, cfg.Hq, cfg.d)
    mx, rl2 = out_errors(out, rec.out)
    assert mx <= ATOL and rl2 <= RTOL_L2, f"{cfg.name} step {t}: max-abs {mx:.3g}, rel-L2 {rl2:.3g}"
    miss = io.miss.cpu().numpy()
    assert np.array_equal(miss, rec.miss), f"{cfg.name} step {t}: miss {miss} vs {rec.miss}"
    if rec.used is not None:
        used = torch.empty(cfg.B * cfg.Hq, dtype=torch.int32, device="cuda")
        cache.stop_counts(used)
        used = used.cpu().numpy().reshape(cfg.B, cfg.Hq)
        assert np.array_equal(used, rec.used), f"{cfg.name} step {t}: blocks visited\n{used}\n{rec.used}"
    rc, err = cache.check()
    assert rc == nosa.NOSA_OK and err == 0, (rc, err)
    if check_state and rec.state:
        st = rec.state
        nb = cfg.max_blocks
        assert np.array_equal(cache.t["seq_len"].cpu().numpy(), st["len"])
        assert np.array_equal(bits_to_flags(cache.t["prev_sel"], NG, nb), st["prev_sel"])
        assert np.array_equal(bits_to_flags(cache.t["alive"], NG, nb), st["alive"])
        if cfg.offload:
            bt = cache.t["block_table"].cpu().numpy().reshape(NG, nb)
            base = (np.arange(NG) * cfg.slots)[:, None]
            slot = np.where(bt >= 0, bt - base, -1)
            assert np.array_equal(slot, st["block_slot"]), f"{cfg.name} step {t}: block table"
            assert np.array_equal(cache.t["slot_owner"].cpu().numpy().reshape(NG, cfg.slots),
                                  st["slot_owner"])
            assert np.array_equal(cache.t["last_used"].cpu().numpy().reshape(NG, nb), st["last_used"])
    return mx, rl2


def run_and_compare(case, mode="fused", attn_split=0, check_state=True):
    cfg = case.cfg
    cache = setup(cfg, case.inputs, attn_split)
    io = StepIO(cfg)
    worst = (0.0, 0.0)
    for t, rec in enumerate(case.steps):
        run_step(cache, cfg, case.inputs, rec, t, io, mode)
        e = compare_step(cache, cfg, rec, io, t, check_state)
        worst = (max(worst[0], e[0]), max(worst[1], e[1]))
    return cache, worst
