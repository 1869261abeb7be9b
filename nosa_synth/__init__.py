"""Seeded synthetic inputs for the NOSA sparse-decode step.

Shared by the tests, the benchmark and the oracle. Nothing here computes any
part of the method (pooling, selection, residency or attention): it only draws
random numbers and shapes them into the workloads the pages describe
(GQA attention layers at Llama-3.1-8B shape, 128K-token offload, sink keys).

The C part (``synth.c``) is built by :func:`build` into ``libnosa_synth.so``
next to this file.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass, field, replace
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "libnosa_synth.so")
_SRC = os.path.join(_HERE, "synth.c")

# stream ids (tensor field of the counter key)
T_K, T_V, T_Q, T_KNEW, T_VNEW, T_EVICT, T_PLANT, T_SINK, T_RESID, T_DRIFT, T_FCAST = range(1, 12)


def build(force: bool = False) -> str:
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-o", _SO, _SRC, "-lm"])
    return _SO


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_SO)
        u64, u32, i64, i32 = ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int64, ctypes.c_int32
        vp = ctypes.c_void_p
        L.synth_hash_u64.argtypes = [u64, u32, u32, u32, u32, u64, u64, vp]
        L.synth_uniform_f64.argtypes = [u64, u32, u32, u32, u32, u64, u64, vp]
        L.synth_gauss_f64.argtypes = [u64, u32, u32, u32, u32, u64, u64, vp]
        L.synth_round_bf16.argtypes = [vp, u64, vp]
        L.synth_round_f32.argtypes = [vp, u64, vp]
        L.synth_gauss_rows_bf16.argtypes = [u64, u32, u32, u32, u32, i64, i64, i32,
                                            ctypes.c_double, vp, vp, vp, i64]
        for f in (L.synth_hash_u64, L.synth_uniform_f64, L.synth_gauss_f64, L.synth_round_bf16,
                  L.synth_round_f32, L.synth_gauss_rows_bf16):
            f.restype = None
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def hashes(seed, tensor, a, b, c, n, i0=0) -> np.ndarray:
    out = np.empty(n, np.uint64)
    lib().synth_hash_u64(seed, tensor, a, b, c, i0, n, _p(out))
    return out


def uniform(seed, tensor, a, b, c, n, i0=0) -> np.ndarray:
    out = np.empty(n, np.float64)
    lib().synth_uniform_f64(seed, tensor, a, b, c, i0, n, _p(out))
    return out


def gauss(seed, tensor, a, b, c, n, i0=0) -> np.ndarray:
    out = np.empty(n, np.float64)
    lib().synth_gauss_f64(seed, tensor, a, b, c, i0, n, _p(out))
    return out


def round_bf16(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, np.float64)
    out = np.empty(x.shape, np.uint16)
    lib().synth_round_bf16(_p(x), x.size, _p(out))
    return out


def round_f32(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, np.float64)
    out = np.empty(x.shape, np.float32)
    lib().synth_round_f32(_p(x), x.size, _p(out))
    return out


def bf16_to_f64(u: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns."""
    return (u.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# --------------------------------------------------------------------------- configs


@dataclass(frozen=True)
class NosaConfig:
    """One workload of the decode step (shapes, budgets and input recipe)."""
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    T: tuple            # prefill length per batch entry
    block: int
    sub_block: int
    k_q: int
    k_e: int
    steps: int
    recipe: str = "plain"      # plain | planted | sink
    ar_rho: float = 0.0        # AR(1) coefficient of the query process over steps
    drift: float = 0.0         # sd of the per-step random walk of eviction scores
    slots: int = 0             # HBM pages per group; 0 = every block resident in HBM
    resident_frac: float = 0.25
    n_score_rows: int = 0      # 0 = the G query heads of the group; 1 = one forecast row
    cfg_id: int = 0
    seed: int = 0
    n_planted: int = 8
    plant_shift: float = 1.5
    score_mode: int = 0        # scoring variant bits: 1 overlapping windows, 2 per-row softmax
    stop_tau: float = 0.0      # S2O early stop threshold on gain / mass (0: attend every block)
    kc_bf16: int = 0           # 1: sub-block mean keys stored as bf16

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def k(self) -> int:
        return self.k_q + self.k_e

    @property
    def rows(self) -> int:
        return self.n_score_rows or self.G

    @property
    def max_blocks(self) -> int:
        return -(-(max(self.T) + self.steps) // self.block)

    @property
    def max_sub(self) -> int:
        return self.max_blocks * (self.block // self.sub_block)

    @property
    def offload(self) -> bool:
        return self.slots > 0

    @property
    def n_slots(self) -> int:
        return self.slots if self.slots else self.max_blocks

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def with_(self, **kw) -> "NosaConfig":
        if "T" in kw and isinstance(kw["T"], int):
            kw["T"] = (kw["T"],) * kw.get("B", self.B)
        return replace(self, **kw)


def _T(B, T):
    return tuple([T] * B) if isinstance(T, int) else tuple(T)


def sweep_points():
    pts = []
    i = 0
    for T in (8192, 65536):
        for bs in (32, 64, 128):
            for pct in (1, 5, 10):
                n = T // bs
                k = max(4, -(-pct * n // 100))
                k_e = (3 * k * 2 + 4) // 8  # floor(0.75 k + 0.5)
                k_q = k - k_e
                pts.append(NosaConfig(f"sweep_T{T}_b{bs}_p{pct}", 8, 32, 8, 128, _T(8, T), bs, 16,
                                      k_q, k_e, 16, cfg_id=100 + i))
                i += 1
    return pts


def configs() -> dict:
    c = {}
    c["tiny"] = NosaConfig("tiny", 1, 8, 2, 64, _T(1, 4096), 64, 16, 8, 8, 8, cfg_id=1)
    c["llama"] = NosaConfig("llama", 16, 32, 8, 128, _T(16, 32768), 64, 16, 16, 48, 32,
                            recipe="planted", ar_rho=0.95, cfg_id=2)
    c["offload"] = NosaConfig("offload", 4, 32, 8, 128, _T(4, 131072), 64, 16, 32, 96, 64,
                              drift=0.05, slots=512, cfg_id=3)
    c["sink"] = NosaConfig("sink", 64, 16, 4, 128, _T(64, 16384), 64, 16, 8, 24, 16,
                           recipe="sink", cfg_id=4)
    for p in sweep_points():
        c[p.name] = p
    # variants pinned to closed forms or used for fast parity
    c["tiny_dense"] = c["tiny"].with_(name="tiny_dense", k_q=57, cfg_id=11)
    c["tiny_static"] = c["tiny"].with_(name="tiny_static", T=(4000,), cfg_id=12)
    c["tiny_forecast"] = c["tiny"].with_(name="tiny_forecast", n_score_rows=1, cfg_id=13)
    c["llama_small"] = c["llama"].with_(name="llama_small", B=2, T=(4096, 4096), steps=6, cfg_id=21)
    c["offload_small"] = c["offload"].with_(name="offload_small", B=1, Hq=8, Hkv=2, T=(16384,),
                                            k_q=8, k_e=24, slots=64, steps=12, cfg_id=31)
    c["sink_small"] = c["sink"].with_(name="sink_small", B=4, T=(2048,) * 4, steps=4, cfg_id=41)
    c["ragged"] = NosaConfig("ragged", 3, 8, 2, 128, (1000, 4096, 37), 32, 16, 6, 10, 5,
                             cfg_id=51)
    c["ragged_offload"] = NosaConfig("ragged_offload", 3, 8, 2, 128, (1000, 4096, 37), 32, 16, 6,
                                     10, 6, slots=40, drift=0.05, cfg_id=52)
    c["empty"] = NosaConfig("empty", 2, 4, 1, 64, (0, 33), 32, 16, 2, 2, 70, cfg_id=53)
    c["bs128_d64"] = NosaConfig("bs128_d64", 2, 16, 2, 64, (3000, 2900), 128, 16, 3, 5, 4,
                                recipe="sink", cfg_id=54)
    c["g8"] = NosaConfig("g8", 2, 16, 2, 128, (1500, 1537), 64, 32, 5, 6, 3, cfg_id=55)
    # query-agnostic set only (k_q = 0) from a prefill shorter than k_e blocks that ends on a
    # block boundary: Gamma_e falls short while new blocks appear, and the query-aware set
    # fills S(t) up to k
    c["short_kq0"] = NosaConfig("short_kq0", 2, 8, 2, 64, (64, 96), 32, 16, 0, 5, 120, cfg_id=56)
    c["short_kq0_offload"] = c["short_kq0"].with_(name="short_kq0_offload", steps=250, slots=8,
                                                  drift=0.05, cfg_id=57)
    # lookahead (SparDA order: select from the forecast row, then append, then attend)
    c["lookahead"] = c["offload"].with_(name="lookahead", n_score_rows=1, cfg_id=61)
    c["lookahead_small"] = c["offload_small"].with_(name="lookahead_small", n_score_rows=1,
                                                    cfg_id=62)
    c["lookahead_hbm"] = c["llama_small"].with_(name="lookahead_hbm", n_score_rows=1, cfg_id=63)
    c["lookahead_ragged"] = c["ragged_offload"].with_(name="lookahead_ragged", n_score_rows=1,
                                                      cfg_id=64)
    c["lookahead_tiny"] = c["tiny"].with_(name="lookahead_tiny", n_score_rows=1, cfg_id=65)
    c["lookahead_dense"] = c["tiny"].with_(name="lookahead_dense", n_score_rows=1, k_q=57,
                                           cfg_id=66)
    # scoring variants: overlapping (2s, s) windows, per-row softmax then sum, both
    for m, tag in ((1, "window"), (2, "softmax"), (3, "window_softmax")):
        c[f"tiny_{tag}"] = c["tiny"].with_(name=f"tiny_{tag}", score_mode=m, cfg_id=70 + m)
        c[f"ragged_{tag}"] = c["ragged_offload"].with_(name=f"ragged_{tag}", score_mode=m,
                                                       cfg_id=73 + m)
        c[f"llama_small_{tag}"] = c["llama_small"].with_(name=f"llama_small_{tag}", score_mode=m,
                                                         cfg_id=76 + m)
    c["llama_window"] = c["llama"].with_(name="llama_window", score_mode=1, cfg_id=81)
    c["llama_softmax"] = c["llama"].with_(name="llama_softmax", score_mode=2, cfg_id=82)
    c["forecast_softmax"] = c["tiny_forecast"].with_(name="forecast_softmax", score_mode=2,
                                                     cfg_id=83)
    # S2O early stop over the selected blocks, visited in decreasing block score
    c["tiny_stop"] = c["tiny"].with_(name="tiny_stop", stop_tau=0.1, cfg_id=85)
    c["tiny_dense_stop"] = c["tiny_dense"].with_(name="tiny_dense_stop", stop_tau=0.03, cfg_id=86)
    c["ragged_stop"] = c["ragged_offload"].with_(name="ragged_stop", stop_tau=0.1, cfg_id=87)
    c["llama_small_stop"] = c["llama_small"].with_(name="llama_small_stop", stop_tau=0.02, cfg_id=88)
    c["llama_stop"] = c["llama"].with_(name="llama_stop", stop_tau=0.02, cfg_id=89)
    # bf16 sub-block mean keys (half the score kernel's bytes)
    c["tiny_kc16"] = c["tiny"].with_(name="tiny_kc16", kc_bf16=1, cfg_id=93)
    c["ragged_kc16"] = c["ragged_offload"].with_(name="ragged_kc16", kc_bf16=1, cfg_id=94)
    c["llama_small_kc16"] = c["llama_small"].with_(name="llama_small_kc16", kc_bf16=1, cfg_id=95)
    c["g8_kc16"] = c["g8"].with_(name="g8_kc16", kc_bf16=1, score_mode=3, cfg_id=96)
    c["bs128_d64_kc16"] = c["bs128_d64"].with_(name="bs128_d64_kc16", kc_bf16=1, cfg_id=97)
    c["llama_kc16"] = c["llama"].with_(name="llama_kc16", kc_bf16=1, cfg_id=98)
    return c


# --------------------------------------------------------------------------- inputs


@dataclass
class Inputs:
    """Raw inputs of a config: prefill pages, initial residency and per-step tensors."""
    cfg: NosaConfig
    pool_k: np.ndarray          # uint16 [B][Hkv][max_blocks*block][d]; rows >= T are zero
    pool_v: np.ndarray
    resident: Optional[np.ndarray]  # uint8 [B][Hkv][max_blocks] initial HBM residency, or None
    evict: np.ndarray           # float32 [steps][B][Hkv][max_blocks]
    k_new: np.ndarray           # uint16 [steps][B][Hkv][d]
    v_new: np.ndarray
    fcast_base: Optional[np.ndarray] = None
    _q_state: dict = field(default_factory=dict)
    sink_mu: Optional[np.ndarray] = None


def _q_z(cfg: NosaConfig, t: int, b: int, h: int, retry: int) -> np.ndarray:
    return gauss(cfg.seed, T_Q, cfg.cfg_id * 4096 + b, h, (t & 0xFFFFF) | (retry << 20), cfg.d)


def query_step(cfg: NosaConfig, t: int, prev: Optional[np.ndarray], retry: np.ndarray):
    """Query rows at step t (fp64 state [B][Hq][d]) for per-group retry counters [B][Hkv].

    q_0 = z_0; q_t = rho * q_{t-1} + sqrt(1 - rho^2) * z_t. The stored input is bf16(q_t).
    """
    B, Hq, G, d = cfg.B, cfg.Hq, cfg.G, cfg.d
    st = np.empty((B, Hq, d), np.float64)
    a = cfg.ar_rho
    c = math.sqrt(max(0.0, 1.0 - a * a))
    for b in range(B):
        for h in range(Hq):
            z = _q_z(cfg, t, b, h, int(retry[b, h // G]))
            st[b, h] = z if (prev is None or t == 0) else a * prev[b, h] + c * z
    return st


def forecast_step(cfg: NosaConfig, t: int, retry: np.ndarray) -> np.ndarray:
    """One forecast row per group (SparDA's compact indexer input), fp64 [B][Hkv][d]."""
    out = np.empty((cfg.B, cfg.Hkv, cfg.d))
    for b in range(cfg.B):
        for g in range(cfg.Hkv):
            out[b, g] = gauss(cfg.seed, T_FCAST, cfg.cfg_id * 4096 + b, g,
                              (t & 0xFFFFF) | (int(retry[b, g]) << 20), cfg.d)
    return out


def _unit(v):
    return v / np.linalg.norm(v)


def make_inputs(cfg: NosaConfig, with_pools: bool = True) -> Inputs:
    B, Hkv, d, bs, G = cfg.B, cfg.Hkv, cfg.d, cfg.block, cfg.G
    nb = cfg.max_blocks
    cap = nb * bs
    L = lib()
    pool_k = np.zeros((B, Hkv, cap, d), np.uint16) if with_pools else None
    pool_v = np.zeros((B, Hkv, cap, d), np.uint16) if with_pools else None
    sink_mu = None
    if cfg.recipe == "sink":
        sink_mu = np.stack([0.5 * math.sqrt(d) * _unit(gauss(cfg.seed, T_SINK, cfg.cfg_id, g, 0, d))
                            for g in range(Hkv)])
    q0 = None
    if cfg.recipe == "planted":
        q0 = query_step(cfg, 0, None, np.zeros((B, Hkv), np.int64))
    for b in range(B):
        T = cfg.T[b]
        n0 = -(-T // bs)
        for g in range(Hkv):
            offs, row_off = None, None
            if cfg.recipe == "planted" and T > 0:
                u = _unit(q0[b, g * G:(g + 1) * G].sum(0))
                offs = np.ascontiguousarray((cfg.plant_shift * u)[None, :])
                hh = hashes(cfg.seed, T_PLANT, cfg.cfg_id * 4096 + b, g, 0, n0)
                planted = np.argsort(hh, kind="stable")[:min(cfg.n_planted, n0)]
                row_off = np.full(T, -1, np.int8)
                for j in planted:
                    row_off[j * bs:min((j + 1) * bs, T)] = 0
            elif cfg.recipe == "sink" and T > 0:
                offs = np.ascontiguousarray(np.stack([sink_mu[g], -4.0 * sink_mu[g]]))
                row_off = np.zeros(T, np.int8)
                row_off[0] = 1
            if with_pools and T > 0:
                for arr, tid in ((pool_k, T_K), (pool_v, T_V)):
                    use_off = tid == T_K and offs is not None
                    L.synth_gauss_rows_bf16(cfg.seed, tid, cfg.cfg_id * 4096 + b, g, 0, 0, T, d, 1.0,
                                            _p(offs) if use_off else None,
                                            _p(row_off) if use_off else None,
                                            arr[b, g].ctypes.data_as(ctypes.c_void_p), d)
    # new tokens
    S = cfg.steps
    k_new = np.empty((S, B, Hkv, d), np.uint16)
    v_new = np.empty((S, B, Hkv, d), np.uint16)
    for t in range(S):
        for b in range(B):
            for g in range(Hkv):
                zk = gauss(cfg.seed, T_KNEW, cfg.cfg_id * 4096 + b, g, t, d)
                if sink_mu is not None:
                    zk = zk + sink_mu[g]
                k_new[t, b, g] = round_bf16(zk)
                v_new[t, b, g] = round_bf16(gauss(cfg.seed, T_VNEW, cfg.cfg_id * 4096 + b, g, t, d))
    # eviction scores: U(0,1) per block, optionally drifting by N(0, drift^2) per step
    ev = np.empty((S, B, Hkv, nb), np.float32)
    for b in range(B):
        for g in range(Hkv):
            e = uniform(cfg.seed, T_EVICT, cfg.cfg_id * 4096 + b, g, 0, nb)
            for t in range(S):
                if t > 0 and cfg.drift:
                    e = e + cfg.drift * gauss(cfg.seed, T_DRIFT, cfg.cfg_id * 4096 + b, g, t, nb)
                ev[t, b, g] = round_f32(e)
    resident = None
    if cfg.offload:
        resident = np.zeros((B, Hkv, nb), np.uint8)
        for b in range(B):
            T = cfg.T[b]
            n0 = -(-T // bs)
            if n0 == 0:
                continue
            tail = n0 - 1
            n_init = min(int(math.ceil(cfg.resident_frac * n0)), cfg.slots - 2, n0 - 1)
            for g in range(Hkv):
                hh = hashes(cfg.seed, T_RESID, cfg.cfg_id * 4096 + b, g, 0, n0 - 1)
                pick = np.argsort(hh, kind="stable")[:n_init]
                resident[b, g, pick] = 1
                resident[b, g, tail] = 1
    return Inputs(cfg, pool_k, pool_v, resident, ev, k_new, v_new, sink_mu=sink_mu)
