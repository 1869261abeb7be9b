"""fp64 CPU oracle of the NOSA sparse-decode step.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``__graft_entry__.smoke()``
and by ``bench.py``'s CPU-baseline / reference leg, never by the product
package. It shares no code with the CUDA library; the only thing both sides use
is the input generator in ``nosa_synth`` (random numbers, no method arithmetic).

``nosa_oracle.c`` holds the arithmetic (see its header for the passages it
follows); this module loads it with ctypes, keeps the oracle's state in numpy
arrays, and builds margin-checked test cases (:func:`run_case`).

Parity status: every oracle function is pinned by ``tests/test_oracle_pins.py``
(library routines, brute force, closed forms, invariants and a hand-worked
example); none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import shutil
import subprocess
from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np

import nosa_synth as syn

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nosa_oracle.c")
_SO = os.path.join(_HERE, "libnosa_oracle.so")

MARGIN = 1e-3  # score margin required at the query-aware cut
STOP_MARGIN = 1e-3   # early stop: relative distance of every gain/mass ratio from tau
ORDER_MARGIN = 2e-5  # early stop: score gap between blocks adjacent in the visiting order


def compile_oracle(src: str, out: str) -> str:
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", out,
                           src, "-lm"])
    return out


def build(force: bool = False) -> str:
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        compile_oracle(_SRC, _SO)
    return _SO


class OrcCfg(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("B", "Hq", "Hkv", "d", "bs", "s", "k_q", "k_e", "n_rows", "max_blocks", "slots",
                 "offload", "score_mode", "kc_bf16")] + [("scale", ctypes.c_double)]


class OrcState(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("K", "V", "kbar", "len", "prev_sel", "alive", "block_slot", "slot_owner",
                 "last_used")]


_libs = {}


def load(path: Optional[str] = None):
    path = path or build()
    if path not in _libs:
        L = ctypes.CDLL(path)
        vp = ctypes.c_void_p
        L.orc_topm.argtypes = [ctypes.c_int, vp, vp, ctypes.c_int, vp, vp]
        L.orc_topm.restype = ctypes.c_int
        L.orc_init.argtypes = [vp, vp, vp, vp]
        L.orc_init.restype = ctypes.c_int
        L.orc_append.argtypes = [vp, vp, vp, vp]
        L.orc_append.restype = None
        L.orc_block_scores.argtypes = [vp, vp, vp, vp, vp]
        L.orc_block_scores.restype = None
        L.orc_select.argtypes = [vp, vp, vp, vp, vp, vp, vp, ctypes.c_int, vp]
        L.orc_select.restype = None
        L.orc_residency.argtypes = [vp, vp, vp, vp]
        L.orc_residency.restype = ctypes.c_int
        L.orc_attend.argtypes = [vp, vp, vp, vp, vp]
        L.orc_attend.restype = None
        L.orc_attend_stop.argtypes = [vp, vp, vp, vp, vp, ctypes.c_double, vp, vp, vp, vp]
        L.orc_attend_stop.restype = None
        _libs[path] = L
    return _libs[path]


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def topm(key: np.ndarray, cand: np.ndarray, m: int, lib=None):
    """Top-m of key over cand (ties to the lower index): (chosen uint8, gap)."""
    L = lib or load()
    key = np.ascontiguousarray(key, np.float64)
    cand = np.ascontiguousarray(cand, np.uint8)
    ch = np.zeros(key.size, np.uint8)
    gap = np.zeros(1, np.float64)
    L.orc_topm(key.size, _p(key), _p(cand), m, _p(ch), _p(gap))
    return ch, float(gap[0])


class Oracle:
    """Oracle state for one configuration, advanced step by step."""

    def __init__(self, cfg: syn.NosaConfig, pool_k: np.ndarray, pool_v: np.ndarray,
                 resident: Optional[np.ndarray] = None, lib_path: Optional[str] = None,
                 copy: bool = True):
        self.cfg = cfg
        self.L = load(lib_path)
        c = cfg
        NG, nb = c.B * c.Hkv, c.max_blocks
        self.c = OrcCfg(c.B, c.Hq, c.Hkv, c.d, c.block, c.sub_block, c.k_q, c.k_e, c.rows, nb,
                        c.n_slots, int(c.offload), int(c.score_mode), int(c.kc_bf16), c.scale)
        # copy=False: the oracle appends into the caller's arrays (rows >= T change)
        self.K = np.ascontiguousarray(pool_k)
        self.V = np.ascontiguousarray(pool_v)
        if copy:
            self.K, self.V = self.K.copy(), self.V.copy()
        self.kbar = np.zeros((NG, c.max_sub, c.d), np.float64)
        self.len = np.zeros(NG, np.int32)
        self.prev_sel = np.zeros((NG, nb), np.uint8)
        self.alive = np.zeros((NG, nb), np.uint8)
        self.block_slot = np.full((NG, nb), -1, np.int32)
        self.slot_owner = np.full((NG, c.n_slots), -1, np.int32)
        self.last_used = np.zeros((NG, nb), np.int32)
        self.st = OrcState(*[_p(a) for a in (self.K, self.V, self.kbar, self.len, self.prev_sel,
                                              self.alive, self.block_slot, self.slot_owner,
                                              self.last_used)])
        T = np.ascontiguousarray(np.array(c.T, np.int32))
        res = None if resident is None else np.ascontiguousarray(resident, np.uint8)
        rc = self.L.orc_init(ctypes.byref(self.c), ctypes.byref(self.st), _p(T), _p(res))
        if rc != 0:
            raise ValueError(f"orc_init failed ({rc})")

    def append(self, k_new, v_new):
        self.L.orc_append(ctypes.byref(self.c), ctypes.byref(self.st),
                          _p(np.ascontiguousarray(k_new)), _p(np.ascontiguousarray(v_new)))

    def block_scores(self, rows: np.ndarray, out: Optional[np.ndarray] = None,
                     gmask: Optional[np.ndarray] = None) -> np.ndarray:
        c = self.cfg
        if out is None:
            out = np.empty((c.B * c.Hkv, c.max_blocks), np.float64)
        gm = None if gmask is None else np.ascontiguousarray(gmask, np.uint8)
        self.L.orc_block_scores(ctypes.byref(self.c), ctypes.byref(self.st),
                                _p(np.ascontiguousarray(rows)), _p(out), _p(gm))
        return out

    def select(self, scores, evict, commit=True, gmask=None, out=None):
        c = self.cfg
        NG = c.B * c.Hkv
        sel, src, gap = out if out is not None else (np.empty((NG, c.k), np.int32),
                                                      np.empty((NG, c.k), np.int8),
                                                      np.empty(NG, np.float64))
        gm = None if gmask is None else np.ascontiguousarray(gmask, np.uint8)
        self.L.orc_select(ctypes.byref(self.c), ctypes.byref(self.st),
                          _p(np.ascontiguousarray(scores, np.float64)),
                          _p(np.ascontiguousarray(evict, np.float32)), _p(sel), _p(src), _p(gap),
                          int(commit), _p(gm))
        return sel, src, gap

    def residency(self, sel):
        mc = np.zeros(self.cfg.B * self.cfg.Hkv, np.int32)
        rc = self.L.orc_residency(ctypes.byref(self.c), ctypes.byref(self.st),
                                  _p(np.ascontiguousarray(sel, np.int32)), _p(mc))
        if rc != 0:
            raise RuntimeError("oracle residency: no victim available")
        return mc

    def attend(self, q, sel):
        c = self.cfg
        out = np.empty((c.B, c.Hq, c.d), np.float64)
        self.L.orc_attend(ctypes.byref(self.c), ctypes.byref(self.st),
                          _p(np.ascontiguousarray(q)), _p(np.ascontiguousarray(sel, np.int32)),
                          _p(out))
        return out

    def attend_stop(self, q, sel, scores, tau):
        """S2O early-stop attention: (out, blocks used per head, decision margin per group,
        order gap per group); see orc_attend_stop."""
        c = self.cfg
        NG = c.B * c.Hkv
        out = np.empty((c.B, c.Hq, c.d), np.float64)
        used = np.empty((c.B, c.Hq), np.int32)
        mg, og = np.empty(NG), np.empty(NG)
        self.L.orc_attend_stop(ctypes.byref(self.c), ctypes.byref(self.st),
                               _p(np.ascontiguousarray(q)), _p(np.ascontiguousarray(sel, np.int32)),
                               _p(np.ascontiguousarray(scores, np.float64)), float(tau), _p(out),
                               _p(used), _p(mg), _p(og))
        return out, used, mg, og

    def snapshot(self) -> dict:
        return {k: getattr(self, k).copy() for k in
                ("len", "prev_sel", "alive", "block_slot", "slot_owner", "last_used")}


@dataclass
class StepRecord:
    q: np.ndarray               # uint16 [B][Hq][d]
    rows: np.ndarray            # uint16 [B][Hkv][R][d] scoring rows (q regrouped or forecast)
    forecast: Optional[np.ndarray]
    scores: np.ndarray          # fp64 [B*Hkv][max_blocks]
    sel: np.ndarray             # int32 [B*Hkv][k]
    src: np.ndarray             # int8
    gap: np.ndarray             # fp64 [B*Hkv]
    miss: np.ndarray            # int32 [B*Hkv]
    out: np.ndarray             # fp64 [B][Hq][d]
    retries: np.ndarray         # int [B][Hkv]
    state: dict = field(default_factory=dict)
    used: Optional[np.ndarray] = None   # int32 [B][Hq] blocks visited (early stop)


@dataclass
class Case:
    cfg: syn.NosaConfig
    inputs: syn.Inputs
    steps: List[StepRecord]


def _log_gap(scores, sel, src, gap):
    """The query-aware cut's margin in log units: softmax scores are probabilities of order
    1/M, so their absolute gaps say nothing about how safely fp32 ranks them; the ratio of
    the last selected to the first unselected score does."""
    out = np.array(gap, dtype=np.float64, copy=True)
    for gi in range(scores.shape[0]):
        if not np.isfinite(out[gi]):
            continue
        q = [int(j) for j, w in zip(sel[gi], src[gi]) if j >= 0 and w == 2]
        lo = min(scores[gi][j] for j in q)
        nxt = lo - out[gi]
        out[gi] = np.log(lo) - np.log(nxt) if nxt > 0 else np.inf
    return out


def run_case(cfg: syn.NosaConfig, steps: Optional[int] = None, margin: float = MARGIN,
             max_retry: int = 64, keep_state: bool = True, lib_path: Optional[str] = None,
             lookahead: bool = False) -> Case:
    """Generate a config's inputs and run the oracle over its steps.

    Margin enforcement: once the step's scores exist the query-aware cut of every
    group is checked; when the fp64 gap between the last selected and the first
    unselected block score is below `margin`, that group's query (or forecast)
    row is redrawn from the next retry stream. The final inputs are the ones
    recorded, so the GPU and the oracle consume identical arrays.

    lookahead: SparDA's decoupled order (gist.science/de/paper/2606.04511, section 2,
    "Trainierbare Lookahead Sparse-Selektion"): the blocks a step attends are chosen, and
    their residency planned, from the forecast row before the step's token is appended;
    the token is then appended and the query attends over the chosen blocks. Needs a
    forecast config (one scoring row per group) and a non-empty prefill.
    """
    if lookahead and cfg.n_score_rows != 1:
        raise ValueError("lookahead selection scores with the forecast row (n_score_rows == 1)")
    if lookahead and min(cfg.T) < 1:
        raise ValueError("lookahead needs a non-empty prefill")
    if lookahead and cfg.stop_tau > 0:
        raise ValueError("early stop is defined on the standard step order")
    inp = syn.make_inputs(cfg)
    # the oracle appends in place: inp.pool_k / pool_v rows >= T then hold the decode tokens
    orc = Oracle(cfg, inp.pool_k, inp.pool_v, inp.resident, lib_path, copy=False)
    S = cfg.steps if steps is None else steps
    G, R = cfg.G, cfg.rows
    prev = None
    recs = []
    for t in range(S):
        if not lookahead:
            orc.append(inp.k_new[t], inp.v_new[t])
        retry = np.zeros((cfg.B, cfg.Hkv), np.int64)
        todo = np.ones(cfg.B * cfg.Hkv, np.uint8)
        scores = np.empty((cfg.B * cfg.Hkv, cfg.max_blocks), np.float64)
        prev_out = (np.empty((cfg.B * cfg.Hkv, cfg.k), np.int32),
                    np.empty((cfg.B * cfg.Hkv, cfg.k), np.int8), np.empty(cfg.B * cfg.Hkv))
        while True:
            qs = syn.query_step(cfg, t, prev, retry)
            q16 = syn.round_bf16(qs)
            fc = None
            if cfg.n_score_rows == 1:
                fc = syn.round_bf16(syn.forecast_step(cfg, t, retry))
                rows = fc.reshape(cfg.B, cfg.Hkv, 1, cfg.d)
            else:
                rows = q16.reshape(cfg.B, cfg.Hkv, G, cfg.d)
            orc.block_scores(rows, out=scores, gmask=todo)
            sel_t, src_t, gap = orc.select(scores, inp.evict[t], commit=False, gmask=todo, out=prev_out)
            if cfg.score_mode & 2:
                gap = _log_gap(scores, sel_t, src_t, gap)
            bad = (gap < margin) & (todo != 0)
            if cfg.stop_tau > 0:
                # early stop: every stop decision must sit clearly on one side of tau, and
                # the visiting order must not hinge on near-equal scores
                _, _, dm, og = orc.attend_stop(q16, sel_t, scores, cfg.stop_tau)
                bad |= ((dm < STOP_MARGIN) | (og < ORDER_MARGIN)) & (todo != 0)
            if not bad.any():
                break
            bad2 = bad.reshape(cfg.B, cfg.Hkv)
            if (retry[bad2] >= max_retry).any():
                raise RuntimeError(f"{cfg.name}: no query with margin {margin} at step {t}")
            retry[bad2] += 1
            todo = bad.astype(np.uint8)
        prev = qs
        sel, src, gap = orc.select(scores, inp.evict[t], commit=True)
        miss = orc.residency(sel)
        if lookahead:
            orc.append(inp.k_new[t], inp.v_new[t])
        used = None
        if cfg.stop_tau > 0:
            out, used, _, _ = orc.attend_stop(q16, sel, scores, cfg.stop_tau)
        else:
            out = orc.attend(q16, sel)
        recs.append(StepRecord(q16, np.ascontiguousarray(rows), fc, scores, sel, src, gap, miss, out,
                               retry, orc.snapshot() if keep_state else {}, used))
    case = Case(cfg, inp, recs)
    case.oracle = orc
    return case
