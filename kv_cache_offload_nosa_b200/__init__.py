"""Python binding of libnosa.so: one NOSA sparse-decode step on a B200.

Argument marshalling only. Every step of the path (append, pooled scoring,
dual selection, residency and UVA gather, split-K attention and combine) runs
in the CUDA kernels of ``libnosa.so``; there is no CPU or PyTorch fallback, and
loading fails loudly when the library is missing. PyTorch provides device
memory, pinned host memory and streams.

The function names mirror the C ABI of ``include/nosa.h``; tensors are passed
by their data pointers and must already have the documented dtype, shape and
placement.

What the step computes follows NOSA: Native and Offloadable Sparse Attention
(technical summary at gist.science/es/paper/2510.13602, "Metodologia" 1 and 2);
the lookahead calls (plan_ahead, prefetch, attend) follow SparDA's decoupled
selection (gist.science/de/paper/2606.04511, section 2) and the early stop
follows S2O's stopping rule (gist.science/it/paper/2602.22575).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libnosa.so")

NOSA_OK, NOSA_EINVAL, NOSA_ENOMEM, NOSA_ECUDA, NOSA_EDEVICE, NOSA_ETIMEOUT = range(6)
ERR_BLOCK_TABLE, ERR_SEL, ERR_NO_VICTIM, ERR_TIMEOUT, ERR_FULL, ERR_INIT = 1, 2, 4, 8, 16, 32

EXPORTS = ("nosa_state_sizes", "nosa_workspace_size", "nosa_workspace_init", "nosa_state_init",
           "nosa_append", "nosa_score_blocks", "nosa_select", "nosa_gather", "nosa_decode_attn",
           "nosa_step", "nosa_check_device", "nosa_status_string", "nosa_last_error",
           "nosa_decode_attn_noalloc", "nosa_uva_read_probe", "nosa_plan_ahead", "nosa_prefetch", "nosa_attend", "nosa_stop_counts",
           "nosa_step_launches", "nosa_step_geometry")


NOSA_SCORE_WINDOW, NOSA_SCORE_SOFTMAX = 1, 2


class nosa_config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("B", "Hq", "Hkv", "d", "block_size", "sub_block", "k_q", "k_e", "max_blocks",
                 "slots", "n_score_rows", "attn_split")] + [("scale", ctypes.c_float),
                                                             ("score_mode", ctypes.c_int32),
                                                             ("stop_tau", ctypes.c_float),
                                                             ("kc_bf16", ctypes.c_int32),
                                                             ("wait_us", ctypes.c_int32)]


STATE_FIELDS = ("seq_len", "kc", "prev_sel", "alive", "last_used", "block_table", "slot_owner",
                "k_pool", "v_pool", "host_k", "host_v", "err")


class nosa_state(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in STATE_FIELDS]


class nosa_sizes(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in STATE_FIELDS]


class NosaError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"nosa status {status}: {msg}")
        self.status = status


_lib = None


def load(path: Optional[str] = None):
    """Loads libnosa.so (raises if it is missing: there is no fallback)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise ImportError(f"libnosa.so not built at {p}; run kv_cache_offload_nosa_b200/build.py")
    L = ctypes.CDLL(p)
    vp, sz, i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
    cfgp, stp = ctypes.POINTER(nosa_config), ctypes.POINTER(nosa_state)
    sig = {
        "nosa_state_sizes": [cfgp, ctypes.POINTER(nosa_sizes)],
        "nosa_workspace_size": [cfgp, ctypes.POINTER(ctypes.c_size_t)],
        "nosa_workspace_init": [vp, sz, vp],
        "nosa_state_init": [cfgp, stp, vp, vp, vp, sz, vp],
        "nosa_append": [cfgp, stp, vp, vp, vp],
        "nosa_score_blocks": [cfgp, stp, vp, vp, vp],
        "nosa_select": [cfgp, stp, vp, vp, vp, vp],
        "nosa_gather": [cfgp, stp, vp, vp, vp, sz, vp],
        "nosa_decode_attn": [cfgp, stp, vp, vp, vp, vp, sz, vp],
        "nosa_step": [cfgp, stp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp, vp],
        "nosa_check_device": [stp, vp, ctypes.POINTER(ctypes.c_uint32)],
        "nosa_decode_attn_noalloc": [cfgp, stp, vp, vp, vp, vp],
        "nosa_uva_read_probe": [vp, vp, sz, i32, vp],
        "nosa_plan_ahead": [cfgp, stp, vp, vp, vp, vp, vp, sz, vp],
        "nosa_prefetch": [cfgp, stp, vp, sz, vp],
        "nosa_stop_counts": [cfgp, vp, sz, vp, vp],
        "nosa_attend": [cfgp, stp, vp, vp, vp, vp, vp, vp, sz, vp],
        "nosa_step_launches": [cfgp, stp, ctypes.POINTER(ctypes.c_int32)],
        "nosa_step_geometry": [cfgp, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, vp],
    }
    for name, args in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = i32
    L.nosa_status_string.argtypes = [i32]
    L.nosa_status_string.restype = ctypes.c_char_p
    L.nosa_last_error.argtypes = []
    L.nosa_last_error.restype = ctypes.c_char_p
    if path is None:
        _lib = L
    return L


def _check(rc: int):
    if rc != NOSA_OK:
        L = load()
        raise NosaError(rc, f"{L.nosa_status_string(rc).decode()}: {L.nosa_last_error().decode()}")


def _ptr(x) -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def make_config(B, Hq, Hkv, d, block_size, sub_block, k_q, k_e, max_blocks, slots=None,
                n_score_rows=None, attn_split=0, scale=None, score_mode=0, stop_tau=0.0,
                kc_bf16=0, wait_us=0) -> nosa_config:
    G = Hq // Hkv
    return nosa_config(B, Hq, Hkv, d, block_size, sub_block, k_q, k_e, max_blocks,
                       max_blocks if slots is None else slots, G if n_score_rows is None else n_score_rows,
                       attn_split, (1.0 / d ** 0.5) if scale is None else scale, score_mode, stop_tau,
                       kc_bf16, wait_us)


def state_sizes(cfg: nosa_config) -> nosa_sizes:
    s = nosa_sizes()
    _check(load().nosa_state_sizes(ctypes.byref(cfg), ctypes.byref(s)))
    return s


def workspace_size(cfg: nosa_config) -> int:
    n = ctypes.c_size_t()
    _check(load().nosa_workspace_size(ctypes.byref(cfg), ctypes.byref(n)))
    return n.value


def workspace_init(ws, nbytes: int, stream=None):
    _check(load().nosa_workspace_init(_ptr(ws), nbytes, _stream(stream)))


def state_init(cfg, st: nosa_state, prefill_len, resident, ws, ws_bytes, stream=None):
    _check(load().nosa_state_init(ctypes.byref(cfg), ctypes.byref(st), _ptr(prefill_len),
                                  _ptr(resident), _ptr(ws), ws_bytes, _stream(stream)))


def append(cfg, st, k_new, v_new, stream=None):
    _check(load().nosa_append(ctypes.byref(cfg), ctypes.byref(st), _ptr(k_new), _ptr(v_new),
                              _stream(stream)))


def score_blocks(cfg, st, rows, block_scores, stream=None):
    _check(load().nosa_score_blocks(ctypes.byref(cfg), ctypes.byref(st), _ptr(rows),
                                    _ptr(block_scores), _stream(stream)))


def select(cfg, st, block_scores, evict, sel, stream=None):
    _check(load().nosa_select(ctypes.byref(cfg), ctypes.byref(st), _ptr(block_scores), _ptr(evict),
                              _ptr(sel), _stream(stream)))


def gather(cfg, st, sel, miss_count, ws, ws_bytes, stream=None):
    _check(load().nosa_gather(ctypes.byref(cfg), ctypes.byref(st), _ptr(sel), _ptr(miss_count),
                              _ptr(ws), ws_bytes, _stream(stream)))


def decode_attn(cfg, st, q, sel, out, ws, ws_bytes, stream=None):
    _check(load().nosa_decode_attn(ctypes.byref(cfg), ctypes.byref(st), _ptr(q), _ptr(sel),
                                   _ptr(out), _ptr(ws), ws_bytes, _stream(stream)))


def decode_attn_noalloc(cfg, st, q, sel, out, stream=None):
    """nosa_decode_attn without a workspace (scratch in the library's static device array).

    For callers that cannot allocate device memory when attention runs; see include/nosa.h
    for the size limit and the rule that overlapping calls race on the shared scratch.
    """
    _check(load().nosa_decode_attn_noalloc(ctypes.byref(cfg), ctypes.byref(st), _ptr(q), _ptr(sel),
                                           _ptr(out), _stream(stream)))


def step(cfg, st, q, score_rows, k_new, v_new, evict, sel, out, miss_count, ws, ws_bytes,
         stream=None, events: Optional[Sequence] = None):
    ev = None
    if events is not None:
        ev = (ctypes.c_void_p * 4)(*[e.cuda_event if e is not None else None for e in events])
    _check(load().nosa_step(ctypes.byref(cfg), ctypes.byref(st), _ptr(q), _ptr(score_rows),
                            _ptr(k_new), _ptr(v_new), _ptr(evict), _ptr(sel), _ptr(out),
                            _ptr(miss_count), _ptr(ws), ws_bytes, _stream(stream), ev))


def uva_read_probe(host, dev, nbytes: int, ctas: int = 0, stream=None):
    """Measurement helper: copies nbytes of pinned host memory to device memory by 16-byte UVA
    loads (the gather's access); its time is the PCIe read ceiling of the gather."""
    _check(load().nosa_uva_read_probe(_ptr(host), _ptr(dev), nbytes, ctas, _stream(stream)))


def plan_ahead(cfg, st, score_rows, evict, sel, miss_count, ws, ws_bytes, stream=None):
    """Lookahead call 1: select and plan from score_rows on the cache as it stands."""
    _check(load().nosa_plan_ahead(ctypes.byref(cfg), ctypes.byref(st), _ptr(score_rows), _ptr(evict),
                                  _ptr(sel), _ptr(miss_count), _ptr(ws), ws_bytes, _stream(stream)))


def prefetch(cfg, st, ws, ws_bytes, stream=None):
    """Lookahead call 2: host -> HBM copies of the planned pages (no-op without host pools)."""
    _check(load().nosa_prefetch(ctypes.byref(cfg), ctypes.byref(st), _ptr(ws), ws_bytes, _stream(stream)))


def attend(cfg, st, q, k_new, v_new, sel, out, ws, ws_bytes, stream=None):
    """Lookahead call 3: append the token, attend over the blocks plan_ahead chose."""
    _check(load().nosa_attend(ctypes.byref(cfg), ctypes.byref(st), _ptr(q), _ptr(k_new), _ptr(v_new),
                              _ptr(sel), _ptr(out), _ptr(ws), ws_bytes, _stream(stream)))


def stop_counts(cfg, ws, ws_bytes, used, stream=None):
    """Blocks each query head visited in the last early-stop step ([B*Hq] int32, device)."""
    _check(load().nosa_stop_counts(ctypes.byref(cfg), _ptr(ws), ws_bytes, _ptr(used), _stream(stream)))


def step_launches(cfg, st) -> int:
    """Kernels nosa_step launches without events (1: the fused persistent step kernel)."""
    n = ctypes.c_int32()
    _check(load().nosa_step_launches(ctypes.byref(cfg), ctypes.byref(st), ctypes.byref(n)))
    return n.value


class nosa_geometry(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("score_chunk", "score_ctas", "attn_tasks_per_cta", "attn_ctas")]


def step_geometry(cfg, host_pools: bool, sms: int, attn_ctas_per_sm: int) -> dict:
    """Launch geometry nosa_step chooses on a GPU with `sms` SMs (no CUDA call)."""
    g = nosa_geometry()
    _check(load().nosa_step_geometry(ctypes.byref(cfg), int(bool(host_pools)), sms, attn_ctas_per_sm,
                                     ctypes.byref(g)))
    return {n: getattr(g, n) for n, _ in nosa_geometry._fields_}


def check_device(st, stream=None):
    """Synchronises; returns (status, error word) without raising."""
    e = ctypes.c_uint32()
    rc = load().nosa_check_device(ctypes.byref(st), _stream(stream), ctypes.byref(e))
    return rc, e.value


from .cache import NosaCache  # noqa: E402  (allocation helper on top of the ABI)
