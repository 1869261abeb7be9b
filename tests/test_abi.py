"""The C-ABI library loads, exports what include/nosa.h declares, and validates on the host.

No kernel is launched here (CPU only).
"""
import ctypes
import os
import re

import pytest

import kv_cache_offload_nosa_b200 as nosa
from kv_cache_offload_nosa_b200 import build as nb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "nosa.h")


@pytest.fixture(scope="module")
def lib():
    nb.build()
    return nosa.load()


def declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(nosa_[a-z_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(lib):
    names = declared()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), n
    assert set(nosa.EXPORTS) <= set(names)


def cfg(**kw):
    base = dict(B=2, Hq=8, Hkv=2, d=128, block_size=64, sub_block=16, k_q=4, k_e=4, max_blocks=40)
    base.update(kw)
    return nosa.make_config(**base)


@pytest.mark.parametrize("bad", [dict(d=96), dict(block_size=48), dict(sub_block=24),
                                 dict(Hq=12, Hkv=4, ), dict(Hq=7), dict(k_q=0, k_e=0),
                                 dict(k_q=30, k_e=20), dict(max_blocks=9000), dict(slots=0),
                                 dict(n_score_rows=2), dict(scale=0.0), dict(sub_block=128),
                                 dict(score_mode=4), dict(score_mode=-1), dict(kc_bf16=2),
                                 dict(stop_tau=-1.0), dict(wait_us=-1), dict(wait_us=60000001)])
def test_bad_config_is_rejected_on_host(lib, bad):
    c = cfg(**bad)
    n = ctypes.c_size_t()
    rc = lib.nosa_workspace_size(ctypes.byref(c), ctypes.byref(n))
    assert rc == nosa.NOSA_EINVAL
    assert lib.nosa_last_error()


def test_sizes_follow_the_documented_layout(lib):
    c = cfg()
    s = nosa.state_sizes(c)
    NG, nb_, d, bs = 4, 40, 128, 64
    assert s.kc == NG * nb_ * (bs // 16) * d * 4
    assert s.prev_sel == NG * 2 * 4
    assert s.k_pool == NG * nb_ * bs * d * 2
    assert s.host_k == NG * nb_ * bs * d * 2
    assert nosa.workspace_size(c) > 0


def test_score_variants_reserve_their_values(lib):
    """Variants keep per-sub-block values in the workspace: one per sub-block for windows of
    the mean, one per scoring row and sub-block for softmax."""
    base = nosa.workspace_size(cfg())
    NG, max_sub = 4, 40 * 4
    win = nosa.workspace_size(cfg(score_mode=nosa.NOSA_SCORE_WINDOW))
    soft = nosa.workspace_size(cfg(score_mode=nosa.NOSA_SCORE_SOFTMAX))
    assert win - base >= NG * max_sub * 4
    assert soft - base >= NG * 4 * max_sub * 4      # G = 4 rows
    assert nosa.workspace_size(cfg(score_mode=3, n_score_rows=1)) - base >= NG * max_sub * 4


def test_bf16_kc_halves_its_buffer(lib):
    assert nosa.state_sizes(cfg(kc_bf16=1)).kc * 2 == nosa.state_sizes(cfg()).kc


def test_status_strings(lib):
    for code in range(6):
        assert lib.nosa_status_string(code)


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(ImportError):
        nosa.load(str(tmp_path / "libnosa.so"))


def test_every_synthetic_config_passes_the_library_checks(lib):
    """Each workload the tests and the benchmark run is one the library accepts (its config
    checks run on the host), and offload ones have the slots the state check asks for."""
    import nosa_synth as syn
    for name, c in syn.configs().items():
        cc = nosa.make_config(c.B, c.Hq, c.Hkv, c.d, c.block, c.sub_block, c.k_q, c.k_e, c.max_blocks,
                              slots=c.n_slots, n_score_rows=c.rows, scale=c.scale,
                              score_mode=c.score_mode, stop_tau=c.stop_tau, kc_bf16=c.kc_bf16)
        nosa.state_sizes(cc)
        assert nosa.workspace_size(cc) > 0, name
        if c.offload:
            assert c.k + 2 <= c.n_slots <= c.max_blocks, (name, c.k, c.n_slots, c.max_blocks)


class _AsCuda:
    """A CPU tensor that reports itself as a CUDA tensor (size checks only; nothing launches)."""

    def __init__(self, t, device=None):
        import torch
        self.t = t
        self.is_cuda = True
        self.device = device if device is not None else torch.device("cuda", 0)

    def is_contiguous(self):
        return self.t.is_contiguous()

    def numel(self):
        return self.t.numel()

    def element_size(self):
        return self.t.element_size()


@pytest.mark.parametrize("name", ["tiny", "tiny_forecast", "offload_small", "ragged_offload", "g8",
                                  "empty", "lookahead_tiny", "tiny_stop", "short_kq0"])
def test_cache_buffer_checks_accept_the_harness_buffers(name):
    """The NosaCache size checks accept every buffer the GPU tests pass, built the same way
    (the oracle's records and the synthetic inputs, viewed as the library's dtypes)."""
    import numpy as np
    import torch
    import nosa_synth as syn
    import oracle as O
    from kv_cache_offload_nosa_b200.cache import NosaCache, buffer_bytes
    cfg = syn.configs()[name]
    case = O.run_case(cfg, steps=2, lookahead=name.startswith("lookahead"))
    cc = nosa.make_config(cfg.B, cfg.Hq, cfg.Hkv, cfg.d, cfg.block, cfg.sub_block, cfg.k_q, cfg.k_e,
                          cfg.max_blocks, slots=cfg.n_slots, n_score_rows=cfg.rows, scale=cfg.scale,
                          score_mode=cfg.score_mode, stop_tau=cfg.stop_tau, kc_bf16=cfg.kc_bf16)
    cache = NosaCache.__new__(NosaCache)
    cache._bytes = buffer_bytes(cc)
    cache.device = torch.device("cuda", 0)

    def dev(a):
        t = torch.from_numpy(np.ascontiguousarray(a))
        return _AsCuda(t.view(torch.int16) if t.dtype == torch.uint16 else t)

    NG = cfg.B * cfg.Hkv
    sel = _AsCuda(torch.empty(NG * cfg.k, dtype=torch.int32))
    out = _AsCuda(torch.empty(cfg.B * cfg.Hq * cfg.d, dtype=torch.float32))
    miss = _AsCuda(torch.empty(NG, dtype=torch.int32))
    scores = _AsCuda(torch.empty(NG * cfg.max_blocks, dtype=torch.float32))
    inp, rec = case.inputs, case.steps[0]
    cache._check(prefill_len=dev(np.array(cfg.T, np.int32)),
                 resident=dev(inp.resident.reshape(NG, cfg.max_blocks)) if cfg.offload else None)
    cache._check(q=dev(rec.q), k_new=dev(inp.k_new[0]), v_new=dev(inp.v_new[0]),
                 evict=dev(inp.evict[0]), sel=sel, out=out, miss_count=miss,
                 score_rows=dev(rec.rows), block_scores=scores,
                 used=_AsCuda(torch.empty(cfg.B * cfg.Hq, dtype=torch.int32)))
    # too small, not on the device, not contiguous: refused before anything launches
    with pytest.raises(nosa.NosaError):
        cache._check(sel=_AsCuda(torch.empty(NG * cfg.k - 1, dtype=torch.int32)))
    with pytest.raises(nosa.NosaError):
        cache._check(out=torch.empty(cfg.B * cfg.Hq * cfg.d, dtype=torch.float32))
    with pytest.raises(nosa.NosaError):
        cache._check(q=_AsCuda(torch.empty(2 * cfg.B * cfg.Hq * cfg.d, dtype=torch.int16)[::2]))
    # the right size on another GPU: refused (its pointer is not the state's device's memory)
    with pytest.raises(nosa.NosaError, match="state is on"):
        cache._check(sel=_AsCuda(torch.empty(NG * cfg.k, dtype=torch.int32), torch.device("cuda", 1)))


def test_workspace_one_byte_short_is_refused_before_any_cuda_call(lib):
    """nosa_step with a workspace one byte below nosa_workspace_size returns NOSA_ENOMEM from
    its argument checks, before any CUDA call (the addresses are never dereferenced: no GPU
    is needed), and the reason names both sizes."""
    c = cfg()
    need = nosa.workspace_size(c)
    fake = [0x10000 * (i + 1) for i in range(12)]           # 16-byte aligned, never read
    st = nosa.nosa_state(*fake[:9], None, None, fake[9])   # no host pools: no pointer query
    args = [0x200000 + 0x1000 * i for i in range(7)]       # q, k_new, v_new, evict, sel, out, miss
    q, kn, vn, ev, sel, out, miss = args
    rc = lib.nosa_step(ctypes.byref(c), ctypes.byref(st), q, None, kn, vn, ev, sel, out, miss,
                       0x4000000, need - 1, None, None)
    assert rc == nosa.NOSA_ENOMEM
    msg = lib.nosa_last_error().decode()
    assert str(need) in msg and str(need - 1) in msg, msg


def test_step_launch_count_on_host(lib):
    """nosa_step_launches answers from the configuration and state alone (no GPU: the
    addresses are never dereferenced): every block in HBM -> 2 kernels (score + selection,
    attention); a NULL output or a bad configuration is refused."""
    c = cfg()
    fake = [0x10000 * (i + 1) for i in range(12)]
    st = nosa.nosa_state(*fake[:9], None, None, fake[9])
    assert nosa.step_launches(c, st) == 2
    n = ctypes.c_int32(-1)
    assert lib.nosa_step_launches(ctypes.byref(c), ctypes.byref(st), None) == nosa.NOSA_EINVAL
    bad = cfg()
    bad.k_q = bad.k_e = 0
    assert lib.nosa_step_launches(ctypes.byref(bad), ctypes.byref(st), ctypes.byref(n)) == nosa.NOSA_EINVAL
    assert n.value == -1


def _syn_config(name, **over):
    import nosa_synth as syn
    c = syn.configs()[name]
    kw = dict(slots=c.n_slots, n_score_rows=c.rows, scale=c.scale, score_mode=c.score_mode,
              stop_tau=c.stop_tau, kc_bf16=c.kc_bf16)
    kw.update(over)
    return c, nosa.make_config(c.B, c.Hq, c.Hkv, c.d, c.block, c.sub_block, c.k_q, c.k_e, c.max_blocks, **kw)


@pytest.mark.parametrize("name,host,want", [
    # Llama-shaped: 2052 sub-blocks per group in 6 chunks of 384; k = 64 in halves (one CTA per
    # resident slot: 296 slots, 256 CTAs)
    ("llama", False, dict(score_chunk=384, score_ctas=128 * 6, attn_tasks_per_cta=32, attn_ctas=256)),
    # sink: 1028 sub-blocks in 3 chunks; k = 32, 1 MB of pages per group: the divisor rule, W = 32
    ("sink", False, dict(score_chunk=384, score_ctas=256 * 3, attn_tasks_per_cta=32, attn_ctas=256)),
    # T = 65536, 1 %: k = 11 pages (352 KB) per group, 64 groups: one CTA per group
    ("sweep_T65536_b64_p1", False, dict(score_chunk=384, score_ctas=64 * 11, attn_tasks_per_cta=11, attn_ctas=64)),
    # k = 103 is prime and 3.4 MB per group: no divisor near a CTA per slot, W = ceil(6592 / 296)
    ("sweep_T65536_b64_p10", False, dict(score_chunk=384, score_ctas=64 * 11, attn_tasks_per_cta=23, attn_ctas=287)),
    # tiny: 2 groups, so at least ~3 score CTAs per SM in all means 5 chunks of 64 sub-blocks
    # (260 in all); the attention keeps the smallest width the 16 partial slots allow
    ("tiny", False, dict(score_chunk=64, score_ctas=2 * 5, attn_tasks_per_cta=2, attn_ctas=16)),
    # offload: 8196 sub-blocks in 22 chunks; with host pools the finest split, ceil(128 / 15)
    ("offload", True, dict(score_chunk=384, score_ctas=32 * 22, attn_tasks_per_cta=9, attn_ctas=456)),
    # early stop: one CTA per group
    ("llama_stop", False, dict(score_chunk=384, score_ctas=128 * 6, attn_tasks_per_cta=64, attn_ctas=128)),
])
def test_step_geometry(lib, name, host, want):
    """The launch geometry nosa_step picks on a B200 (148 SMs, two attention CTAs per SM),
    computed on the host from the configuration alone."""
    _, cc = _syn_config(name)
    assert nosa.step_geometry(cc, host, 148, 2) == want


def test_step_geometry_rules(lib):
    """An explicit split is kept; the score chunks cover every sub-block with at most 384 per
    CTA and are multiples of 64; bad arguments are refused."""
    c, cc = _syn_config("llama", attn_split=8)
    g = nosa.step_geometry(cc, False, 148, 2)
    assert g["attn_tasks_per_cta"] == 8 and g["attn_ctas"] == 128 * 64 // 8
    import nosa_synth as syn
    for name, s in syn.configs().items():
        _, cfg = _syn_config(name)
        g = nosa.step_geometry(cfg, s.offload, 148, 2)
        ch = g["score_chunk"]
        assert ch % 64 == 0 and 64 <= ch <= 384, (name, ch)
        per_group = g["score_ctas"] // (s.B * s.Hkv)
        assert (per_group - 1) * ch < s.max_sub <= per_group * ch, (name, ch, per_group)
        W = g["attn_tasks_per_cta"]
        assert g["attn_ctas"] == -(-s.B * s.Hkv * s.k // W), name
        assert -(-(s.k - 1) // W) + 1 <= 16, (name, W)  # a group spans at most 16 partial slots
    out = nosa.nosa_geometry()
    assert lib.nosa_step_geometry(ctypes.byref(cc), 0, 0, 2, ctypes.byref(out)) == nosa.NOSA_EINVAL
    assert lib.nosa_step_geometry(ctypes.byref(cc), 0, 148, 2, None) == nosa.NOSA_EINVAL
