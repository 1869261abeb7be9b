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
                                 dict(stop_tau=-1.0)])
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
