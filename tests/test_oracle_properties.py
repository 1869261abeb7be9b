"""The oracle's pins, applied to configurations drawn across the shapes the library accepts.

The fixed workloads cover a handful of shapes; here a seeded (derandomized) hypothesis search
draws others: G in {1, 2, 4, 8}, d in {64, 128}, block size in {32, 64, 128} with every
sub-block size that divides it, ragged and empty prefills, budgets with k_q = 0 or k_e = 0,
host pools, forecast rows, the scoring variants, bf16 means and early stop. Every drawn
configuration must be one the C library accepts, and on each the oracle must meet the same
pins as on the fixed workloads: brute-force top-m of both sets and the selection invariants,
the residency invariants, block scores equal torch pooling of token-level logits (or the
bf16 codes numpy computes), and outputs equal torch softmax attention over the selected (or,
with early stop, the visited) tokens.
"""
import math

import pytest
from hypothesis import HealthCheck, assume, given, settings, strategies as st

import kv_cache_offload_nosa_b200 as nosa
import nosa_synth as syn
import oracle_pins as P
from kv_cache_offload_nosa_b200 import build as nb


@st.composite
def drawn_configs(draw, lookahead=False):
    G = draw(st.sampled_from([1, 2, 4, 8]))
    Hkv = draw(st.integers(1, 2))
    B = draw(st.integers(1, 2))
    d = draw(st.sampled_from([64, 128]))
    bs = draw(st.sampled_from([32, 64, 128]))
    s = draw(st.sampled_from([x for x in (8, 16, 32) if bs % x == 0]))
    T = tuple(draw(st.integers(1 if lookahead else 0, 5 * bs)) for _ in range(B))
    steps = draw(st.integers(1, 4))
    max_blocks = -(-(max(T) + steps) // bs)
    k_e = draw(st.integers(0, 4))
    k_q = draw(st.integers(0 if k_e else 1, 4))
    k = k_q + k_e
    assume(k <= max_blocks)
    slots = 0
    if max_blocks >= k + 2 and draw(st.booleans()):
        slots = draw(st.integers(k + 2, max_blocks))
    rows = 1 if lookahead else draw(st.sampled_from([0, 1]))
    mode = draw(st.sampled_from([0, 0, 1, 2, 3]))
    kc16 = draw(st.sampled_from([0, 1])) if mode == 0 else 0
    stop = 0.0 if lookahead else draw(st.sampled_from([0.0, 0.0, 0.05, 0.2]))
    return syn.NosaConfig("drawn", B, G * Hkv, Hkv, d, T, bs, s, k_q, k_e, steps, slots=slots,
                          n_score_rows=rows, score_mode=mode, kc_bf16=kc16, stop_tau=stop,
                          drift=0.05 if slots else 0.0, cfg_id=900)


@pytest.fixture(scope="module")
def lib():
    nb.build()
    return nosa.load()


@settings(max_examples=60, deadline=None, derandomize=True,
          suppress_health_check=[HealthCheck.too_slow, HealthCheck.function_scoped_fixture])
@given(cfg=drawn_configs())
def test_pins_hold_on_drawn_configs(lib, cfg):
    cc = nosa.make_config(cfg.B, cfg.Hq, cfg.Hkv, cfg.d, cfg.block, cfg.sub_block, cfg.k_q, cfg.k_e,
                          cfg.max_blocks, slots=cfg.n_slots, n_score_rows=cfg.rows, scale=cfg.scale,
                          score_mode=cfg.score_mode, stop_tau=cfg.stop_tau, kc_bf16=cfg.kc_bf16)
    nosa.state_sizes(cc)  # raises if the library refuses the shape
    assert math.isclose(cfg.scale, 1.0 / math.sqrt(cfg.d))
    if cfg.stop_tau > 0:
        case = P.check_early_stop(cfg)
    else:
        case = P.check_attention_subset(cfg)
    P.check_selection_trace(case)
    if cfg.offload:
        P.check_residency_trace(case)
    if cfg.kc_bf16:
        P.check_kc_bf16(cfg, steps=cfg.steps)
    else:
        P.check_score_variants(cfg, steps=cfg.steps)


@settings(max_examples=30, deadline=None, derandomize=True,
          suppress_health_check=[HealthCheck.too_slow, HealthCheck.function_scoped_fixture])
@given(cfg=drawn_configs(lookahead=True))
def test_lookahead_pins_hold_on_drawn_configs(lib, cfg):
    """SparDA's order (select and plan before the append, attend after it) on drawn shapes:
    the selection and residency invariants at the pre-append length, and the outputs equal
    torch softmax attention over the chosen blocks' tokens after the append."""
    cc = nosa.make_config(cfg.B, cfg.Hq, cfg.Hkv, cfg.d, cfg.block, cfg.sub_block, cfg.k_q, cfg.k_e,
                          cfg.max_blocks, slots=cfg.n_slots, n_score_rows=cfg.rows, scale=cfg.scale,
                          score_mode=cfg.score_mode, kc_bf16=cfg.kc_bf16)
    nosa.state_sizes(cc)
    case = P.check_attention_subset(cfg, lookahead=True)
    P.check_selection_trace(case, lookahead=True)
    if cfg.offload:
        P.check_residency_trace(case, lookahead=True)
