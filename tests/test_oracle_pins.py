"""The oracle against what the pages and mathematics fix (CPU only)."""
import numpy as np
import pytest
import torch

import nosa_synth as syn
import oracle as O
import oracle_pins as P

CS = syn.configs()


def test_generator_bf16_matches_torch_rne():
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-8, 8, 20000),
                        [0.0, -0.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 3.0e38, 1e-40]])
    want = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(syn.round_bf16(x), want)


def test_generator_is_counter_based():
    a = syn.gauss(0, syn.T_K, 3, 4, 5, 1000)
    b = syn.gauss(0, syn.T_K, 3, 4, 5, 400, i0=600)
    assert np.array_equal(a[600:], b)
    assert abs(a.mean()) < 0.1 and abs(a.std() - 1) < 0.1
    u = syn.uniform(0, syn.T_EVICT, 0, 0, 0, 100000)
    assert 0 < u.min() and u.max() < 1 and abs(u.mean() - 0.5) < 0.01


def test_topm_matches_bruteforce_rank_count():
    P.check_topm_bruteforce()


def test_hand_worked_dual_selection():
    P.check_hand_dual_selection()


@pytest.mark.parametrize("golden", ["hand_residency.json", "hand_residency_order.json"])
def test_hand_worked_residency(golden):
    P.check_hand_residency(name=golden)


def test_static_eviction_closed_form():
    P.check_static_closed_form()


def test_dense_selection_equals_sdpa():
    P.check_attention_dense_sdpa()


@pytest.mark.parametrize("name", ["tiny", "ragged", "tiny_forecast", "bs128_d64", "g8", "empty"])
def test_pooling_equals_library_pools(name):
    P.check_pooling_library(CS[name], steps=2 if name != "empty" else 6)


@pytest.mark.parametrize("name", ["tiny", "ragged", "ragged_offload", "offload_small", "sink_small", "g8",
                                  "empty", "tiny_forecast", "short_kq0", "short_kq0_offload"])
def test_attention_and_selection_trace(name):
    case = P.check_attention_subset(CS[name])
    P.check_selection_trace(case)
    if case.cfg.offload:
        P.check_residency_trace(case)


@pytest.mark.parametrize("name", ["tiny_window", "tiny_softmax", "tiny_window_softmax", "ragged_window",
                                  "ragged_softmax", "ragged_window_softmax", "forecast_softmax",
                                  "llama_small_window_softmax"])
def test_score_variants_equal_torch_pooling(name):
    P.check_score_variants(CS[name])


@pytest.mark.parametrize("name", ["tiny_stop", "tiny_dense_stop", "ragged_stop", "llama_small_stop"])
def test_early_stop_equals_torch_rule(name):
    P.check_early_stop(CS[name])


@pytest.mark.parametrize("name", ["tiny_kc16", "ragged_kc16", "llama_small_kc16", "bs128_d64_kc16"])
def test_kc_bf16_codes_equal_numpy(name):
    P.check_kc_bf16(CS[name])


def test_lookahead_dense_equals_sdpa():
    P.check_lookahead_dense_sdpa()


@pytest.mark.parametrize("name", ["lookahead_tiny", "lookahead_ragged", "lookahead_small"])
def test_lookahead_attention_and_selection_trace(name):
    case = P.check_attention_subset(CS[name], lookahead=True)
    P.check_selection_trace(case, lookahead=True)
    if case.cfg.offload:
        P.check_residency_trace(case, lookahead=True)


def test_lookahead_needs_forecast_rows_and_prefill():
    with pytest.raises(ValueError):
        O.run_case(CS["tiny"], steps=1, lookahead=True)
    with pytest.raises(ValueError):
        O.run_case(CS["empty"].with_(n_score_rows=1), steps=1, lookahead=True)


def test_margin_enforced():
    case = O.run_case(CS["llama_small"])
    for rec in case.steps:
        assert np.all(rec.gap >= O.MARGIN)
