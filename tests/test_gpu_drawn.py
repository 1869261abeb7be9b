"""GPU parity on configurations drawn across the shapes the library accepts.

The oracle's pins run on configurations a seeded hypothesis search draws (the strategy of
``test_oracle_properties.py``: G in {1, 2, 4, 8}, d in {64, 128}, block size 32/64/128 with
every sub-block size that divides it, ragged and empty prefills, k_q = 0 or k_e = 0, host
pools, forecast rows, scoring variants, bf16 means, early stop). Here the same draws run
through the CUDA library step by step -- the fused step, and SparDA's lookahead calls -- and
are compared with the oracle: selections, bitmasks, miss counts and block tables bit for
bit, outputs within max-abs 2e-3 and relative L2 1e-3 of fp64. A fixed grid adds the shapes
no workload uses, G in {1, 2} with sub-blocks of 8, at several attention splits (including
splits that do not divide k, so CTA ranges cross group boundaries).
"""
import pytest
import torch
from hypothesis import HealthCheck, given, settings

import nosa_synth as syn
import oracle as O
from test_oracle_properties import drawn_configs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


@settings(max_examples=40, deadline=None, derandomize=True,
          suppress_health_check=[HealthCheck.too_slow, HealthCheck.function_scoped_fixture])
@given(cfg=drawn_configs())
def test_gpu_matches_oracle_on_drawn_configs(cfg):
    import gpu_harness as H
    H.run_and_compare(O.run_case(cfg))


@settings(max_examples=20, deadline=None, derandomize=True,
          suppress_health_check=[HealthCheck.too_slow, HealthCheck.function_scoped_fixture])
@given(cfg=drawn_configs(lookahead=True))
def test_gpu_lookahead_matches_oracle_on_drawn_configs(cfg):
    import gpu_harness as H
    H.run_and_compare(O.run_case(cfg, lookahead=True), mode="lookahead")


def _grid():
    out = []
    i = 0
    for G in (1, 2):
        for d in (64, 128):
            for bs in (32, 64, 128):
                for offload in (False, True):
                    T = (5 * bs + 5, bs - 1) if not offload else (12 * bs + 3, 5 * bs)
                    k_q, k_e = (2, 3) if not offload else (3, 2)
                    steps = 3
                    nb = -(-(max(T) + steps) // bs)
                    slots = k_q + k_e + 3 if offload else 0
                    out.append(syn.NosaConfig(f"g{G}_d{d}_bs{bs}_s8_{'off' if offload else 'hbm'}",
                                              2, 2 * G, 2, d, T, bs, 8, k_q, k_e, steps,
                                              slots=slots if slots <= nb else 0,
                                              drift=0.05 if offload else 0.0, cfg_id=950 + i))
                    i += 1
    return out


_GRID = _grid()


@pytest.mark.parametrize("cfg", _GRID, ids=[c.name for c in _GRID])
@pytest.mark.parametrize("split", [0, 1, 3])
def test_gpu_small_groups_and_8_token_sub_blocks(cfg, split):
    """G = 1 or 2 and sub-block 8 at every block size and head dim, with and without host
    pools, through the fused step at the automatic split and at splits 1 and 3 (3 does not
    divide k = 5: CTA ranges cross group boundaries)."""
    import gpu_harness as H
    H.run_and_compare(O.run_case(cfg), attn_split=split)


@pytest.mark.parametrize("cfg", [c for c in _GRID if c.d == 128], ids=[c.name for c in _GRID if c.d == 128])
def test_gpu_small_groups_lookahead(cfg):
    """The same shapes in SparDA's lookahead order (one forecast row per group)."""
    import dataclasses
    import gpu_harness as H
    f = dataclasses.replace(cfg, n_score_rows=1, name=cfg.name + "_la")
    H.run_and_compare(O.run_case(f, lookahead=True), mode="lookahead")
