"""Parity at the workloads' full sizes and step counts (needs a B200).

Each workload runs through nosa_step exactly as the benchmark launches it; every
step's selections, bitmasks, miss counts (and, with host pools, block table and
slot owners) must equal the fp64 oracle's bit for bit, and every output head
must be within max-abs 2e-3 / relative L2 1e-3 of fp64.
"""
import pytest
import torch

import nosa_synth as syn
import oracle as O

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

CS = syn.configs()
FULL = ["llama", "offload", "sink"] + [p.name for p in syn.sweep_points()]


@pytest.mark.parametrize("name", FULL)
def test_full_size_parity(name):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import gpu_harness as H
    case = O.run_case(CS[name])
    _, (mx, rl2) = H.run_and_compare(case)
    assert mx <= H.ATOL and rl2 <= H.RTOL_L2


def test_full_size_lookahead_parity():
    """The offload workload with a forecast row, in lookahead order, at full size."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import gpu_harness as H
    case = O.run_case(CS["lookahead"], steps=16, lookahead=True)
    _, (mx, rl2) = H.run_and_compare(case, mode="lookahead")
    assert mx <= H.ATOL and rl2 <= H.RTOL_L2
