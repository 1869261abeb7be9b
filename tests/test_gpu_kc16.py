"""bf16 sub-block mean keys on the GPU (needs a B200): state set-up and appends store each
mean rounded to bf16, the score kernels read half the bytes. Selections, bitmasks, miss
counts and tables bit-exact with the fp64 oracle run with the same quantisation, outputs
within max-abs 2e-3 / relative L2 1e-3."""
import pytest
import torch

import nosa_synth as syn
import oracle as O

pytestmark = pytest.mark.gpu
CS = syn.configs()


def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


@pytest.mark.parametrize("name", ["tiny_kc16", "ragged_kc16", "llama_small_kc16", "g8_kc16", "bs128_d64_kc16"])
def test_kc16_parity(name):
    _need_gpu()
    import gpu_harness as H
    case = O.run_case(CS[name])
    _, (mx, rl2) = H.run_and_compare(case)
    assert mx <= H.ATOL and rl2 <= H.RTOL_L2


def test_kc16_lookahead():
    _need_gpu()
    import gpu_harness as H
    cfg = CS["lookahead_small"].with_(name="lookahead_small_kc16", kc_bf16=1, cfg_id=99)
    case = O.run_case(cfg, lookahead=True)
    _, (mx, rl2) = H.run_and_compare(case, mode="lookahead")
    assert mx <= H.ATOL and rl2 <= H.RTOL_L2


@pytest.mark.slow
def test_kc16_full_size():
    _need_gpu()
    import gpu_harness as H
    case = O.run_case(CS["llama_kc16"], steps=8)
    _, (mx, rl2) = H.run_and_compare(case)
    assert mx <= H.ATOL and rl2 <= H.RTOL_L2
