"""Scoring variants on the GPU (needs a B200): overlapping windows of two sub-blocks and the
per-row softmax summed over the rows, alone and together, through nosa_step and the
lookahead calls. Selections, bitmasks, miss counts and tables bit-exact with the fp64 oracle
(softmax margins in log units), outputs within max-abs 2e-3 / relative L2 1e-3."""
import pytest
import torch

import nosa_synth as syn
import oracle as O

pytestmark = pytest.mark.gpu
CS = syn.configs()
NAMES = [f"{base}_{tag}" for base in ("tiny", "ragged", "llama_small")
         for tag in ("window", "softmax", "window_softmax")] + ["forecast_softmax"]


def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


@pytest.mark.parametrize("name", NAMES)
def test_score_variant_parity(name):
    _need_gpu()
    import gpu_harness as H
    case = O.run_case(CS[name])
    _, (mx, rl2) = H.run_and_compare(case)
    assert mx <= H.ATOL and rl2 <= H.RTOL_L2


def test_score_variant_lookahead():
    _need_gpu()
    import gpu_harness as H
    cfg = CS["lookahead_small"].with_(name="lookahead_small_window_softmax", score_mode=3, cfg_id=91)
    case = O.run_case(cfg, lookahead=True)
    _, (mx, rl2) = H.run_and_compare(case, mode="lookahead")
    assert mx <= H.ATOL and rl2 <= H.RTOL_L2


def test_score_variants_refused_by_standalone_scoring():
    _need_gpu()
    import gpu_harness as H
    import kv_cache_offload_nosa_b200 as nosa
    case = O.run_case(CS["tiny_softmax"], steps=1)
    cache = H.setup(case.cfg, case.inputs)
    io = H.StepIO(case.cfg)
    with pytest.raises(nosa.NosaError) as e:
        cache.score_blocks(H.dev(case.steps[0].q), io.scores)
    assert e.value.status == nosa.NOSA_EINVAL


@pytest.mark.slow
@pytest.mark.parametrize("name", ["llama_window", "llama_softmax"])
def test_score_variant_full_size(name):
    _need_gpu()
    import gpu_harness as H
    case = O.run_case(CS[name], steps=8)
    _, (mx, rl2) = H.run_and_compare(case)
    assert mx <= H.ATOL and rl2 <= H.RTOL_L2
