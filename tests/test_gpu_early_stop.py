"""S2O early stop on the GPU (needs a B200): blocks visited in decreasing score, each head
stopping after the first block whose gain in softmax mass is below tau times the mass so far.
The number of blocks each head visited must equal the fp64 oracle's exactly (decisions and
order margins enforced on the inputs), selections and tables bit-exact, outputs within
max-abs 2e-3 / relative L2 1e-3."""
import pytest
import torch

import nosa_synth as syn
import oracle as O

pytestmark = pytest.mark.gpu
CS = syn.configs()


def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


@pytest.mark.parametrize("name", ["tiny_stop", "tiny_dense_stop", "ragged_stop", "llama_small_stop"])
def test_early_stop_parity(name):
    _need_gpu()
    import gpu_harness as H
    case = O.run_case(CS[name])
    _, (mx, rl2) = H.run_and_compare(case)
    assert mx <= H.ATOL and rl2 <= H.RTOL_L2


@pytest.mark.parametrize("name", ["tiny_stop", "ragged_stop", "llama_small_stop"])
def test_early_stop_parity_with_events(name):
    """The same with events between the kernels: the stop kernel waits for the whole score
    grid (and, with host pools, the grid-wide page copy) instead of its group's flag."""
    _need_gpu()
    import gpu_harness as H
    case = O.run_case(CS[name])
    _, (mx, rl2) = H.run_and_compare(case, mode="events")
    assert mx <= H.ATOL and rl2 <= H.RTOL_L2


def test_early_stop_refused_outside_the_step():
    _need_gpu()
    import gpu_harness as H
    import kv_cache_offload_nosa_b200 as nosa
    case = O.run_case(CS["tiny_stop"], steps=1)
    cache = H.setup(case.cfg, case.inputs)
    io = H.StepIO(case.cfg)
    q = H.dev(case.steps[0].q)
    with pytest.raises(nosa.NosaError) as e:
        cache.decode_attn(q, io.sel, io.out)
    assert e.value.status == nosa.NOSA_EINVAL
    with pytest.raises(nosa.NosaError) as e:
        nosa.decode_attn_noalloc(cache.cfg, cache.state, q, io.sel, io.out)
    assert e.value.status == nosa.NOSA_EINVAL


@pytest.mark.slow
def test_early_stop_full_size():
    _need_gpu()
    import gpu_harness as H
    case = O.run_case(CS["llama_stop"], steps=8)
    _, (mx, rl2) = H.run_and_compare(case)
    assert mx <= H.ATOL and rl2 <= H.RTOL_L2
