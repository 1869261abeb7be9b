"""CUDA path vs the fp64 oracle on the same seeded inputs (needs a B200).

Selections, masks, miss counts and the block table must match bit for bit;
attention outputs within max-abs 2e-3 and relative L2 1e-3 of fp64.
"""
import numpy as np
import pytest
import torch

import nosa_synth as syn
import oracle as O

pytestmark = pytest.mark.gpu

CS = syn.configs()
SMALL = ["tiny", "tiny_dense", "tiny_static", "tiny_forecast", "llama_small", "offload_small",
         "sink_small", "ragged", "ragged_offload", "empty", "bs128_d64", "g8", "short_kq0",
         "short_kq0_offload"]

_cases = {}


def case(name, steps=None):
    key = (name, steps)
    if key not in _cases:
        _cases[key] = O.run_case(CS[name], steps=steps)
    return _cases[key]


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import gpu_harness  # noqa: F401


@pytest.mark.parametrize("name", SMALL)
def test_step_parity_fused(name):
    import gpu_harness as H
    H.run_and_compare(case(name))


@pytest.mark.parametrize("name", ["tiny", "offload_small", "ragged_offload", "tiny_forecast", "bs128_d64"])
def test_step_parity_separate_calls(name):
    import gpu_harness as H
    H.run_and_compare(case(name), mode="separate")


@pytest.mark.parametrize("name", ["tiny", "offload_small", "ragged_offload", "llama_small", "g8"])
def test_step_parity_with_events(name):
    """nosa_step given events (the form bench.py times kernel by kernel): the kernels chain by
    whole grids instead of per-group flags, and host pools go through the grid-wide copy kernel.
    Same selections, state and outputs as the oracle."""
    import gpu_harness as H
    H.run_and_compare(case(name), mode="events")


@pytest.mark.parametrize("name", ["tiny", "ragged", "bs128_d64", "g8"])
def test_block_scores_vs_oracle(name):
    import gpu_harness as H
    c = case(name)
    cfg = c.cfg
    cache = H.setup(cfg, c.inputs)
    io = H.StepIO(cfg)
    NG = cfg.B * cfg.Hkv
    for t, rec in enumerate(c.steps):
        cache.append(H.dev(c.inputs.k_new[t]), H.dev(c.inputs.v_new[t]))
        rows = H.dev(rec.rows)
        cache.score_blocks(rows, io.scores)
        got = io.scores.cpu().numpy().reshape(NG, cfg.max_blocks).astype(np.float64)
        want = rec.scores
        fin = np.isfinite(want)
        assert np.array_equal(np.isneginf(got), np.isneginf(want))
        np.testing.assert_allclose(got[fin], want[fin], rtol=1e-5, atol=1e-6)
        # the GPU's selection is exactly the top-k rule applied to the GPU's own scores
        cache.select(io.scores, H.dev(c.inputs.evict[t]), io.sel)
        cache.decode_attn(H.dev(rec.q), io.sel, io.out)
        torch.cuda.synchronize()
        assert np.array_equal(io.sel.cpu().numpy().reshape(NG, cfg.k), rec.sel)


@pytest.mark.parametrize("split", [1, 2, 3, 5, 8, 16])
def test_split_count_invariance(split):
    """The split-K partition does not change the result beyond fp32 rounding."""
    import gpu_harness as H
    c = case("llama_small")
    base, _ = None, None
    outs = []
    for sp in (0, split):
        cache = H.setup(c.cfg, c.inputs, attn_split=sp)
        io = H.StepIO(c.cfg)
        H.run_step(cache, c.cfg, c.inputs, c.steps[0], 0, io)
        outs.append(io.out.cpu().numpy())
    d = np.abs(outs[0] - outs[1]).max()
    assert d <= 1e-6 * max(1.0, np.abs(outs[0]).max()), d


@pytest.mark.parametrize("name", ["offload_small", "llama_small"])
def test_fused_equals_separate(name):
    """The fused step and the separate calls select the same blocks and make the same misses,
    bit for bit, and give the same outputs up to fp32 summation order: the fused step attends a
    group's query-agnostic blocks first (they are published before the query-aware half),
    the separate calls attend S(t) in ascending order."""
    import gpu_harness as H
    c = case(name)
    res = []
    for mode in ("fused", "separate"):
        cache = H.setup(c.cfg, c.inputs)
        io = H.StepIO(c.cfg)
        outs = []
        for t, rec in enumerate(c.steps[:4]):
            H.run_step(cache, c.cfg, c.inputs, rec, t, io, mode)
            outs.append((io.sel.cpu().numpy().copy(), io.out.cpu().numpy().copy(), io.miss.cpu().numpy().copy()))
        res.append(outs)
    for (sa, oa, ma), (sb, ob, mb) in zip(*res):
        assert np.array_equal(sa, sb) and np.array_equal(ma, mb)
        np.testing.assert_allclose(oa, ob, rtol=1e-5, atol=1e-6)
