"""A decode step captured in a CUDA graph and replayed, step after step, vs the fp64 oracle.

Step 0 runs with direct launches (the warm-up before capture); then one graph per cache is
captured and replayed for every later step with that step's inputs staged into its buffers:
selections, masks, miss counts and the block table must match the oracle bit for bit and
outputs within the usual tolerances, exactly as for direct launches (the cross-step flags and
tickets are reset on the device, not by the host).
"""
import types

import pytest
import torch

import nosa_synth as syn
import oracle as O

pytestmark = pytest.mark.gpu

CS = syn.configs()


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


@pytest.mark.parametrize("name", ["tiny", "tiny_forecast", "offload_small", "ragged_offload",
                                  "tiny_stop", "short_kq0_offload", "llama_small_window"])
def test_graph_replay_matches_oracle(name):
    import gpu_harness as H
    from kv_cache_offload_nosa_b200.graph import StepGraph
    case = O.run_case(CS[name])
    cfg = case.cfg
    cache = H.setup(cfg, case.inputs)
    io0 = H.StepIO(cfg)
    H.run_step(cache, cfg, case.inputs, case.steps[0], 0, io0)
    H.compare_step(cache, cfg, case.steps[0], io0, 0)
    g = StepGraph(cache, forecast_rows=cfg.n_score_rows == 1)
    io = types.SimpleNamespace(sel=g.sel, out=g.out, miss=g.miss[:cfg.B * cfg.Hkv])
    assert len(case.steps) >= 3
    for t, rec in enumerate(case.steps):
        if t == 0:
            continue
        rows = H.dev(rec.rows) if cfg.n_score_rows == 1 else None
        g.run(H.dev(rec.q), H.dev(case.inputs.k_new[t]), H.dev(case.inputs.v_new[t]),
              H.dev(case.inputs.evict[t]), rows)
        torch.cuda.synchronize()
        H.compare_step(cache, cfg, rec, io, t)


def test_graph_needs_forecast_buffer_when_configured():
    import gpu_harness as H
    from kv_cache_offload_nosa_b200.graph import StepGraph
    cfg = CS["tiny_forecast"]
    cache = H.setup(cfg, syn.make_inputs(cfg))
    with pytest.raises(ValueError):
        StepGraph(cache, forecast_rows=False)
