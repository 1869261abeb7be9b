"""Lookahead decoding (SparDA order) through nosa_plan_ahead / nosa_prefetch / nosa_attend
(needs a B200).

Every step selects and plans from the forecast row on the cache before its token is
appended, copies the planned pages, then appends and attends. Selections, miss counts and
(with host pools) the block and slot tables must equal the fp64 oracle run in the same order
bit for bit; outputs within max-abs 2e-3 / relative L2 1e-3.
"""
import pytest
import torch

import nosa_synth as syn
import oracle as O

pytestmark = pytest.mark.gpu
CS = syn.configs()


def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


@pytest.mark.parametrize("name", ["lookahead_small", "lookahead_hbm", "lookahead_ragged", "lookahead_tiny",
                                  "lookahead_dense"])
def test_lookahead_parity(name):
    _need_gpu()
    import gpu_harness as H
    case = O.run_case(CS[name], lookahead=True)
    _, (mx, rl2) = H.run_and_compare(case, mode="lookahead")
    assert mx <= H.ATOL and rl2 <= H.RTOL_L2


def test_lookahead_on_side_streams():
    """Plan and copies on two side streams, attention on the main one after an event: same
    results as one stream."""
    _need_gpu()
    import gpu_harness as H
    case = O.run_case(CS["lookahead_small"], lookahead=True)
    cfg = case.cfg
    cache = H.setup(cfg, case.inputs)
    io = H.StepIO(cfg)
    ps, cs = torch.cuda.Stream(), torch.cuda.Stream()
    main = torch.cuda.current_stream()
    for t, rec in enumerate(case.steps):
        q, rows = H.dev(rec.q), H.dev(rec.rows)
        kn, vn = H.dev(case.inputs.k_new[t]), H.dev(case.inputs.v_new[t])
        ev = H.dev(case.inputs.evict[t])
        ps.wait_stream(main)
        cache.plan_ahead(rows, ev, io.sel, io.miss, stream=ps)
        planned = torch.cuda.Event()
        planned.record(ps)
        cs.wait_event(planned)
        cache.prefetch(stream=cs)
        copied = torch.cuda.Event()
        copied.record(cs)
        main.wait_event(copied)
        cache.attend(q, kn, vn, io.sel, io.out, stream=main)
        torch.cuda.synchronize()
        H.compare_step(cache, cfg, rec, io, t)


@pytest.mark.parametrize("layers", [2, 4])
def test_lookahead_pipeline_layers(layers):
    """LookaheadPipeline over several layers (independent caches): each layer equals its own
    oracle run. With 4 layers the plans of layers 2 and 3 wait for the attention of layers 0
    and 1 (their forecast rows' inputs) on another stream."""
    _need_gpu()
    import gpu_harness as H
    from kv_cache_offload_nosa_b200.lookahead import LookaheadPipeline
    base = CS["lookahead_small"]
    cases = [O.run_case(base.with_(cfg_id=base.cfg_id + 1000 * l), lookahead=True) for l in range(layers)]
    caches = [H.setup(c.cfg, c.inputs) for c in cases]
    ios = [H.StepIO(c.cfg) for c in cases]
    pipe = LookaheadPipeline(caches)
    for t in range(len(cases[0].steps)):
        recs = [c.steps[t] for c in cases]
        pipe.token([H.dev(r.rows) for r in recs], [H.dev(c.inputs.evict[t]) for c in cases],
                   [H.dev(r.q) for r in recs], [H.dev(c.inputs.k_new[t]) for c in cases],
                   [H.dev(c.inputs.v_new[t]) for c in cases], [io.sel for io in ios],
                   [io.miss for io in ios], [io.out for io in ios])
        torch.cuda.synchronize()
        for c, cache, io, r in zip(cases, caches, ios, recs):
            H.compare_step(cache, c.cfg, r, io, t)
