"""Device-side error paths, made to happen without faulting the GPU.

Each case plants a host-written bad input (a selected block outside [0, N), a block-table
entry outside the pools) or a wait that nothing will end (a per-group flag no kernel sets,
under a short wait limit). The kernels' own checks must skip the bad access and record it in
the state's error word, every other group must still match the oracle, and the context and
library must stay usable: a fresh state then runs the workload against the oracle again.
Every bad index here is refused by the attention producer's checks before any load is issued
(the selected index against N, the page against the pool size), and every wait is bounded by
the configuration's wait limit.
"""
import numpy as np
import pytest
import torch

import kv_cache_offload_nosa_b200 as nosa
import nosa_synth as syn
import oracle as O

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _run_first_step(name, wait_us=0):
    import gpu_harness as H
    cfg = syn.configs()[name]
    case = O.run_case(cfg, steps=2)
    cache = H.setup(cfg, case.inputs)
    if wait_us:
        cache.cfg.wait_us = wait_us
    io = H.StepIO(cfg)
    H.run_step(cache, cfg, case.inputs, case.steps[0], 0, io)
    H.compare_step(cache, cfg, case.steps[0], io, 0)
    return cfg, case, cache, io


def _other_groups_match(cfg, rec, out, bad_group):
    import gpu_harness as H
    got = out.cpu().numpy().reshape(cfg.B * cfg.Hkv, cfg.G, cfg.d)
    want = rec.out.reshape(cfg.B * cfg.Hkv, cfg.G, cfg.d)
    keep = np.arange(cfg.B * cfg.Hkv) != bad_group
    mx, rl2 = H.out_errors(got[keep], want[keep])
    assert mx <= H.ATOL and rl2 <= H.RTOL_L2, (mx, rl2)


def _rerun_clean(cfg, case, cache):
    """After a recorded fault: zero the error word and the workspace, rebuild the state from the
    prefill and run the workload's steps against the oracle again."""
    import gpu_harness as H
    cache.t["err"].zero_()
    nosa.workspace_init(cache.ws, cache.ws_bytes)
    cache.init(cache._plen, cache._res)
    torch.cuda.synchronize()
    io = H.StepIO(cfg)
    for t, rec in enumerate(case.steps):
        H.run_step(cache, cfg, case.inputs, rec, t, io)
        H.compare_step(cache, cfg, rec, io, t)


@pytest.mark.parametrize("name", ["tiny", "offload_small"])
def test_selected_block_past_the_context_is_skipped_and_recorded(name):
    """sel holds a block index >= N for one group: that block is not read, NOSA_ERR_SEL is
    recorded, nosa_check_device returns NOSA_EDEVICE and the other groups' outputs are the
    oracle's."""
    cfg, case, cache, io = _run_first_step(name)
    rec = case.steps[0]
    bad = 1 % (cfg.B * cfg.Hkv)
    sel = rec.sel.copy()
    N = -(-(cfg.T[bad // cfg.Hkv] + 1) // cfg.block)
    sel[bad, 0] = N + 3
    out = torch.full((cfg.B * cfg.Hq * cfg.d,), float("nan"), device="cuda")
    cache.decode_attn(torch.from_numpy(rec.q).view(torch.int16).cuda(), torch.from_numpy(sel).cuda(), out)
    rc, err = cache.check()
    assert rc == nosa.NOSA_EDEVICE and err & nosa.ERR_SEL, (rc, hex(err))
    assert not err & ~(nosa.ERR_SEL), hex(err)
    _other_groups_match(cfg, rec, out, bad)
    _rerun_clean(cfg, case, cache)


def test_block_table_entry_outside_the_pools_is_skipped_and_recorded():
    """With host pools the attention reads the block table: one selected block's entry points
    past the last HBM page. The page is not read, NOSA_ERR_BLOCK_TABLE is recorded and the
    other groups' outputs are the oracle's."""
    cfg, case, cache, io = _run_first_step("offload_small")
    rec = case.steps[0]
    bad = 0
    j = int(rec.sel[bad][0])
    total_pages = cfg.B * cfg.Hkv * cfg.n_slots
    bt = cache.t["block_table"].view(cfg.B * cfg.Hkv, cfg.max_blocks)
    bt[bad, j] = total_pages + 7
    out = torch.full((cfg.B * cfg.Hq * cfg.d,), float("nan"), device="cuda")
    cache.decode_attn(torch.from_numpy(rec.q).view(torch.int16).cuda(),
                      torch.from_numpy(rec.sel).cuda(), out)
    rc, err = cache.check()
    assert rc == nosa.NOSA_EDEVICE and err == nosa.ERR_BLOCK_TABLE, (rc, hex(err))
    _other_groups_match(cfg, rec, out, bad)
    _rerun_clean(cfg, case, cache)


@pytest.mark.parametrize("name", ["lookahead_tiny", "offload_small"])
def test_flag_that_never_arrives_times_out(name):
    """nosa_attend with no nosa_plan_ahead / nosa_prefetch before it: the per-group flags it
    acquires are never set. Under a 20 ms wait limit every wait gives up, the kernels return,
    NOSA_ERR_TIMEOUT is recorded and nosa_check_device returns NOSA_ETIMEOUT. Every selected
    entry is -1, so nothing is read whatever the flags. The library then runs the workload
    against the oracle again on a rebuilt state."""
    import time
    cfg, case, cache, io = _run_first_step(name, wait_us=20000)
    nosa.workspace_init(cache.ws, cache.ws_bytes)  # no flag is left set by the step
    rec = case.steps[1]
    NG = cfg.B * cfg.Hkv
    sel = torch.full((NG * cfg.k,), -1, dtype=torch.int32, device="cuda")
    out = torch.empty(cfg.B * cfg.Hq * cfg.d, dtype=torch.float32, device="cuda")
    kn = torch.from_numpy(case.inputs.k_new[1]).view(torch.int16).cuda()
    vn = torch.from_numpy(case.inputs.v_new[1]).view(torch.int16).cuda()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    cache.attend(torch.from_numpy(rec.q).view(torch.int16).cuda(), kn, vn, sel, out)
    rc, err = cache.check()
    dt = time.perf_counter() - t0
    assert rc == nosa.NOSA_ETIMEOUT and err & nosa.ERR_TIMEOUT, (rc, hex(err))
    assert dt < 5.0, dt  # the 20 ms limit, not the 4 s default
    _rerun_clean(cfg, case, cache)


def test_workspace_one_byte_short_is_refused_before_any_launch():
    """nosa_step with ws_bytes one byte below nosa_workspace_size: NOSA_ENOMEM, and the state is
    untouched (nothing was launched)."""
    import gpu_harness as H
    cfg = syn.configs()["tiny"]
    case = O.run_case(cfg, steps=1)
    cache = H.setup(cfg, case.inputs)
    io = H.StepIO(cfg)
    rec = case.steps[0]
    seq0 = cache.t["seq_len"].clone()
    q = torch.from_numpy(rec.q).view(torch.int16).cuda()
    kn = torch.from_numpy(case.inputs.k_new[0]).view(torch.int16).cuda()
    vn = torch.from_numpy(case.inputs.v_new[0]).view(torch.int16).cuda()
    ev = torch.from_numpy(case.inputs.evict[0]).cuda()
    with pytest.raises(nosa.NosaError) as e:
        nosa.step(cache.cfg, cache.state, q, None, kn, vn, ev, io.sel, io.out, io.miss, cache.ws,
                  cache.ws_bytes - 1)
    assert e.value.status == nosa.NOSA_ENOMEM
    torch.cuda.synchronize()
    assert torch.equal(cache.t["seq_len"], seq0)
    rc, err = cache.check()
    assert rc == nosa.NOSA_OK and err == 0
