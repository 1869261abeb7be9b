"""nosa_decode_attn_noalloc: the workspace-free attention entry point (needs a B200).

Callers that cannot allocate device memory when attention runs (plugins whose
host framework owns all device memory, serving loops that must not allocate)
use this entry point; its scratch lives in a static device array
inside the library. It must give the same output as nosa_decode_attn, call
after call, since every call reuses (and must re-zero) the same scratch.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import numpy as np
import pytest
import torch

import nosa_synth as syn
import oracle as O

pytestmark = pytest.mark.gpu


# (workload, attention split): all blocks in HBM at the automatic split; host pools, so the
# kernel reads the block table; and a split that does not divide k, so CTA ranges cross group
# boundaries and several segments of a group share the static partials.
CASES = [("llama_small", 0), ("offload_small", 0), ("llama_small", 7), ("offload_small", 3)]


@pytest.fixture(scope="module", params=CASES, ids=[f"{n}-W{w}" for n, w in CASES])
def prepared(request):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import gpu_harness as H
    name, split = request.param
    case = O.run_case(syn.configs()[name], steps=2)
    cfg = case.cfg
    cache = H.setup(cfg, case.inputs, attn_split=split)
    io = H.StepIO(cfg)
    H.run_step(cache, cfg, case.inputs, case.steps[0], 0, io)   # a real step: append, select, attend
    q = H.dev(case.steps[0].q)
    return H, case, cache, io, q


def test_noalloc_matches_workspace_entry_point_on_two_calls(prepared):
    import kv_cache_offload_nosa_b200 as nosa
    H, case, cache, io, q = prepared
    cfg = case.cfg
    cache.decode_attn(q, io.sel, io.out)         # existing entry point, caller workspace
    torch.cuda.synchronize()
    ref = io.out.clone()
    want = case.steps[0].out
    for call in range(2):
        out = torch.full_like(ref, float("nan"))
        nosa.decode_attn_noalloc(cache.cfg, cache.state, q, io.sel, out)
        torch.cuda.synchronize()
        got = out.cpu().numpy().reshape(cfg.B, cfg.Hq, cfg.d)
        mx, rl2 = H.out_errors(got, ref.cpu().numpy().reshape(cfg.B, cfg.Hq, cfg.d).astype(np.float64))
        assert mx <= H.ATOL and rl2 <= H.RTOL_L2, (call, mx, rl2)
        mx, rl2 = H.out_errors(got, want)          # and against the fp64 oracle
        assert mx <= H.ATOL and rl2 <= H.RTOL_L2, (call, mx, rl2)
    rc, err = cache.check()
    assert rc == nosa.NOSA_OK and err == 0


def test_noalloc_rejects_configs_beyond_its_scratch(prepared):
    import kv_cache_offload_nosa_b200 as nosa
    H, case, cache, io, q = prepared
    c = cache.cfg
    big = nosa.make_config(4096, c.Hq, c.Hkv, c.d, c.block_size, c.sub_block, c.k_q, c.k_e,
                           c.max_blocks)
    with pytest.raises(nosa.NosaError) as e:
        nosa.decode_attn_noalloc(big, cache.state, q, io.sel, io.out)
    assert e.value.status == nosa.NOSA_ENOMEM
