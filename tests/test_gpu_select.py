"""Selection kernel vs the oracle on adversarial score patterns (needs a B200).

Block and eviction scores are fed directly (fp32, identical on both sides), so
every decision must match bit for bit, ties included: few distinct values,
all-equal scores, +0.0 vs -0.0, negatives, and candidate sets large enough to
take the radix path of the top-m routine.
"""
import numpy as np
import pytest
import torch

import nosa_synth as syn
import oracle as O

pytestmark = pytest.mark.gpu


def _patterns(rng, n, kind):
    if kind == "few":
        return rng.integers(0, 3, n).astype(np.float32)
    if kind == "equal":
        return np.full(n, 0.5, np.float32)
    if kind == "signed_zero":
        v = rng.choice(np.array([0.0, -0.0, 1.0, -1.0], np.float32), n)
        return v.astype(np.float32)
    if kind == "neg":
        return (-rng.random(n) * 10).astype(np.float32)
    if kind == "quant":
        return (np.round(rng.random(n) * 8) / 8).astype(np.float32)
    return rng.standard_normal(n).astype(np.float32)


@pytest.mark.parametrize("T,bs,kq,ke", [(65536, 32, 32, 96), (8000, 64, 16, 48), (300, 32, 3, 5),
                                        (4096, 128, 1, 30)])
@pytest.mark.parametrize("kind", ["few", "equal", "signed_zero", "neg", "quant", "normal"])
def test_select_matches_oracle_bitwise(T, bs, kq, ke, kind):
    import gpu_harness as H
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    cfg = syn.NosaConfig("sel_unit", 2, 8, 2, 64, (T, T - 7), bs, 16, kq, ke, 1, cfg_id=77)
    nb = cfg.max_blocks
    NG = cfg.B * cfg.Hkv
    z = np.zeros((cfg.B, cfg.Hkv, nb * bs, cfg.d), np.uint16)
    orc = O.Oracle(cfg, z, z, None, copy=False)
    inputs = syn.Inputs(cfg, z, z, None, np.zeros((1, cfg.B, cfg.Hkv, nb), np.float32),
                        np.zeros((1, cfg.B, cfg.Hkv, cfg.d), np.uint16), np.zeros((1, cfg.B, cfg.Hkv, cfg.d), np.uint16))
    cache = H.setup(cfg, inputs)
    io = H.StepIO(cfg)
    rng = np.random.default_rng(hash((T, bs, kind)) % 2**32)
    for step in range(4):
        sc = np.stack([_patterns(rng, nb, kind) for _ in range(NG)])
        ev = np.stack([_patterns(rng, nb, kind) for _ in range(NG)])
        sel, _, _ = orc.select(sc.astype(np.float64), ev)
        cache.select(torch.from_numpy(sc).cuda(), torch.from_numpy(ev).cuda(), io.sel)
        torch.cuda.synchronize()
        got = io.sel.cpu().numpy().reshape(NG, cfg.k)
        assert np.array_equal(got, sel), f"step {step}: first diff group {np.argwhere((got != sel).any(1))[:1]}"
        assert np.array_equal(H.bits_to_flags(cache.t["alive"], NG, nb), orc.alive)
        assert np.array_equal(H.bits_to_flags(cache.t["prev_sel"], NG, nb), orc.prev_sel)
    rc, err = cache.check()
    assert rc == 0 and err == 0
