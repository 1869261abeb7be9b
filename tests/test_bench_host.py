"""Host-side arithmetic of bench.py (CPU only): algorithmic bytes, clock records, traffic record.

The roofline's numerator is the algorithmic bytes of a step, per group: the sub-block means
read (M*d*4, or M*d*2 for bf16 means), K and V of the selected blocks (|S|*bs*d*2*2), the
eviction scores (N*4), the two selection bitmasks read and written, q (G*d*2), out (G*d*4)
and the appended token (2*d*2); a few bookkeeping words (block scores, the selection) add
well under 1 %. Pages copied from host memory add one HBM write and one PCIe read each.
"""
import os
import shutil

import pytest

import bench
import nosa_synth as syn


def per_group_bytes(c, L, nsel=None):
    N = -(-L // c.block)
    M = -(-L // c.sub_block)
    S = min(c.k, N) if nsel is None else nsel
    masks = 2 * 2 * 4 * -(-N // 32)
    return (M * c.d * (2 if c.kc_bf16 else 4) + S * c.block * c.d * 2 * 2 + N * 4 + masks
            + c.G * c.d * 2 + c.G * c.d * 4 + 2 * c.d * 2)


@pytest.mark.parametrize("name", ["tiny", "llama", "offload", "sink", "llama_kc16", "ragged", "g8"])
def test_step_bytes_is_the_per_group_sum(name):
    c = syn.configs()[name]
    for L in (max(c.T) + 1, max(c.T) + c.steps):
        tot, attn, score, pcie = bench.step_bytes(c, L)
        want = c.B * c.Hkv * per_group_bytes(c, L)
        assert want <= tot <= 1.01 * want, (name, L, tot, want)
        assert tot == attn + score and pcie == 0
        # the attention kernel's share: the selected pages plus q and out
        kv = c.B * c.Hkv * min(c.k, -(-L // c.block)) * c.block * c.d * 4
        assert kv < attn <= 1.01 * kv + c.B * c.Hkv * (c.G * c.d * 6 + 8 * c.k)


def test_step_bytes_table_sizes():
    """The per-step sizes the workloads were chosen for: ~0.66 MB (tiny), ~403 MB (the
    Llama-shaped and sink layers), ~269 MB of HBM (offload)."""
    for name, mb in (("tiny", 0.66), ("llama", 403.0), ("sink", 403.0), ("offload", 269.0)):
        c = syn.configs()[name]
        tot = bench.step_bytes(c, c.T[0] + 1)[0] / 1e6
        assert abs(tot / mb - 1) < 0.01, (name, tot, mb)


def test_step_bytes_misses_and_early_stop():
    c = syn.configs()["offload"]
    L = c.T[0] + 1
    base = bench.step_bytes(c, L)
    page = c.block * c.d * 2
    got = bench.step_bytes(c, L, misses=10)
    assert got[0] - base[0] == 10 * 2 * page and got[3] == 10 * 2 * page
    s = syn.configs()["llama_stop"]
    L = s.T[0] + 1
    full, part = bench.step_bytes(s, L), bench.step_bytes(s, L, visited=40.0)
    assert full[1] - part[1] == pytest.approx(s.B * s.Hkv * (s.k - 40) * s.block * s.d * 4)
    assert full[2] == part[2]


def test_bf16_means_halve_the_score_bytes():
    c = syn.configs()["llama"]
    h = syn.configs()["llama_kc16"]
    L = c.T[0] + 1
    M = -(-L // c.sub_block)
    assert bench.step_bytes(c, L)[2] - bench.step_bytes(h, L)[2] == c.B * c.Hkv * M * c.d * 2


def test_clock_summary_reads_median_and_reasons(tmp_path):
    clk = bench.Clocks(0)
    clk.path = str(tmp_path / "clocks.csv")
    rows = [
        "0, 1965, 1965, 700.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1950, 1965, 990.5, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1965, 1965, 800.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "garbage line",
    ]
    open(clk.path, "w").write("\n".join(rows) + "\n")
    clk.p = object()  # a sampler ran
    s = clk.summary()
    assert s["sm_mhz"] == 1965.0 and s["sm_max_mhz"] == 1965.0 and s["samples"] == 3
    assert s["reasons"] == ["sw_power_cap"]
    assert not os.path.exists(clk.path)


def test_clock_summary_without_sampler():
    clk = bench.Clocks(0)
    assert clk.summary()["reasons"] == ["nvidia-smi unavailable"]


def test_traffic_record_needs_the_captured_source(tmp_path, monkeypatch):
    """The ncu traffic figure is reported only while the attention kernel's source hashes to
    the one that was captured, scaled from the captured batch by the number of groups."""
    import json
    root = tmp_path / "r"
    csrc = root / "kv_cache_offload_nosa_b200" / "csrc"
    csrc.mkdir(parents=True)
    (root / "profiles").mkdir()
    for f in ("nosa_attn.cuh", "nosa_common.cuh"):
        shutil.copy(os.path.join(bench.ROOT, "kv_cache_offload_nosa_b200", "csrc", f), csrc / f)
    monkeypatch.setattr(bench, "ROOT", str(root))
    assert bench.attn_traffic(16) is None  # no record
    (root / "profiles" / "attn_traffic.json").write_text(json.dumps(
        {"batch": 8, "dram_bytes_per_launch": 1000, "source_sha256": bench.kernel_source_sha()}))
    assert bench.attn_traffic(16) == 2000
    with open(csrc / "nosa_attn.cuh", "a") as f:
        f.write("// changed\n")
    assert bench.attn_traffic(16) is None


def test_committed_traffic_record_is_well_formed():
    """profiles/attn_traffic.json, when present, names its batch, bytes, source hash and the
    ncu command it came from (which leaves the clocks alone)."""
    import json
    p = os.path.join(bench.ROOT, "profiles", "attn_traffic.json")
    if not os.path.exists(p):
        pytest.skip("no traffic record committed")
    rec = json.load(open(p))
    assert rec["batch"] > 0 and rec["dram_bytes_per_launch"] > 0
    assert len(rec["source_sha256"]) == 64
    assert "--clock-control none" in rec["command"]


def test_profile_commands_leave_clocks_alone_and_run_committed_files():
    """Every ncu command recorded under profiles/ unlocks nothing it did not lock
    (--clock-control none) and runs only the committed benchmark."""
    import re
    pdir = os.path.join(bench.ROOT, "profiles")
    names = sorted(f for f in os.listdir(pdir) if f.endswith((".md", ".txt")))
    assert names
    for f in names:
        text = open(os.path.join(pdir, f)).read()
        cmds = [l for l in text.splitlines() if re.search(r"(^|\s)ncu\s+--", l)]
        assert cmds, f"{f}: no ncu command recorded"
        for l in cmds:
            assert "--clock-control none" in l, (f, l)
        for script in re.findall(r"python\s+(\S+\.py)", text):
            assert os.path.exists(os.path.join(bench.ROOT, script)), (f, script)
