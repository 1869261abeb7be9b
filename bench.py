"""Benchmark of one NOSA sparse-decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload llama] [--impl reference]

One step = append -> pooled block scores -> dual selection -> (gather) -> split-K
attention + combine for every GQA group of the workload, through the C ABI
(nosa_step). Default workload: a Llama-3.1-8B-shaped attention layer (B=16,
Hq=32, Hkv=8, d=128, T=32768, block 64, sub-block 16, k=64 with k_q=16 and
k_e=48, 8 planted high-affinity blocks per group), synthetic seeded inputs.

Printed: one JSON line. `value` is queries/s (query-head vectors, B*Hq per
step, summed over ranks) from CUDA-event time of the timed steps, inputs
resident in HBM, L2 flushed before every timed step (256 MiB written, then
256 MiB read so the write-back of dirty lines happens before the timed region). `e2e` is
the same metric with each step's inputs copied from pinned host memory and the
outputs copied back inside the timed region (on a copy stream, double-buffered, so the
copies of neighbouring steps overlap a step's compute). `roofline` is for the attention
kernel (the largest share of the step), `cpu_baseline` times the fp64 oracle on
a bounded sample of the same workload on this host's cores.

--impl reference times the oracle itself (the only reference implementation
that exists for this method) and prints the same JSON line with impl=reference.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import nosa_synth as syn  # noqa: E402

METRIC = "sparse decode attn: queries/s, step µs, achieved HBM GB/s (% of peak)"
L2_FLUSH_BYTES = 256 << 20


def workload(name: str, steps: int, batch: int = 0) -> syn.NosaConfig:
    base = syn.configs()[name]
    if batch:  # smaller batch of the same layer (profiling captures)
        base = base.with_(B=batch, T=base.T[:1] * batch)
    return base.with_(steps=steps)


def describe(cfg: syn.NosaConfig) -> str:
    return (f"{cfg.name}: B={cfg.B} Hq={cfg.Hq} Hkv={cfg.Hkv} d={cfg.d} T={cfg.T[0]} "
            f"block={cfg.block} sub_block={cfg.sub_block} k={cfg.k} (k_q={cfg.k_q}, k_e={cfg.k_e})"
            + (f" slots={cfg.slots} offload" if cfg.offload else " all KV in HBM")
            + (f" score_mode={cfg.score_mode}" if cfg.score_mode else "")
            + (f" stop_tau={cfg.stop_tau}" if cfg.stop_tau else "")
            + (" kc=bf16" if cfg.kc_bf16 else ""))


def step_bytes(cfg: syn.NosaConfig, L: int, misses: int = 0, visited: float = None):
    """Algorithmic bytes of one step at context length L (after the append), per step.

    `misses`: pages (K and V each) the step copied from host memory; each is read over PCIe
    once and written to HBM once. Returns (total HBM, attention kernel, score/select kernel,
    PCIe)."""
    NG, G, d, bs = cfg.B * cfg.Hkv, cfg.G, cfg.d, cfg.block
    N = -(-L // bs)
    M = -(-L // cfg.sub_block)
    nsel = min(cfg.k, N)
    if visited is not None:  # early stop: pages actually streamed per group
        nsel = min(nsel, visited)
    tail_tokens = L - (N - 1) * bs
    # K and V of the selected blocks; the tail block (always among them once k >= N) at its
    # present tokens only when it is selected -- counted as full pages otherwise
    kv = nsel * bs * d * 2 * 2
    attn = NG * (kv + G * d * 2 + G * d * 4 + cfg.k * 4 + cfg.k * 4)
    score = NG * (M * d * (2 if cfg.kc_bf16 else 4) + N * 4 + 2 * 2 * 4 * (-(-N // 32)) + cfg.rows * d * 2
                  + 2 * d * 2 + N * 4 * 2 + cfg.k * 4)
    page = bs * d * 2
    return attn + score + misses * 2 * page, attn, score, misses * 2 * page


def pcie_ceiling(nosa, torch, mib: int = 256, reps: int = 5):
    """PCIe read ceiling: best rate of the library's plain UVA read probe (16-byte loads from
    pinned host memory, the gather's access) over `mib` MiB, CUDA events."""
    n = mib << 20
    h = torch.empty(n, dtype=torch.uint8).pin_memory()
    dv = torch.empty(n, dtype=torch.uint8, device="cuda")
    rates = []
    for i in range(reps + 1):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        nosa.uva_read_probe(h, dv, n)
        b.record()
        torch.cuda.synchronize()
        if i:
            rates.append(n / (a.elapsed_time(b) / 1e3) / 1e9)
    return max(rates)


class Clocks:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.p = None
        self.path = os.path.join("/tmp", f"nosa_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            self.f = open(self.path, "w")
            self.p = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                                       "--format=csv,noheader,nounits", "-lms", "100"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.p = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.p is not None:
            time.sleep(0.2)
            self.p.terminate()
            self.p.wait()
            self.f.close()

    def summary(self):
        if self.p is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


def kernel_source_sha(root: str = None) -> str:
    """sha256 of the attention kernel's source (the files a traffic record was captured from)."""
    import hashlib
    h = hashlib.sha256()
    for f in ("nosa_attn.cuh", "nosa_common.cuh"):
        h.update(open(os.path.join(root or ROOT, "kv_cache_offload_nosa_b200", "csrc", f), "rb").read())
    return h.hexdigest()


def attn_traffic(batch: int):
    """DRAM bytes per attention launch from the committed traffic record
    (profiles/attn_traffic.json, written from one ncu capture), scaled from its batch to
    `batch` (traffic grows with the number of groups); None when the record is missing or the
    kernel source changed since the capture."""
    p = os.path.join(ROOT, "profiles", "attn_traffic.json")
    if not os.path.exists(p):
        return None
    rec = json.load(open(p))
    if rec.get("source_sha256") != kernel_source_sha():
        return None
    return int(rec["dram_bytes_per_launch"]) * batch / int(rec["batch"])


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        j = json.load(open(p))
        return float(j["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# ----------------------------------------------------------------------------- CPU oracle
def _omp(fn: str, *a):
    """Calls libgomp (the OpenMP runtime the oracle's parallel regions use) in this process."""
    import ctypes
    try:
        return getattr(ctypes.CDLL("libgomp.so.1"), fn)(*a)
    except (OSError, AttributeError):
        return None


def oracle_sample(cfg: syn.NosaConfig, steps: int, budget_s: float = 20.0, batch: int = 2,
                  min_steps: int = 3):
    """Times the fp64 oracle (append, score, select, residency, attention) on a bounded
    sample of the workload: the first `batch` entries of the same layer, decode steps until
    `budget_s` of oracle time (at least `min_steps`, at most `steps`)."""
    import oracle as O
    B_s = max(1, min(cfg.B, batch))
    sub = cfg.with_(name=cfg.name + "_sample", B=B_s, T=cfg.T[:B_s], steps=steps)
    inp = syn.make_inputs(sub)
    orc = O.Oracle(sub, inp.pool_k, inp.pool_v, inp.resident)
    prev = None
    zero = np.zeros((sub.B, sub.Hkv), np.int64)
    times = []
    for t in range(steps):
        prev = syn.query_step(sub, t, prev, zero)
        q16 = syn.round_bf16(prev)
        t0 = time.perf_counter()
        orc.append(inp.k_new[t], inp.v_new[t])
        rows = q16.reshape(sub.B, sub.Hkv, sub.G, sub.d)
        sc = orc.block_scores(rows)
        sel, _, _ = orc.select(sc, inp.evict[t])
        orc.residency(sel)
        orc.attend(q16, sel)
        times.append(time.perf_counter() - t0)
        if len(times) >= min_steps and sum(times) > budget_s:
            break
    n = len(times)
    tot = sum(times)
    cores = _omp("omp_get_max_threads") or int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return {"value": sub.B * sub.Hq * n / tot, "unit": "queries/s", "cores": cores, "kind": "oracle",
            "sample": f"{n} decode steps of {B_s} of {cfg.B} batch entries of the same layer "
                      f"(fp64 C oracle, OpenMP over groups), {tot:.2f} s"}, times


def cpu_baseline(args):
    """The oracle on this host: all cores (OpenMP over groups) for about `cpu_budget` seconds
    of oracle time, then one thread for about a third of that."""
    budget = min(args.cpu_budget, 3.0)
    cfg = workload(args.workload, 400)
    cb, _ = oracle_sample(cfg, 400, budget_s=budget, batch=4)
    cores = cb["cores"]
    _omp("omp_set_num_threads", 1)
    one, _ = oracle_sample(cfg, 400, budget_s=budget / 3, batch=4, min_steps=2)
    _omp("omp_set_num_threads", int(cores))
    if one["cores"] == 1:  # the runtime took the one-thread setting
        cb["one_thread"] = {"value": one["value"], "unit": one["unit"], "cores": 1,
                            "sample": one["sample"]}
    return cb


def run_reference(args, cfg):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    steps = args.warmup + args.steps
    res, times = oracle_sample(cfg, steps, budget_s=1e9)
    timed = times[args.warmup:]
    B_s = max(1, min(cfg.B, 2))
    val = B_s * cfg.Hq * len(timed) / sum(timed)
    cb = dict(res)
    cb["value"] = val
    cb["sample"] = f"{len(timed)} timed decode steps (+{args.warmup} warm-up) of {B_s} of {cfg.B} batch entries"
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "queries/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * sum(timed) / len(timed), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": describe(cfg), "sample_batch": B_s},
            "cpu_baseline": cb,
            "e2e": {"value": val, "unit": "queries/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- GPU arm
def measure_gpu(args, cfg, rank, world, local):
    """Times nosa_step on the workload `cfg` (args: steps, warmup, e2e_steps, launch); returns
    the JSON line's fields on rank 0, None on the other ranks."""
    import torch
    import kv_cache_offload_nosa_b200 as nosa
    from kv_cache_offload_nosa_b200 import dist as D

    # each rank is an independent replica with its own seeded batch (weak scaling)
    if world > 1:
        cfg = cfg.with_(cfg_id=cfg.cfg_id + 1000 * rank)
    n_e2e = args.e2e_steps
    n_prof = 3
    total_steps = args.warmup + 1 + args.steps + n_prof + n_e2e
    cfg = cfg.with_(steps=total_steps)
    inp = syn.make_inputs(cfg)
    NG = cfg.B * cfg.Hkv
    cc = nosa.make_config(cfg.B, cfg.Hq, cfg.Hkv, cfg.d, cfg.block, cfg.sub_block, cfg.k_q, cfg.k_e,
                          cfg.max_blocks, slots=cfg.n_slots, n_score_rows=cfg.rows, scale=cfg.scale, score_mode=cfg.score_mode,
                          stop_tau=cfg.stop_tau, kc_bf16=cfg.kc_bf16)
    cache = nosa.NosaCache(cc, offload=cfg.offload)
    n_kernels = nosa.step_launches(cc, cache.state)  # kernels per nosa_step
    pk = torch.from_numpy(inp.pool_k.reshape(NG, cfg.max_blocks, cfg.block, cfg.d)).view(torch.int16)
    pv = torch.from_numpy(inp.pool_v.reshape(NG, cfg.max_blocks, cfg.block, cfg.d)).view(torch.int16)
    resident = None
    if cfg.offload:
        cache.pool_view("host_k").copy_(pk)
        cache.pool_view("host_v").copy_(pv)
        resident = torch.from_numpy(inp.resident.reshape(NG, -1)).cuda()
    else:
        cache.pool_view("k_pool").copy_(pk)
        cache.pool_view("v_pool").copy_(pv)
    del pk, pv
    inp.pool_k = inp.pool_v = None
    plen = torch.tensor(cfg.T, dtype=torch.int32, device="cuda")
    cache.init(plen, resident)
    if cfg.offload:
        # the first launch of each kernel loads its module: do that on a small cache of the same
        # shapes so that step 0 below is timed without it
        small = syn.configs()["offload_small"].with_(steps=2)
        si = syn.make_inputs(small)
        sc = nosa.make_config(small.B, small.Hq, small.Hkv, small.d, small.block, small.sub_block,
                              small.k_q, small.k_e, small.max_blocks, slots=small.n_slots,
                              n_score_rows=small.rows, scale=small.scale)
        scache = nosa.NosaCache(sc, offload=True)
        sng = small.B * small.Hkv
        scache.pool_view("host_k").copy_(torch.from_numpy(si.pool_k.reshape(sng, small.max_blocks, small.block, small.d)).view(torch.int16))
        scache.pool_view("host_v").copy_(torch.from_numpy(si.pool_v.reshape(sng, small.max_blocks, small.block, small.d)).view(torch.int16))
        scache.init(torch.tensor(small.T, dtype=torch.int32, device="cuda"),
                    torch.from_numpy(si.resident.reshape(sng, -1)).cuda())
        sq = torch.from_numpy(syn.round_bf16(syn.query_step(small, 0, None, np.zeros((small.B, small.Hkv), np.int64)))).view(torch.int16).cuda()
        scache.step(sq, torch.from_numpy(si.k_new[0]).view(torch.int16).cuda(),
                    torch.from_numpy(si.v_new[0]).view(torch.int16).cuda(), torch.from_numpy(si.evict[0]).cuda(),
                    torch.empty(sng * small.k, dtype=torch.int32, device="cuda"),
                    torch.empty(small.B * small.Hq * small.d, dtype=torch.float32, device="cuda"),
                    torch.empty(sng, dtype=torch.int32, device="cuda"))
        torch.cuda.synchronize()
        del scache
    # per-step inputs (queries follow the workload's process, no margin redraws)
    prev, zero = None, np.zeros((cfg.B, cfg.Hkv), np.int64)
    qs = []
    for t in range(total_steps):
        prev = syn.query_step(cfg, t, prev, zero)
        qs.append(syn.round_bf16(prev))
    h_q = torch.from_numpy(np.stack(qs)).view(torch.int16)
    h_kn = torch.from_numpy(inp.k_new).view(torch.int16)
    h_vn = torch.from_numpy(inp.v_new).view(torch.int16)
    h_ev = torch.from_numpy(inp.evict)
    def per_step(x):
        # one row per step, each row starting on a 16-byte boundary (the library's alignment)
        flat = x.reshape(x.shape[0], -1)
        n = flat.shape[1]
        per = 16 // flat.element_size()
        d = torch.zeros((flat.shape[0], -(-n // per) * per), dtype=flat.dtype, device="cuda")
        d[:, :n].copy_(flat)
        return d[:, :n]

    d_q, d_kn, d_vn, d_ev = (per_step(x) for x in (h_q, h_kn, h_vn, h_ev))
    sel = torch.empty(NG * cfg.k, dtype=torch.int32, device="cuda")
    out = torch.empty(cfg.B * cfg.Hq * cfg.d, dtype=torch.float32, device="cuda")
    # every step writes its miss counts to its own row (nothing extra runs in the timed region)
    # (rows padded to 16 bytes: the library wants 16-byte aligned buffers)
    miss_all = torch.zeros((total_steps, -(-NG // 4) * 4), dtype=torch.int32, device="cuda")
    # L2 flush between timed steps: write a buffer larger than L2, then read another one so
    # the dirty lines are written back before the timed region starts, not inside it
    flush_w = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    flush_r = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    flush_sink = torch.empty(1, dtype=torch.float32, device="cuda")

    class _Flush:
        @staticmethod
        def zero_():
            flush_w.zero_()
            torch.sum(flush_r, dim=0, out=flush_sink)

    flush = _Flush()
    stream = torch.cuda.current_stream()

    def do_step(t, events=None):
        cache.step(d_q[t], d_kn[t], d_vn[t], d_ev[t], sel, out, miss_all[t, :NG], stream=stream, events=events)

    # graph launch: the step is captured once (after step 0 has loaded its kernels) and
    # replayed; each step's inputs are first copied into the graph's input buffers and its
    # miss counts copied out afterwards, both outside the timed region
    sg = None

    def stage(t):
        if sg is not None:
            sg.stage(d_q[t], d_kn[t], d_vn[t], d_ev[t])

    def launch(t):
        if sg is not None:
            sg.replay()
        else:
            do_step(t)

    def collect(t):
        if sg is not None:
            miss_all[t, :NG].copy_(sg.miss[:NG])

    t = 0
    # step 0 (S(-1) = every prefill block; with offload, the initial residency misses) is the
    # first warm-up step, timed on its own
    s0, e0_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    flush.zero_()
    s0.record(stream)
    do_step(t)
    e0_.record(stream)
    t += 1
    torch.cuda.synchronize()
    launch_note = "direct launches"
    if args.launch == "graph":
        from kv_cache_offload_nosa_b200.graph import StepGraph
        try:
            sg = StepGraph(cache)
            launch_note = ("cuda graph: one captured nosa_step replayed per step, inputs staged "
                           "into its buffers before the timed region")
        except Exception as e:  # capture refused: time the same kernels launched directly
            sg = None
            launch_note = f"direct launches (graph capture failed: {type(e).__name__}: {str(e)[:120]})"
            torch.cuda.synchronize()
    for _ in range(args.warmup - 1):
        stage(t)
        launch(t)
        collect(t)
        t += 1
    torch.cuda.synchronize()
    step0_ms = s0.elapsed_time(e0_)
    torch.cuda.synchronize()
    rc, err = cache.check()
    if rc != 0:
        raise RuntimeError(f"device fault after warm-up: rc={rc} err={err}")
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    Ls = []
    D.barrier()
    torch.cuda.synchronize()
    with Clocks(local) as clk:
        # the clock sampler's start leaves the GPU idle for a moment: one more untimed step
        # brings the clocks back up before the timed ones
        stage(t)
        flush.zero_()
        launch(t)
        collect(t)
        t += 1
        for i in range(args.steps):
            stage(t)
            flush.zero_()
            starts[i].record(stream)
            launch(t)
            ends[i].record(stream)
            collect(t)
            Ls.append((cfg.T[0] + t + 1, t))
            t += 1
        torch.cuda.synchronize()
    D.barrier()
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    tot_ms = sum(step_ms)
    # per-kernel times of the same step (instrumented steps, events between kernels)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n_prof)]
    for e4 in evs:
        for e in e4:
            e.record(stream)
    torch.cuda.synchronize()
    prof_L = []
    for i in range(n_prof):
        flush.zero_()
        do_step(t, events=evs[i])
        prof_L.append((cfg.T[0] + t + 1, t))
        t += 1
    torch.cuda.synchronize()
    k_score = [e[0].elapsed_time(e[1]) for e in evs]
    k_gather = [e[1].elapsed_time(e[2]) for e in evs]
    k_attn = [e[2].elapsed_time(e[3]) for e in evs]
    # end to end: every step's inputs come from pinned host memory and its outputs go back to
    # pinned host memory, inside the timed region. Each step's inputs sit packed in one pinned
    # buffer (one host->device copy) and the library writes the step's outputs into views of
    # one device buffer (one device->host copy). The copies run on their own stream with two
    # device buffer sets, so step i computes while step i+1's inputs come in and step i-1's
    # outputs go out (each step still waits for its own inputs); inputs and outputs travel on
    # separate streams so that both copy engines work.
    parts = (h_q, h_kn, h_vn, h_ev)
    sizes = [x[0].numel() * x.element_size() for x in parts]
    offs = [0]
    for nb_ in sizes:
        offs.append(offs[-1] + -(-nb_ // 256) * 256)
    in_bytes = offs[-1]
    h_in = torch.empty((n_e2e, in_bytes), dtype=torch.uint8).pin_memory()
    for i in range(n_e2e):
        for x, o, nb_ in zip(parts, offs, sizes):
            h_in[i, o:o + nb_].copy_(x[t + i].reshape(-1).view(torch.uint8))
    o_sizes = [out.numel() * 4, sel.numel() * 4, NG * 4]
    o_offs = [0]
    for nb_ in o_sizes:
        o_offs.append(o_offs[-1] + -(-nb_ // 256) * 256)
    out_bytes = o_offs[-1]
    h_out = torch.empty(out_bytes, dtype=torch.uint8).pin_memory()
    dev_in = [torch.empty(in_bytes, dtype=torch.uint8, device="cuda") for _ in range(2)]
    dev_out = [torch.empty(out_bytes, dtype=torch.uint8, device="cuda") for _ in range(2)]

    def in_views(buf):
        return [buf[o:o + nb_].view(x.dtype).view(x[0].shape) for x, o, nb_ in zip(parts, offs, sizes)]

    def out_views(buf):
        return (buf[o_offs[0]:o_offs[0] + o_sizes[0]].view(torch.float32),
                buf[o_offs[1]:o_offs[1] + o_sizes[1]].view(torch.int32),
                buf[o_offs[2]:o_offs[2] + o_sizes[2]].view(torch.int32))
    views_in = [in_views(b) for b in dev_in]      # built once, outside the timed region
    views_out = [out_views(b) for b in dev_out]

    def e2e_step(k):
        bq, bk, bv, be = views_in[k]
        o_dev, s_dev, m_dev = views_out[k]
        cache.step(bq, bk, bv, be, s_dev, o_dev, m_dev, stream=torch.cuda.current_stream())

    e2e_graphs = None
    if sg is not None:
        # one captured step per buffer set (capture records the launches, nothing runs)
        e2e_graphs = []
        for k in range(2):
            g = torch.cuda.CUDAGraph()
            torch.cuda.synchronize()
            with torch.cuda.graph(g, capture_error_mode="relaxed"):
                e2e_step(k)
            e2e_graphs.append(g)
    h2d_done = [torch.cuda.Event() for _ in range(2)]
    step_done = [torch.cuda.Event() for _ in range(2)]
    d2h_done = [torch.cuda.Event() for _ in range(2)]
    hs, ds = torch.cuda.Stream(), torch.cuda.Stream()  # inputs in, outputs out: two copy engines
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    hs.wait_stream(stream)
    ds.wait_stream(stream)
    with torch.cuda.stream(hs):
        dev_in[0].copy_(h_in[0], non_blocking=True)
        h2d_done[0].record(hs)
    for i in range(n_e2e):
        k = i % 2
        if i + 1 < n_e2e:
            with torch.cuda.stream(hs):
                if i >= 1:
                    hs.wait_event(step_done[1 - k])  # step i-1 has read buffer set 1-k
                dev_in[1 - k].copy_(h_in[i + 1], non_blocking=True)
                h2d_done[1 - k].record(hs)
        stream.wait_event(h2d_done[k])
        if i >= 2:
            stream.wait_event(d2h_done[k])  # step i-2's outputs have left buffer set k
        if e2e_graphs is not None:
            e2e_graphs[k].replay()
        else:
            e2e_step(k)
        step_done[k].record(stream)
        with torch.cuda.stream(ds):
            ds.wait_event(step_done[k])
            h_out.copy_(dev_out[k], non_blocking=True)
            d2h_done[k].record(ds)
        t += 1
    stream.wait_stream(ds)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / n_e2e
    rc, err = cache.check()
    if rc != 0:
        raise RuntimeError(f"device fault in timed steps: rc={rc} err={err}")

    misses = miss_all.sum(dim=1).cpu().numpy()  # K (and V) pages copied per step
    visited = None
    if cfg.stop_tau > 0:
        # early stop: a group streams the blocks its most persistent head visits (counts of
        # the last step, taken as representative of the timed ones)
        used = torch.empty(cfg.B * cfg.Hq, dtype=torch.int32, device="cuda")
        cache.stop_counts(used)
        per_group = used.view(cfg.B * cfg.Hkv, cfg.G).max(dim=1).values.float()
        visited = float(per_group.mean().item())
    pcie_peak = pcie_ceiling(nosa, torch) if cfg.offload else None
    # max over ranks
    tot_ms, e2e_ms = D.max_over_ranks([tot_ms, e2e_ms], device="cuda")
    if rank != 0:
        return None
    q_per_step = cfg.B * cfg.Hq * world
    value = q_per_step * args.steps / (tot_ms / 1e3)
    hbm_peak, peak_kind = peaks()
    step_b = [step_bytes(cfg, L, int(misses[ti]), visited)[0] for L, ti in Ls]
    pcie_b = [step_bytes(cfg, L, int(misses[ti]))[3] for L, ti in Ls]
    hbm_gbs = sum(step_b) / (tot_ms / 1e3) / 1e9
    attn_b = [step_bytes(cfg, L, 0, visited)[1] for L, _ in prof_L]
    attn_ms = float(np.mean(k_attn))
    achieved = float(np.mean(attn_b)) / (attn_ms / 1e3) / 1e9
    roof = {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
            "frac": achieved / hbm_peak, "traffic": attn_traffic(cfg.B) if cfg.name == "llama" else None,
            "kernel": "attn_stop_kernel" if cfg.stop_tau > 0 else "attn_kernel", "peak_kind": peak_kind,
            "bytes_per_launch": float(np.mean(attn_b))}
    pcie = None
    if cfg.offload:
        # the step is bound by the slower of its HBM bytes at the HBM peak and its PCIe bytes
        # at the UVA read ceiling; when PCIe is slower the gather kernel is the dominant one
        t_hbm = float(np.mean(step_b)) / (hbm_peak * 1e9)
        t_pcie = float(np.mean(pcie_b)) / (pcie_peak * 1e9)
        gather_pcie = [step_bytes(cfg, L, int(misses[ti]))[3] for L, ti in prof_L]
        g_ms = float(np.mean(k_gather))
        pcie = {"bytes_per_step": float(np.mean(pcie_b)), "pages_per_step": float(np.mean([misses[ti] for _, ti in Ls])),
                "step0_pages": int(misses[0]), "probe_gbs": pcie_peak,
                "gather_gbs": float(np.mean(gather_pcie)) / (g_ms / 1e3) / 1e9 if g_ms > 0 else None,
                "step_bound_us": 1e6 * max(t_hbm, t_pcie), "step_bound": "pcie" if t_pcie > t_hbm else "hbm",
                "step_frac": 1e6 * max(t_hbm, t_pcie) / (1e3 * tot_ms / args.steps)}
        if t_pcie > t_hbm and pcie["gather_gbs"]:
            roof = {"bound": "pcie", "achieved": pcie["gather_gbs"], "peak": pcie_peak, "unit": "GB/s",
                    "frac": pcie["gather_gbs"] / pcie_peak, "traffic": None, "kernel": "copy_kernel",
                    "peak_kind": "measured (UVA read probe, this run)",
                    "bytes_per_launch": float(np.mean(gather_pcie))}
    clocks = clk.summary()
    h2d = sum(sizes)
    d2h = sum(o_sizes)
    line = {
        "metric": METRIC, "value": value, "unit": "queries/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": tot_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": describe(cfg), "global_batch": cfg.B * world, "seq_len": cfg.T[0],
                   "parallelism": f"replicas x{world} (batch-sharded, no collective)",
                   "l2": "flushed before every timed step (256 MiB write, then 256 MiB read so no dirty line is written back inside the timed region)",
                   "queries_per_step": q_per_step},
        "launch": launch_note,
        "tokens_per_s": cfg.B * world * args.steps / (tot_ms / 1e3),
        "step_us": 1e3 * tot_ms / args.steps,
        "step_us_median": 1e3 * float(np.median(step_ms)),
        "step_us_pct": {f"p{q}": 1e3 * float(np.percentile(step_ms, q)) for q in (0, 10, 50, 90, 100)},
        "hbm_gbs": hbm_gbs, "hbm_frac": hbm_gbs / hbm_peak,
        "bytes_per_step": float(np.mean(step_b)),
        "kernel_us": {"score_select": 1e3 * float(np.mean(k_score)),
                      "gather": 1e3 * float(np.mean(k_gather)), "attention": 1e3 * attn_ms},
        "step_kernels": n_kernels,
        "roofline": roof,
        "step0_us": 1e3 * step0_ms,
        "e2e": {"value": q_per_step / (e2e_ms / 1e3), "unit": "queries/s", "steps": n_e2e,
                "overlap": "inputs of step i+1 and outputs of step i-1 copied during step i",
                "l2": "not flushed: every step reads more than L2 holds",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": args.steps * n_kernels,
        "clocks": clocks,
    }
    if pcie is not None:
        line["pcie"] = pcie
    if visited is not None:
        line["early_stop"] = {"tau": cfg.stop_tau, "blocks_streamed_per_group": visited, "k": cfg.k,
                              "kernel": "attn_stop_kernel (one CTA per group)"}
    return line


# ----------------------------------------------------------------------------- lookahead
def measure_lookahead(args, cfg, rank, world, local):
    """Tokens through `--layers` offload layers (independent caches of the workload's shape):
    SparDA's lookahead pipeline (plans ahead, layer-ordered copies on their own stream,
    attention after each layer's copies) against the same layers stepped one after another
    with nosa_step. Reports both token times and the time the pipeline hides."""
    import torch
    import kv_cache_offload_nosa_b200 as nosa
    from kv_cache_offload_nosa_b200 import dist as D
    from kv_cache_offload_nosa_b200.lookahead import LookaheadPipeline

    nl = args.layers
    total = 2 * (args.warmup + args.steps) + 1
    cfgs = [cfg.with_(cfg_id=cfg.cfg_id + 1000 * l + 100000 * rank, steps=total) for l in range(nl)]
    NG = cfg.B * cfg.Hkv
    caches, ins = [], []
    for c in cfgs:
        inp = syn.make_inputs(c)
        cc = nosa.make_config(c.B, c.Hq, c.Hkv, c.d, c.block, c.sub_block, c.k_q, c.k_e, c.max_blocks,
                              slots=c.n_slots, n_score_rows=c.rows, scale=c.scale, score_mode=c.score_mode)
        cache = nosa.NosaCache(cc, offload=True)
        cache.pool_view("host_k").copy_(torch.from_numpy(inp.pool_k.reshape(NG, c.max_blocks, c.block, c.d)).view(torch.int16))
        cache.pool_view("host_v").copy_(torch.from_numpy(inp.pool_v.reshape(NG, c.max_blocks, c.block, c.d)).view(torch.int16))
        inp.pool_k = inp.pool_v = None
        cache.init(torch.tensor(c.T, dtype=torch.int32, device="cuda"),
                   torch.from_numpy(inp.resident.reshape(NG, -1)).cuda())
        zero = np.zeros((c.B, c.Hkv), np.int64)
        qs, prev = [], None
        for t in range(total):
            prev = syn.query_step(c, t, prev, zero)
            qs.append(syn.round_bf16(prev))
        fc = np.stack([syn.round_bf16(syn.forecast_step(c, t, zero)) for t in range(total)])
        ins.append({"q": torch.from_numpy(np.stack(qs)).view(torch.int16).cuda(),
                    "f": torch.from_numpy(fc).view(torch.int16).cuda(),
                    "kn": torch.from_numpy(inp.k_new).view(torch.int16).cuda(),
                    "vn": torch.from_numpy(inp.v_new).view(torch.int16).cuda(),
                    "ev": torch.from_numpy(inp.evict).cuda()})
        caches.append(cache)
    sel = [torch.empty(NG * cfg.k, dtype=torch.int32, device="cuda") for _ in range(nl)]
    out = [torch.empty(cfg.B * cfg.Hq * cfg.d, dtype=torch.float32, device="cuda") for _ in range(nl)]
    miss = torch.zeros((total, nl, -(-NG // 4) * 4), dtype=torch.int32, device="cuda")
    flush_w = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    flush_r = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    flush_sink = torch.empty((), dtype=torch.float32, device="cuda")
    pipe = LookaheadPipeline(caches)
    stream = torch.cuda.current_stream()

    def pipelined(t):
        pipe.token([x["f"][t] for x in ins], [x["ev"][t] for x in ins], [x["q"][t] for x in ins],
                   [x["kn"][t] for x in ins], [x["vn"][t] for x in ins], sel,
                   [miss[t, l, :NG] for l in range(nl)], out, stream=stream)

    def serial(t):
        for l, (c, x) in enumerate(zip(caches, ins)):
            c.step(x["q"][t], x["kn"][t], x["vn"][t], x["ev"][t], sel[l], out[l], miss[t, l, :NG],
                   score_rows=x["f"][t], stream=stream)

    def timed(fn, t0, n):
        ms = []
        for i in range(n):
            flush_w.zero_()
            torch.sum(flush_r, dim=0, out=flush_sink)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn(t0 + i)
            b.record(stream)
            torch.cuda.synchronize()
            ms.append(a.elapsed_time(b))
        return ms

    t = 0
    timed(pipelined, t, args.warmup)
    t += args.warmup
    D.barrier()
    with Clocks(local) as clk:
        timed(pipelined, t, 1)  # the sampler's start left the GPU idle: one untimed token first
        t += 1
        pipe_ms = timed(pipelined, t, args.steps)
    t += args.steps
    pipe_misses = miss[t - args.steps:t].sum().item()
    timed(serial, t, args.warmup)
    t += args.warmup
    ser_ms = timed(serial, t, args.steps)
    ser_misses = miss[t - args.steps:t].sum().item()
    for c in caches:
        rc, err = c.check()
        if rc != 0:
            raise RuntimeError(f"device fault: rc={rc} err={err}")
    pcie_peak = pcie_ceiling(nosa, torch)
    tok_ms, ser_tok_ms = D.max_over_ranks([float(np.sum(pipe_ms)), float(np.sum(ser_ms))], device="cuda")
    if rank != 0:
        return None
    tok = tok_ms / args.steps
    ser = ser_tok_ms / args.steps
    page = cfg.block * cfg.d * 2
    pcie_tok = pipe_misses / args.steps * 2 * page      # bytes per token (all layers)
    q_tok = cfg.B * cfg.Hq * nl * world
    line = {
        "metric": METRIC, "value": q_tok / (tok / 1e3), "unit": "queries/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": tok / nl, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": describe(cfg) + f" x {nl} layers, lookahead pipeline (forecast row per group)",
                   "global_batch": cfg.B * world, "seq_len": cfg.T[0], "layers": nl,
                   "parallelism": f"replicas x{world} (batch-sharded, no collective)",
                   "l2": "flushed before every timed token (256 MiB write, then 256 MiB read)"},
        "token_us": 1e3 * tok, "serial_token_us": 1e3 * ser, "hidden_us": 1e3 * (ser - tok),
        "speedup_vs_serial": ser / tok,
        "pcie": {"bytes_per_token": pcie_tok, "probe_gbs": pcie_peak,
                 "bound_token_us": 1e6 * pcie_tok / (pcie_peak * 1e9),
                 "frac": 1e6 * pcie_tok / (pcie_peak * 1e9) / (1e3 * tok),
                 "serial_pages_per_token": ser_misses / args.steps,
                 "pipelined_pages_per_token": pipe_misses / args.steps},
        "gpu_launches": args.steps * nl * 4,
        "clocks": clk.summary(),
    }
    return line


# ----------------------------------------------------------------------------- driver
# Workloads measured after the headline in the same process (one GPU only), each at a few
# steps: every configuration of the decode step besides the headline layer.
PER_CONFIG = ("tiny", "offload", "sink", "sweep_T65536_b64_p1", "sweep_T65536_b64_p5",
              "sweep_T65536_b64_p10", "llama_stop", "llama_kc16", "lookahead")


def summarize(name: str, line: dict) -> dict:
    """The per-configuration entry: step time, queries/s and the HBM (or PCIe) fraction."""
    if name == "lookahead":
        keys = ("token_us", "serial_token_us", "hidden_us", "speedup_vs_serial", "pcie")
        e = {"workload": line["config"]["workload"], "queries_per_s": line["value"]}
        e.update({k: line[k] for k in keys})
        return e
    e = {"workload": line["config"]["workload"], "step_us": line["step_us"],
         "step_us_median": line["step_us_median"], "queries_per_s": line["value"],
         "hbm_gbs": line["hbm_gbs"], "hbm_frac": line["hbm_frac"], "bytes_per_step": line["bytes_per_step"],
         "kernel_us": line["kernel_us"], "roofline_frac": line["roofline"]["frac"],
         "roofline_kernel": line["roofline"]["kernel"], "step0_us": line["step0_us"],
         "launch": line["launch"], "clocks": line["clocks"], "step_kernels": line["step_kernels"]}
    for k in ("pcie", "early_stop"):
        if k in line:
            e[k] = line[k]
    return e


def per_config(args, rank, world, local):
    import copy
    import torch
    out = {}
    for name in PER_CONFIG:
        a = copy.copy(args)
        a.steps, a.warmup, a.e2e_steps = args.per_config_steps, 3, 4
        a.no_cpu_baseline = True
        cfg = workload(name, a.warmup + a.steps)
        t0 = time.perf_counter()
        try:
            fn = measure_lookahead if name == "lookahead" else measure_gpu
            line = fn(a, cfg, rank, world, local)
            out[name] = summarize(name, line)
        except Exception as e:  # one configuration's failure must not lose the headline line
            out[name] = {"error": f"{type(e).__name__}: {str(e)[:300]}"}
        out[name]["wall_s"] = time.perf_counter() - t0
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
    return out


def run_gpu(args, cfg):
    import torch
    from kv_cache_offload_nosa_b200 import build as nb
    from kv_cache_offload_nosa_b200 import dist as D

    rank, world, local = D.rank_info()
    torch.cuda.set_device(local)
    D.init("nccl", timeout_s=300)
    nb.build()
    fn = measure_lookahead if cfg.name == "lookahead" else measure_gpu
    line = fn(args, cfg, rank, world, local)
    if rank == 0:
        torch.cuda.empty_cache()
        if cfg.name != "lookahead" and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(args)
        if world == 1 and args.per_config_steps > 0 and cfg.name == "llama" and not args.batch:
            line["per_config"] = per_config(args, rank, world, local)
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="llama")
    ap.add_argument("--batch", type=int, default=0, help="override the batch (profiling only)")
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-budget", type=float, default=20.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--layers", type=int, default=4, help="layers of the lookahead workload")
    ap.add_argument("--launch", default="graph", choices=["graph", "direct"],
                    help="timed steps as one replayed CUDA graph per step, or direct launches")
    ap.add_argument("--per-config-steps", type=int, default=10,
                    help="timed steps of each other workload measured after the headline "
                         "(one GPU, default workload only); 0 = none")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    cfg = workload(args.workload, args.warmup + args.steps, args.batch)
    if args.impl == "reference":
        run_reference(args, cfg)
    else:
        run_gpu(args, cfg)


if __name__ == "__main__":
    main()
