"""Benchmark of the VSA forward path on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload fastwan] [--impl ours|reference]

A step is one pass of the whole forward path over one batch of seeded
synthetic input: tile(q), tile(k) with pooled means, tile(v), block scores +
top-k, block-sparse attention, untile(o).  The metric is effective TFLOP/s
over the selected blocks (4 * D * bs^2 FLOPs per selected block pair), with
ms per step beside it.  ``value`` is timed with the inputs already in HBM;
``e2e`` times the same call with pinned host inputs copied in and o copied
back inside every step.

Several GPUs run independent replicas of the same workload (the path has no
exchange step); the time is the maximum over ranks and ``value`` counts the
work of all ranks.  ``--impl reference`` times the CPU oracle (rank 0 only)
on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_sparse_video_gather_b200 import workloads  # noqa: E402

PROFILE = os.path.join(ROOT, "profiles", "attn_fwd_fastwan.md")
ATTN_SOURCES = [os.path.join(ROOT, "block_sparse_video_gather_b200", "csrc", f)
                for f in ("attn_fwd.cu", "fwd_common.cuh", "common.cuh", "tiles.cuh")]
GROUPED_SOURCES = [os.path.join(ROOT, "block_sparse_video_gather_b200", "csrc", f)
                   for f in ("attn_fwd_grouped.cu", "fwd_common.cuh", "nvfp4.cuh", "common.cuh", "tiles.cuh")]
# committed ncu summaries that carry the DRAM traffic of one fine-stage launch:
# workload -> (summary, the kernel sources its source_hash covers)
TRAFFIC_PROFILES = {
    "fastwan": (PROFILE, ATTN_SOURCES),
    "tile64": (os.path.join(ROOT, "profiles", "attn_fwd_grouped64_tile64.md"), GROUPED_SOURCES),
}
FP4_PROFILE = os.path.join(ROOT, "profiles", "attn_fwd_fp4_fastwan.md")
FP4_SOURCES = [os.path.join(ROOT, "block_sparse_video_gather_b200", "csrc", f)
               for f in ("fp4.cu", "nvfp4.cuh", "common.cuh", "tiles.cuh")]
# NVFP4 fine stage: workload -> (summary, sources); 64-token plans run the grouped kernel's NVFP4 variant
FP4_TRAFFIC_PROFILES = {
    "fastwan": (FP4_PROFILE, FP4_SOURCES),
    "tile64": (os.path.join(ROOT, "profiles", "attn_fwd_fp4_grouped64_tile64.md"), GROUPED_SOURCES),
}
WORKLOAD_TEXT = {
    "tiny": "tiny grid 8x16x16, B1 H2 D128, block 4x8x8, topk 4",
    "fastwan": "FastWan2.2-TI2V-5B latent grid 31x22x40, B1 H24 D128, block 4x8x8, topk 64",
    "wan81": "Wan2.1-1.3B 81-frame latent grid 21x30x52, B1 H12 D128, block 4x8x8, topk 32",
    "long": "Wan2.1-1.3B 321-frame latent grid 81x30x52, B1 H12 D128, block 4x8x8, topk 59",
    "tile64": ("non-uniform rows, 64-token tiles: 512 prefix + video 16x32x32, B1 H24 D128, tile 4x4x4, "
               "computed selection: prefix query tiles dense, video query tiles the prefix + top-32 video tiles, "
               "5% rows forced empty"),
    "tile64map": ("non-uniform rows, 64-token tiles: 512 prefix + video 16x32x32, B1 H24 D128, tile 4x4x4, "
                  "caller bool block map (prefix rows dense, video rows prefix + 32 random, 5% rows empty)"),
}


def selected_flops(wl, num: np.ndarray) -> float:
    """4 * D * bs^2 per selected (query block, key block) pair, padding included."""
    return 4.0 * wl.D * wl.block_tokens ** 2 * float(np.asarray(num, dtype=np.int64).sum())


def uniform_flops(wl) -> float:
    return 4.0 * wl.D * wl.block_tokens ** 2 * wl.B * wl.H * wl.num_blocks * wl.topk


def block_real_tokens(wl) -> np.ndarray:
    """[NB] real (non-padding) tokens of each block: shape bookkeeping of the grid."""
    bt, bh, bw = wl.block
    nT, nH, nW = wl.grid_blocks
    grid = np.zeros((nT * bt, nH * bh, nW * bw), dtype=np.int64)
    grid[:wl.T, :wl.Hg, :wl.Wg] = 1
    video = grid.reshape(nT, bt, nH, bh, nW, bw).sum(axis=(1, 3, 5)).reshape(-1)
    bs = wl.block_tokens
    pre = [min(bs, wl.n_prefix - i * bs) for i in range(wl.n_prefix_blocks)]
    return np.concatenate([np.array(pre, dtype=np.int64), video])


def grouped_products(idx: np.ndarray, num: np.ndarray, NB: int) -> int:
    """Q-tile products the grouped 64-token fine stage executes (one 128-row Q
    tile against one 128-key tile, an S and a P V product): per group of four
    query blocks, each Q tile (blocks 0-1, 2-3) walks the union of its two
    selections two blocks per tile; a group whose lists repeat an id walks the
    four lists as given (two ids per tile) for every Q tile.  Ids outside
    [0, NB) are skipped and counts clamped, as the kernel does."""
    idx = np.asarray(idx, dtype=np.int64)
    num = np.clip(np.asarray(num, dtype=np.int64), 0, idx.shape[-1])
    total = 0
    for b in range(idx.shape[0]):
        for h in range(idx.shape[1]):
            for g0 in range(0, NB, 4):
                rows = list(range(g0, min(g0 + 4, NB)))
                cnts = [int(num[b, h, r]) for r in rows]
                lists = [[int(x) for x in idx[b, h, r, :c] if 0 <= x < NB] for r, c in zip(rows, cnts)]
                nq = (len(rows) + 1) // 2
                if any(len(set(lst)) != len(lst) for lst in lists):
                    total += nq * sum((c + 1) // 2 for c in cnts)
                    continue
                for q in range(nq):
                    union = set().union(*lists[2 * q:2 * q + 2])
                    total += (len(union) + 1) // 2
    return total


def real_token_flops(wl, idx: np.ndarray, num: np.ndarray) -> float:
    """4 * D * (real query tokens) * (real key tokens) summed over the selected
    (query block, key block) pairs: the work on real tokens only."""
    real = block_real_tokens(wl)
    idx = np.asarray(idx, dtype=np.int64)
    num = np.asarray(num, dtype=np.int64)
    pos = np.arange(idx.shape[-1])
    listed = (pos < num[..., None]) & (idx >= 0)
    keys = np.where(listed, real[np.clip(idx, 0, len(real) - 1)], 0).sum(axis=-1)  # [B,H,NB]
    return 4.0 * wl.D * float((keys * real[None, None, :]).sum())


def attn_source_hash(sources=None) -> str:
    h = hashlib.sha256()
    for f in sources or ATTN_SOURCES:
        h.update(open(f, "rb").read())
    return h.hexdigest()[:16]


def profile_traffic(workload: str, profile: str = PROFILE, sources=None):
    """DRAM bytes per attention launch from the committed ncu summary, or None when
    the summary is absent, for another workload, or older than the kernel source."""
    if not os.path.exists(profile):
        return None
    text = open(profile).read()
    m_src = re.search(r"source_hash:\s*([0-9a-f]+)", text)
    m_wl = re.search(r"bench_workload:\s*(\w+)", text)
    m_b = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    if not (m_src and m_wl and m_b) or m_src.group(1) != attn_source_hash(sources) or m_wl.group(1) != workload:
        return None
    return float(m_b.group(1))


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return d.get("bf16_tflops"), d.get("bf16_tflops_sustained"), d.get("hbm_gbs"), "measured"
    return 1590.0, 1400.0, 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in out.splitlines():
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for name, val in zip(names, parts[3:7]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


BAD_CLOCK_REASONS = {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}


def clocks_rejected(clocks) -> bool:
    """A timed region to measure again: a hardware or thermal slowdown was active,
    or the SM clock sat well below its maximum with no reason given (a clock lock
    left behind by another user).  sw_power_cap alone is kept."""
    if not clocks:
        return False
    if BAD_CLOCK_REASONS & set(clocks["reasons"]):
        return True
    return not clocks["reasons"] and bool(clocks["sm_max_mhz"]) and clocks["sm_mhz"] < 0.85 * clocks["sm_max_mhz"]


def sync_ranks(pg, device_sync=True):
    """Every rank reaches this point with its device idle (barrier between two
    device synchronisations; the barrier alone without a process group)."""
    if device_sync:
        import torch
        torch.cuda.synchronize()
    if pg:
        pg.barrier()
    if device_sync:
        import torch
        torch.cuda.synchronize()


def rank_max(x: float, pg, device="cuda") -> float:
    """The largest x over all ranks (x itself without a process group): each
    timed figure is the slowest rank's."""
    if not pg:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}: launch N>1 with torch.distributed.run")
    return world, rank, local


def run_reference(args, wl, world, rank):
    """The CPU oracle on a bounded sample of the workload (rank 0 only).

    A step is one head of the workload (heads taken in turn): the oracle's
    tile / pool / score / top-k (or the map compaction), NVFP4 quantisation when
    asked, attention on --ref-rows of that head's query rows drawn at random,
    and untile; its time is scaled to all heads and rows.  So each step costs
    about 1 / H of the front end plus a fixed number of attention rows, and the
    whole run stays within minutes."""
    if rank != 0:
        return
    import oracle
    g = oracle.geometry_of(wl)
    inp = workloads.make_inputs(wl)
    B, Hh = wl.B, wl.H
    head_rows = B * g.Sp
    rng = np.random.default_rng(1)
    sample_rows = min(head_rows, args.ref_rows)
    if wl.map_driven:
        _, num_all = oracle.map_to_index(inp["map"])
        flops = selected_flops(wl, num_all)
    elif wl.prefix_dense:
        qt_all, kt_all = oracle.tile(g, inp["q"]), oracle.tile(g, inp["k"])
        _, num_all = oracle.topk_prefix(oracle.score(oracle.pool(g, qt_all), oracle.pool(g, kt_all)), g.n_pre,
                                        wl.topk, inp["row_keep"], wl.max_k)
        flops = selected_flops(wl, num_all)
    else:
        flops = uniform_flops(wl)

    def step(i):
        h = i % Hh
        head = {n: np.ascontiguousarray(inp[n][:, :, h:h + 1, :]) for n in ("q", "k", "v")}
        t0 = time.perf_counter()
        qt, kt, vt = (oracle.tile(g, head[n]) for n in ("q", "k", "v"))
        if wl.map_driven:
            idx, num = oracle.map_to_index(np.ascontiguousarray(inp["map"][:, h:h + 1]))
        elif wl.prefix_dense:
            qbar, kbar = oracle.pool(g, qt), oracle.pool(g, kt)
            keep = None if inp["row_keep"] is None else np.ascontiguousarray(inp["row_keep"][:, h:h + 1])
            idx, num = oracle.topk_prefix(oracle.score(qbar, kbar), g.n_pre, wl.topk, keep, wl.max_k)
        else:
            qbar, kbar = oracle.pool(g, qt), oracle.pool(g, kt)
            idx, num = oracle.topk(oracle.score(qbar, kbar), wl.topk)
        if args.nvfp4:
            (qc, qs), (kc, ks) = oracle.quant_nvfp4(qt), oracle.quant_nvfp4(kt)
        t1 = time.perf_counter()
        rows = np.sort(rng.choice(head_rows, size=sample_rows, replace=False))
        if args.nvfp4:
            oracle.attn_rows_nvfp4(g, qc, qs, kc, ks, vt, idx, num, rows)
        else:
            oracle.attn_rows(g, qt, kt, vt, idx, num, rows)
        t2 = time.perf_counter()
        ot = np.zeros((B, 1, g.Sp, wl.D), dtype=np.uint16)
        oracle.untile(g, ot)
        t3 = time.perf_counter()
        return ((t1 - t0) + (t3 - t2)) * Hh + (t2 - t1) * Hh * head_rows / sample_rows

    for i in range(args.warmup):
        step(i)
    times = [step(args.warmup + i) for i in range(args.steps)]
    est = float(np.mean(times))
    value = flops / est / 1e12
    cores = oracle.max_threads()
    sample = (f"per step: one head (in turn) of the workload -- oracle tile/pool/score/top-k"
              f"{'/NVFP4 quantisation of q, k' if args.nvfp4 else ''}/untile of that head and attention on "
              f"{sample_rows} of its {head_rows} query rows drawn at random -- scaled to all {Hh} heads and rows")
    line = {
        "impl": "reference", "metric": "VSA sparse-attn fwd effective TFLOP/s (selected blocks) on 1 B200",
        "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": est * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic (seeded)",
        "config": {"workload": WORKLOAD_TEXT.get(args.workload, args.workload)},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def cpu_baseline_sample(wl, seconds_hint=20.0, nvfp4=False):
    """Oracle throughput on a bounded sample of the workload (about 10-30 s of CPU work)."""
    import oracle
    g = oracle.geometry_of(wl)
    inp = workloads.make_inputs(wl)
    t0 = time.perf_counter()
    qt, kt, vt = (oracle.tile(g, inp[n]) for n in ("q", "k", "v"))
    qbar, kbar = oracle.pool(g, qt), oracle.pool(g, kt)
    if wl.map_driven:
        idx, num = oracle.map_to_index(inp["map"])
    elif wl.prefix_dense:
        idx, num = oracle.topk_prefix(oracle.score(qbar, kbar), g.n_pre, wl.topk, inp["row_keep"], wl.max_k)
    else:
        idx, num = oracle.topk(oracle.score(qbar, kbar), wl.topk)
    if nvfp4:
        (qc, qs), (kc, ks) = oracle.quant_nvfp4(qt), oracle.quant_nvfp4(kt)
    oracle.untile(g, qt)
    t_front = time.perf_counter() - t0
    total_rows = wl.B * wl.H * g.Sp
    rng = np.random.default_rng(2)
    n = 256
    t_attn, done = 0.0, 0
    while t_attn < seconds_hint * 0.5 and done < total_rows:
        rows = np.sort(rng.choice(total_rows, size=min(n, total_rows - done), replace=False))
        t1 = time.perf_counter()
        if nvfp4:
            oracle.attn_rows_nvfp4(g, qc, qs, kc, ks, vt, idx, num, rows)
        else:
            oracle.attn_rows(g, qt, kt, vt, idx, num, rows)
        t_attn += time.perf_counter() - t1
        done += len(rows)
        n *= 2
    est = t_front + t_attn * total_rows / done
    value = selected_flops(wl, num) / est / 1e12
    return {"value": value, "unit": "TFLOP/s", "cores": oracle.max_threads(), "kind": "oracle",
            "sample": (f"oracle tile+pool+score+top-k{'+NVFP4 quantisation' if nvfp4 else ''}+untile over the "
                       f"whole workload ({t_front:.1f} s) and "
                       f"attention on {done} sampled of {total_rows} query rows ({t_attn:.1f} s), scaled to all "
                       f"rows; "
                       f"estimated {est:.3g} s per step")}


BWD_SOURCES = [os.path.join(ROOT, "block_sparse_video_gather_b200", "csrc", f)
               for f in ("attn_bwd.cu", "common.cuh", "tiles.cuh")]
BWD_PROFILE = os.path.join(ROOT, "profiles", "attn_bwd_fastwan.md")


def bwd_traffic(workload: str):
    """DRAM bytes per backward call from the committed ncu summary (None if absent or stale)."""
    if not os.path.exists(BWD_PROFILE):
        return None
    h = hashlib.sha256()
    for f in BWD_SOURCES:
        h.update(open(f, "rb").read())
    text = open(BWD_PROFILE).read()
    m_src = re.search(r"source_hash:\s*([0-9a-f]+)", text)
    m_wl = re.search(r"bench_workload:\s*(\w+)", text)
    m_b = re.search(r"traffic_bytes_per_call:\s*([0-9.eE+]+)", text)
    if not (m_src and m_wl and m_b) or m_src.group(1) != h.hexdigest()[:16] or m_wl.group(1) != workload:
        return None
    return float(m_b.group(1))


def bwd_cpu_baseline(wl, inp, do_untiled, idx, num, flops, seconds_hint=20.0):
    """Oracle backward on a bounded sample: dq of sampled query rows, scaled to all rows.
    The oracle's key side costs the same per query row (softmax, dP, then one
    accumulation), so the full backward is estimated at twice the dq cost."""
    import oracle
    g = oracle.geometry_of(wl)
    qt, kt, vt = (oracle.tile(g, inp[n]) for n in ("q", "k", "v"))
    dot = oracle.tile(g, do_untiled)
    total_rows = wl.B * wl.H * g.Sp
    rng = np.random.default_rng(3)
    n, t, done = 128, 0.0, 0
    while t < seconds_hint * 0.5 and done < total_rows:
        rows = np.sort(rng.choice(total_rows, size=min(n, total_rows - done), replace=False))
        t1 = time.perf_counter()
        oracle.attn_bwd_q_rows(g, qt, kt, vt, dot, idx, num, rows)
        t += time.perf_counter() - t1
        done += len(rows)
        n *= 2
    est = 2.0 * t * total_rows / done
    return {"value": flops / est / 1e12, "unit": "TFLOP/s", "cores": oracle.max_threads(), "kind": "oracle",
            "sample": (f"oracle dq on {done} of {total_rows} query rows ({t:.1f} s), scaled to all rows and "
                       f"doubled for dk/dv; estimated {est:.3g} s per backward")}


def run_backward(args, wl, world, rank, local, pg):
    """One step = one vsa_sparse_attn_bwd call (prep, transposed index, dk/dv, dq) on
    inputs resident in HBM; the selection, o and lse come from a forward call."""
    import torch
    import block_sparse_video_gather_b200 as vsa
    inp = workloads.make_inputs(wl, dtype=args.dtype)
    tdt = torch.float16 if args.dtype == "f16" else torch.bfloat16
    plan = vsa.Plan.of(wl)
    rng = np.random.default_rng(5)
    to16 = workloads.f32_to_f16_bits if args.dtype == "f16" else workloads.f32_to_bf16_bits
    do_untiled = to16(rng.standard_normal(inp["q"].shape).astype(np.float32))  # gradient of the untiled o
    dev16 = lambda b: torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).cuda().view(tdt)
    fwd = vsa.Forward(plan, wl.B, wl.H, wl.topk, dtype=tdt, prefix_dense=wl.prefix_dense)
    bmap = torch.from_numpy(inp["map"]).cuda() if wl.map_driven else None
    keep = torch.from_numpy(inp["row_keep"]).cuda() if inp["row_keep"] is not None else None
    fwd(dev16(inp["q"]), dev16(inp["k"]), dev16(inp["v"]), bmap, row_keep=keep)
    do = vsa.tile(plan, dev16(do_untiled))  # tiled; padded rows zero
    ws = torch.empty(vsa.bwd_workspace_bytes(plan, wl.B, wl.H, fwd.idx.shape[-1]), dtype=torch.uint8, device="cuda")
    dq, dk, dv = (torch.empty_like(fwd.qt) for _ in range(3))
    stream = torch.cuda.current_stream()

    def step():
        vsa.sparse_attn_bwd(plan, fwd.qt, fwd.kt, fwd.vt, fwd.ot, fwd.lse, do, fwd.idx, fwd.num, dq, dk, dv, ws)

    def sync_all():
        sync_ranks(pg)

    def max_over_ranks(x: float) -> float:
        return rank_max(x, pg)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert vsa.get_status() == vsa.VSA_OK
    fwd_flops = selected_flops(wl, fwd.num.cpu().numpy())
    flops = 2.5 * fwd_flops  # the usual count: five products of the forward's size, two of them repeated
    mma_flops = 3.5 * fwd_flops  # what the two kernels execute: 4 (dk/dv) + 3 (dq) products of half that size

    props = torch.cuda.get_device_properties(local)
    gpu_id = str(getattr(props, "uuid", local))
    if gpu_id and not gpu_id.startswith("GPU-") and len(gpu_id) >= 32:
        gpu_id = "GPU-" + gpu_id
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for attempt in range(2):  # measured again, once, when the clocks show a slowdown
        sampler = ClockSampler(gpu_id)
        sampler.start()
        time.sleep(0.3)
        sync_all()
        t0.record(stream)
        for i in range(args.steps):
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        t1.record(stream)
        sync_all()
        clocks = sampler.stop()
        if attempt == 1 or rank_max(float(clocks_rejected(clocks)), pg) == 0.0:
            break
    if clocks is not None and attempt == 1:
        clocks["remeasured"] = True
    elapsed = max_over_ranks(t0.elapsed_time(t1) / 1e3)
    call_avg = max_over_ranks(float(np.mean([a.elapsed_time(b) / 1e3 for a, b in ev])))
    assert vsa.get_status() == vsa.VSA_OK

    # end to end: tiled q, k, v, o, do, lse and the selection copied in, dq, dk, dv copied out
    host_in = {n: t.cpu().pin_memory() for n, t in (("q", fwd.qt), ("k", fwd.kt), ("v", fwd.vt), ("o", fwd.ot),
                                                     ("do", do), ("lse", fwd.lse), ("idx", fwd.idx),
                                                     ("num", fwd.num))}
    dev_in = {n: torch.empty_like(t, device="cuda") for n, t in host_in.items()}
    host_out = [torch.empty(dq.shape, dtype=tdt).pin_memory() for _ in range(3)]

    def e2e_step():
        for n in dev_in:
            dev_in[n].copy_(host_in[n], non_blocking=True)
        vsa.sparse_attn_bwd(plan, dev_in["q"], dev_in["k"], dev_in["v"], dev_in["o"], dev_in["lse"], dev_in["do"],
                            dev_in["idx"], dev_in["num"], dq, dk, dv, ws)
        for h, d in zip(host_out, (dq, dk, dv)):
            h.copy_(d, non_blocking=True)

    for _ in range(3):
        e2e_step()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sync_all()
    e0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    e1.record(stream)
    sync_all()
    e2e_elapsed = max_over_ranks(e0.elapsed_time(e1) / 1e3)
    assert vsa.get_status() == vsa.VSA_OK
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = sum(t.numel() * t.element_size() for t in host_out)

    if rank == 0:
        burst, _, _, peak_kind = measured_peaks()
        achieved = mma_flops / call_avg / 1e12
        line = {
            "metric": "VSA sparse-attn bwd effective TFLOP/s (selected blocks) on 1 B200",
            "value": world * flops * args.steps / elapsed / 1e12,
            "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": elapsed / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": args.dtype, "data": "synthetic (seeded; the recipe in block_sparse_video_gather_b200/workloads.py)",
            "config": {
                "workload": WORKLOAD_TEXT[args.workload], "pass": "backward of the fine stage (selection fixed)",
                "B": wl.B, "H": wl.H, "D": wl.D, "grid": [wl.T, wl.Hg, wl.Wg], "block": list(wl.block),
                "num_blocks": wl.num_blocks, "topk": wl.topk,
                "flop_count": "2.5 x the forward's selected-block FLOPs",
                "tflop_per_step": flops / 1e12, "call_ms": call_avg * 1e3,
                "l2": "inputs larger than L2: tiled q, k, v, o, do %.0f MB per step" % (5 * fwd.qt.numel() * 2 / 1e6),
                "parallelism": f"replicas x{world}",
            },
            "roofline": {
                "bound": "tensor", "kernel": "attn_bwd (prep + k2q + dkdv + dq, one call)", "achieved": achieved,
                "peak": burst, "unit": "TFLOP/s", "frac": achieved / burst,
                "flops_counted": "products the kernels execute: 3.5 x the forward's selected-block FLOPs",
                "peak_source": f"{peak_kind} bf16 burst (MEASURED_PEAKS.json)" if peak_kind == "measured"
                else "fallback 1.59 PFLOP/s",
                "traffic": bwd_traffic(args.workload),
            },
            "clocks": clocks,
            "e2e": {"value": world * flops * args.steps / e2e_elapsed / 1e12, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_elapsed / args.steps * 1e3},
            "gpu_launches": args.steps * 4,
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = bwd_cpu_baseline(wl, inp, do_untiled, fwd.idx.cpu().numpy(),
                                                    fwd.num.cpu().numpy(), flops)
        print(json.dumps(line), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="fastwan", choices=list(WORKLOAD_TEXT))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ref-rows", type=int, default=512, help="query rows of one head per reference step")
    ap.add_argument("--dtype", default="bf16", choices=["bf16", "f16"], help="16-bit format of q, k, v, o")
    ap.add_argument("--backward", action="store_true",
                    help="time the fine stage's backward (dq, dk, dv) instead of the forward step")
    ap.add_argument("--unfused", action="store_true",
                    help="run the front end as separate tile / coarse launches instead of one")
    ap.add_argument("--gate", action="store_true",
                    help="add the gate-compress branch (pooled v, block-level attention, gated sum in untile)")
    ap.add_argument("--nvfp4", action="store_true",
                    help="NVFP4 q and k in the fine stage (quantisation + FP4 Q K^T), v and P 16-bit")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--heads", type=int, default=None,
                    help="run the workload with this many heads (a smaller case of the same grid for profiler "
                         "captures; the line then names the head count)")
    ap.add_argument("--frames", type=int, default=None,
                    help="run the workload with this many latent frames T (a smaller case for profiler captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be at least 3")
    wl = workloads.WORKLOADS[args.workload]
    if args.heads is not None or args.frames is not None:
        import dataclasses
        wl = dataclasses.replace(wl, H=args.heads or wl.H, T=args.frames or wl.T)
        WORKLOAD_TEXT[args.workload] = (WORKLOAD_TEXT[args.workload] +
                                        f" (profiling case: H={wl.H}, T={wl.T})")
    world, rank, local = dist_setup(args)

    if args.impl == "reference":
        run_reference(args, wl, world, rank)
        return

    import torch
    import block_sparse_video_gather_b200 as vsa
    from block_sparse_video_gather_b200 import build as vsa_build

    torch.cuda.set_device(local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
        pg = dist
    if rank == 0:
        vsa_build.build()
    if pg:
        pg.barrier()
    vsa.lib()

    if args.backward:
        run_backward(args, wl, world, rank, local, pg)
        return

    inp = workloads.make_inputs(wl, dtype=args.dtype, gate=args.gate)
    tdt = torch.float16 if args.dtype == "f16" else torch.bfloat16
    tensors = ("q", "k", "v", "gate") if args.gate else ("q", "k", "v")
    host = {n: torch.from_numpy(inp[n].view(np.int16)).view(tdt).pin_memory() for n in tensors}
    if wl.map_driven:
        host["map"] = torch.from_numpy(inp["map"].view(np.uint8)).pin_memory()
    if inp["row_keep"] is not None:
        host["row_keep"] = torch.from_numpy(inp["row_keep"]).pin_memory()
    dev = {n: host[n].to("cuda", non_blocking=False) for n in host}
    plan = vsa.Plan.of(wl)
    fwd = vsa.Forward(plan, wl.B, wl.H, wl.topk, dtype=tdt, gated=args.gate, fused=not args.unfused,
                      nvfp4=args.nvfp4, prefix_dense=wl.prefix_dense)
    o_host = torch.empty(fwd.o.shape, dtype=tdt).pin_memory()
    lse_host = torch.empty(fwd.lse.shape, dtype=torch.float32).pin_memory()

    stream = torch.cuda.current_stream()
    attn_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
    front_ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    quant_ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    back_ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]

    def step(i=None):
        if i is not None:
            front_ev[i].record(stream)
        fwd.front(dev["q"], dev["k"], dev["v"], dev.get("map"), dev.get("row_keep"))
        if i is not None:
            quant_ev[i].record(stream)
        fwd.quantize()
        if i is not None:
            attn_ev[i][0].record(stream)
        fwd.attend()
        if i is not None:
            attn_ev[i][1].record(stream)
        fwd.back(dev.get("gate"))
        if i is not None:
            back_ev[i].record(stream)

    def sync_all():
        sync_ranks(pg)

    def max_over_ranks(x: float) -> float:
        return rank_max(x, pg)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert vsa.get_status() == vsa.VSA_OK
    flops = selected_flops(wl, fwd.num.cpu().numpy())
    flops_real = real_token_flops(wl, fwd.idx.cpu().numpy(), fwd.num.cpu().numpy())
    grouped = wl.block_tokens == 64 and wl.num_blocks <= 1024
    # the grouped 64-token kernel computes whole 128x128 products of which the
    # selection uses part: its executed FLOPs, 4 D 128^2 per Q-tile product
    flops_exec = (4.0 * wl.D * 128 * 128 * grouped_products(fwd.idx.cpu().numpy(), fwd.num.cpu().numpy(),
                                                             wl.num_blocks) if grouped else None)
    fp4_cosine = None
    if args.nvfp4 and not args.gate:
        # the page's quality figure for FP4 attention: per-call cosine similarity of
        # o against the 16-bit path on the same inputs (outside the timed region)
        ref16 = vsa.Forward(plan, wl.B, wl.H, wl.topk, dtype=tdt, prefix_dense=wl.prefix_dense)
        o16 = ref16(dev["q"], dev["k"], dev["v"], dev.get("map"), row_keep=dev.get("row_keep"))[0].float()
        o4 = fwd.back(dev.get("gate"), out=torch.empty_like(fwd.o)).float()
        fp4_cosine = float(torch.nn.functional.cosine_similarity(o4.reshape(1, -1), o16.reshape(1, -1)).item())
        del ref16, o16, o4
        torch.cuda.synchronize()

    props = torch.cuda.get_device_properties(local)
    gpu_id = str(getattr(props, "uuid", local))
    if gpu_id and not gpu_id.startswith("GPU-") and len(gpu_id) >= 32:
        gpu_id = "GPU-" + gpu_id
    # ---- device-resident timing (measured again, once, when the clocks show a slowdown)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for attempt in range(2):
        sampler = ClockSampler(gpu_id)
        sampler.start()
        time.sleep(0.3)
        sync_all()
        t0.record(stream)
        for i in range(args.steps):
            step(i)
        t1.record(stream)
        sync_all()
        clocks = sampler.stop()
        if attempt == 1 or rank_max(float(clocks_rejected(clocks)), pg) == 0.0:
            break
    if clocks is not None and attempt == 1:
        clocks["remeasured"] = True
    elapsed = max_over_ranks(t0.elapsed_time(t1) / 1e3)
    attn_s = [a.elapsed_time(b) / 1e3 for a, b in attn_ev]
    front_s = [f.elapsed_time(q) / 1e3 for f, q in zip(front_ev, quant_ev)]
    quant_s = [q.elapsed_time(a[0]) / 1e3 for q, a in zip(quant_ev, attn_ev)]
    back_s = [a[1].elapsed_time(b) / 1e3 for a, b in zip(attn_ev, back_ev)]
    attn_avg = max_over_ranks(float(np.mean(attn_s)))
    # the stages before and after the fine stage as medians over the steps: the
    # first timed step's front end also holds the host's launch latency (its
    # start event is recorded on an idle device)
    front_t, quant_t, back_t = (float(np.median(x)) for x in (front_s, quant_s, back_s))
    assert vsa.get_status() == vsa.VSA_OK

    # ---- the same steps replayed from a CUDA graph of one step (launch gaps
    # removed; reported beside the eager figure, which the roofline uses)
    cg = fwd.graph(dev["q"], dev["k"], dev["v"], dev.get("map"), dev.get("gate"), row_keep=dev.get("row_keep"))
    for _ in range(3):
        cg.replay()
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sync_all()
    g0.record(stream)
    for _ in range(args.steps):
        cg.replay()
    g1.record(stream)
    sync_all()
    graph_elapsed = max_over_ranks(g0.elapsed_time(g1) / 1e3)
    assert vsa.get_status() == vsa.VSA_OK
    del cg

    # ---- end to end through the public API with pinned host buffers: every step
    # copies its q, k, v in and its o out; vsa.HostPipeline overlaps step i's
    # compute with step i+1's upload and step i-1's download (two copy streams)
    pipe = vsa.HostPipeline(fwd)
    extra = dict(block_map=host.get("map"), gate=host.get("gate"), row_keep=host.get("row_keep"), lse=lse_host)
    for _ in range(3):
        pipe.submit(host["q"], host["k"], host["v"], o_host, **extra)
    pipe.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sync_all()
    e0.record(pipe.h2d)
    for _ in range(args.steps):
        pipe.submit(host["q"], host["k"], host["v"], o_host, **extra)
    e1.record(pipe.d2h)
    pipe.synchronize()
    sync_all()
    assert vsa.get_status() == vsa.VSA_OK
    # the same steps with the copies serialised on one stream, for reference
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sync_all()
    s0.record(stream)
    for _ in range(args.steps):
        for n in dev:
            dev[n].copy_(host[n], non_blocking=True)
        fwd(dev["q"], dev["k"], dev["v"], dev.get("map"), gate=dev.get("gate"), row_keep=dev.get("row_keep"))
        o_host.copy_(fwd.o, non_blocking=True)
        lse_host.copy_(fwd.lse, non_blocking=True)
    s1.record(stream)
    sync_all()
    serial_elapsed = max_over_ranks(s0.elapsed_time(s1) / 1e3)
    e2e_elapsed = max_over_ranks(e0.elapsed_time(e1) / 1e3)
    assert vsa.get_status() == vsa.VSA_OK
    h2d = sum(host[n].numel() * host[n].element_size() for n in host)
    d2h = o_host.numel() * 2 + lse_host.numel() * 4  # o and lse: both outputs of the call

    if rank == 0:
        burst, sustained, hbm, peak_kind = measured_peaks()
        peak = burst
        peak_source = (f"{peak_kind} bf16 burst (MEASURED_PEAKS.json)" if peak_kind == "measured"
                       else "fallback 1.59 PFLOP/s")
        if args.nvfp4:
            # half the flops (S = Q K^T) at the FP4 rate, 4x the bf16 rate (nominal 9 / 2.25 PFLOP/s),
            # half (O += P V) at the bf16 rate: 2 / (1/(4P) + 1/P) = 1.6 P
            peak = 1.6 * burst
            peak_source += " x 1.6 (Q K^T at the nominal FP4:bf16 ratio 4, P V at bf16)"
        achieved = flops / attn_avg / 1e12
        achieved_real = flops_real / attn_avg / 1e12
        if args.nvfp4:
            traffic = (profile_traffic(args.workload, *FP4_TRAFFIC_PROFILES[args.workload])
                       if args.workload in FP4_TRAFFIC_PROFILES and args.heads is None and args.frames is None
                       else None)
        elif args.workload in TRAFFIC_PROFILES and args.heads is None and args.frames is None:
            traffic = profile_traffic(args.workload, *TRAFFIC_PROFILES[args.workload])
        else:
            traffic = None
        line = {
            "metric": "VSA sparse-attn fwd effective TFLOP/s (selected blocks) on 1 B200",
            "value": world * flops * args.steps / elapsed / 1e12,
            "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": elapsed / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": f"nvfp4 q,k + {args.dtype} v,p" if args.nvfp4 else args.dtype, "data": "synthetic (seeded; the recipe in block_sparse_video_gather_b200/workloads.py)",
            "config": {
                "workload": WORKLOAD_TEXT[args.workload],
                "B": wl.B, "H": wl.H, "D": wl.D, "grid": [wl.T, wl.Hg, wl.Wg], "block": list(wl.block),
                "num_blocks": wl.num_blocks, "topk": wl.topk, "selected_block_tflop_per_step": flops / 1e12,
                "real_token_tflop_per_step": flops_real / 1e12,
                "flop_count": ("4 * D * bs^2 per selected block pair, padded slots included (the value and the "
                               "roofline); real_token_tflop_per_step counts real query x real key tokens only"),
                "selected_pairs": int(fwd.num.sum().item()),
                "attn_ms": attn_avg * 1e3, "front_ms": front_t * 1e3,
                "quant_ms": quant_t * 1e3,
                "qk_format": "NVFP4 (E2M1, E4M3 scale per 16 channels)" if args.nvfp4 else args.dtype,
                "nvfp4_cosine_vs_16bit": fp4_cosine,
                "back_ms": back_t * 1e3,
                # memory-bound stages: algorithmic bytes (untiled q, k, v read + tiled written; tiled o
                # read + untiled o written, plus the gate when gated) over their event time
                "front_gbs": (3 * host["q"].numel() * 2 + 3 * fwd.qt.numel() * 2) / front_t / 1e9,
                "back_gbs": (fwd.ot.numel() * 2 + fwd.o.numel() * 2 * (2 if args.gate else 1))
                / back_t / 1e9,
                "hbm_peak_gbs": measured_peaks()[2],
                "l2": "inputs larger than L2: q/k/v %.0f MB and tiled q/k/v %.0f MB per step" % (
                    sum(host[n].numel() * 2 for n in ("q", "k", "v")) / 1e6, 3 * fwd.qt.numel() * 2 / 1e6),
                "parallelism": f"replicas x{world}",
                "gate_compress": bool(args.gate),
                "front_end": "separate launches" if args.unfused else "one launch (tile + coarse)",
            },
            "roofline": {
                "bound": "tensor",
                "kernel": ("attn_fwd_grouped64_kernel" + ("<nvfp4>" if args.nvfp4 else "")
                           if (wl.block_tokens == 64 and wl.num_blocks <= 1024)
                           else "attn_fwd_fp4_kernel" if args.nvfp4 else "attn_fwd_kernel"),
                "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                "achieved_real_tokens": achieved_real, "frac_real_tokens": achieved_real / peak,
                **({"executed_tflop_per_launch": flops_exec / 1e12,
                    "achieved_executed": flops_exec / attn_avg / 1e12,
                    "frac_executed": flops_exec / attn_avg / 1e12 / peak} if flops_exec else {}),
                "peak_source": peak_source,
                "traffic": traffic,
            },
            "clocks": clocks,
            "e2e": {"value": world * flops * args.steps / e2e_elapsed / 1e12, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_elapsed / args.steps * 1e3,
                    "api": "vsa.HostPipeline (copies of neighbouring steps overlap the compute)",
                    "serial_ms_per_step": serial_elapsed / args.steps * 1e3},
            "gpu_launches": args.steps * fwd.launches(wl.map_driven),
            "graph": {"value": world * flops * args.steps / graph_elapsed / 1e12, "unit": "TFLOP/s",
                      "ms_per_step": graph_elapsed / args.steps * 1e3,
                      "how": "the same step captured once in a CUDA graph (vsa.Forward.graph), replayed per step"},
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline_sample(wl, nvfp4=args.nvfp4)
        print(json.dumps(line), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()


if __name__ == "__main__":
    main()
