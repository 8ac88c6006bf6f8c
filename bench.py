#!/usr/bin/env python
"""Decode benchmark: tokens/s and effective HBM GB/s of exact top-k sparse decode attention.

One step = one pass of the whole hot path over one decode batch: the exact top-k indexer
(sd_topk_scores + sd_topk_select) followed by sparse decode over the selected rows
(sd_sparse_decode), for one attention layer.  Default workload: 128K context at 50x sparsity
(B=4, 64 query / 8 KV heads, d=128, N=131072, k=2621, bf16, paged KV with page 16, attention
sinks), synthetic seeded inputs resident in HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

Multi-GPU (torchrun, one rank per GPU): every rank runs its own batch (weak scaling; requests are
independent, so there is no data-path collective); times are the max over ranks.  Rank 0 prints
one JSON line.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from sparse_attention_decode_sd_b200 import binding as sdb  # noqa: E402
from sparse_attention_decode_sd_b200 import workloads as wl  # noqa: E402

METRIC = "decode tokens/s and effective HBM GB/s (% of roofline) at 128K ctx, 50x sparsity"
L2_FLUSH_BYTES = 512 << 20
# kernels of one step: threshold, score pass, select; rows, sparse decode
LAUNCHES_PER_STEP = 5
# kernels of one Quest step: last-page box refresh, page score, page select; rows, sparse decode
QUEST_LAUNCHES_PER_STEP = 5
FALLBACK_HBM_GBS = 6650.0


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def source_hash(*names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "sparse_attention_decode_sd_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


KERNEL_SOURCES = {
    "score_pass_kernel": ("topk_score.cu", "common.cuh", "kernels.h"),
    "select_kernel": ("topk_select.cu", "common.cuh", "kernels.h"),
    "sparse_decode_kernel": ("sparse_decode.cu", "common.cuh", "kernels.h"),
}


def traffic_from_profiles(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on this exact source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
        e = t[kernel]
        if e.get("workload") != workload or e.get("source_sha256") != source_hash(*KERNEL_SOURCES[kernel]):
            return None
        return float(e["dram_bytes_per_launch"])
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons for this process's GPU."""

    FIELDS = ("pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        props = torch.cuda.get_device_properties(device)
        try:   # nvidia-smi prints the PCI id as DDDDDDDD:BB:DD.F
            self.bus = f"{int(props.pci_bus_id):02x}:{int(props.pci_device_id):02x}.0"
        except (AttributeError, TypeError, ValueError):
            self.bus = None
        self.proc = None
        self.file = None

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "50"], stdout=self.file, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.2)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        rows = [r.strip().split(", ") for r in self.file.read().splitlines() if r.strip()]
        os.unlink(self.file.name)
        if self.bus:
            mine = [r for r in rows if r and r[0].lower().endswith(self.bus)]
            rows = mine or rows
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                smax.append(float(r[2]))
            except (ValueError, IndexError):
                continue
            for n, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def union_rows(w, idx: torch.Tensor) -> int:
    """|U| summed over (b, kv head): rows selected by at least one head of the group (accounting only)."""
    B, Hq, kmax = idx.shape
    G = w.G
    n_cap = w.max_pages * w.P
    marks = torch.zeros((B, w.Hkv, n_cap + 1), dtype=torch.bool, device=idx.device)
    g = idx.view(B, w.Hkv, G * kmax).long()
    g = torch.where(g < 0, torch.full_like(g, n_cap), g)
    marks.scatter_(2, g, True)
    return int(marks[:, :, :n_cap].sum())


def required_bytes(w, idx: torch.Tensor):
    lens = w.lens.long()
    ks = torch.minimum(w.k.long(), lens)
    needs = (w.k.long() < lens) & (lens > 0)
    q_bytes = w.B * w.Hq * w.d * 2
    out_bytes = w.B * w.Hq * w.d * 4
    idx_bytes = int(ks.sum()) * w.Hq * 4
    U = union_rows(w, idx)
    k_bytes = int((lens * needs).sum()) * w.Hkv * w.d * 2
    return {
        "union_rows": U,
        "topk_scores": k_bytes + q_bytes,                       # K of every request that needs selection, q
        "sparse_decode": U * 2 * w.d * 2 + q_bytes + idx_bytes + out_bytes,
        "dense_decode": int(lens.sum()) * w.Hkv * w.d * 2 * 2 + q_bytes + out_bytes,
        "step": k_bytes + U * 2 * w.d * 2 + q_bytes + idx_bytes + out_bytes,
    }


def request_sample(w, b: int):
    """Request b of a GPU workload as a one-request CPU workload (data movement only)."""
    n = int(w.lens[b])
    npages = max(1, (n + w.P - 1) // w.P)
    pages = w.page_table[b, :npages].long()
    return wl.Workload(name=f"{w.name}[{b}]", B=1, Hq=w.Hq, Hkv=w.Hkv, d=w.d, P=w.P, max_pages=npages,
                       num_pages=npages, k_max=w.k_max, q=w.q[b:b + 1].contiguous().cpu(),
                       K=w.K[pages].contiguous().cpu(), V=w.V[pages].contiguous().cpu(),
                       page_table=torch.arange(npages, dtype=torch.int32).view(1, npages),
                       lens=torch.tensor([n], dtype=torch.int32), k=w.k[b:b + 1].cpu())


def oracle_step(sample):
    """The CPU oracle's index + decode on one request (test infrastructure, timed as a baseline)."""
    import oracle
    shape = sample.shape()
    idx = oracle.topk(shape, sample.q, sample.K, sample.page_table, sample.lens, sample.k)
    oracle.attend(shape, sample.q, sample.K, sample.V, sample.page_table, sample.lens, idx)


def cpu_baseline(w, min_seconds=10.0, max_reps=8):
    import oracle
    oracle.build()
    sample = request_sample(w, 0)
    reps, t0 = 0, time.perf_counter()
    while reps < max_reps:
        oracle_step(sample)
        reps += 1
        if time.perf_counter() - t0 >= min_seconds:
            break
    dt = time.perf_counter() - t0
    return {"value": reps / dt, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{reps} x request 0 of {w.name} (1 of {w.B} requests: {w.Hq} heads x {int(w.lens[0])} "
                      f"positions, exact top-{int(w.k[0])} + attention, fp64), {dt:.1f} s"}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(world, x: float) -> float:
    """Max of a per-rank scalar (a time) over all ranks; the only collective, measurement only."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(workload: str, rank: int) -> int:
    """Each rank decodes its own batch: same shapes, different seeded data."""
    return 1234 + wl.CONFIG_IDS[workload] + 1000 * rank


def job_tokens_per_s(world: int, batch: int, ms_per_step_max: float) -> float:
    """Whole-job throughput: every rank's batch, over the slowest rank's step time."""
    return world * batch / (ms_per_step_max / 1e3)


def config_of(w, args, world):
    return {"workload": f"{w.name}: B={w.B}, Hq={w.Hq}, Hkv={w.Hkv}, d={w.d}, N={int(w.lens.max())}, "
                        f"k={int(w.k.max())}, page={w.P}", "model": "one attention layer, synthetic bf16",
            "global_batch": w.B * world, "seq_len": int(w.lens.max()), "k": int(w.k.max()),
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": "flushed between steps by reading a 512 MiB buffer (untimed); the K/V cache exceeds L2 as well"}


def group_sample(w, b: int, kvh: int):
    """Group (b, kvh) of a workload as a one-request CPU workload with G heads (data movement only)."""
    n = int(w.lens[b])
    npages = max(1, (n + w.P - 1) // w.P)
    pages = w.page_table[b, :npages].long()
    G = w.G
    return wl.Workload(name=f"{w.name}[{b},{kvh}]", B=1, Hq=G, Hkv=1, d=w.d, P=w.P, max_pages=npages,
                       num_pages=npages, k_max=w.k_max, q=w.q[b:b + 1, kvh * G:(kvh + 1) * G].contiguous().cpu(),
                       K=w.K[pages, :, kvh:kvh + 1].contiguous().cpu(), V=w.V[pages, :, kvh:kvh + 1].contiguous().cpu(),
                       page_table=torch.arange(npages, dtype=torch.int32).view(1, npages),
                       lens=torch.tensor([n], dtype=torch.int32), k=w.k[b:b + 1].cpu())


def run_reference(args):
    """The oracle as it stands, on the host cores: each step is one (request, KV head) group of the
    workload (G heads: exact top-k over all N positions + attention), i.e. 1/Hkv of one token."""
    world, rank, _ = dist_setup()
    if rank != 0:
        return
    w = wl.named(args.workload, device="cuda" if torch.cuda.is_available() else "cpu")
    sample = group_sample(w, 0, 0)
    import oracle
    oracle.build()
    for _ in range(args.warmup):
        oracle_step(sample)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle_step(sample)
        times.append(time.perf_counter() - t0)
    per_group = statistics.mean(times)
    value = (1.0 / w.Hkv) / per_group
    cores = oracle.num_threads()
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_group * 1e3 * w.B * w.Hkv,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded)", "config": config_of(w, args, 1),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": f"each step: group (request 0, KV head 0) of {w.name} = {w.G} heads x "
                                       f"{int(w.lens[0])} positions, exact top-{int(w.k[0])} + attention in fp64; "
                                       f"1/{w.Hkv} token per step; ms_per_step extrapolates to the full batch"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_ours(args):
    world, rank, local = dist_setup()
    dev = torch.device("cuda", local)
    kw = {"ratio": args.ratio} if args.workload == "sweep128k" else {}
    w = wl.named(args.workload, device=dev, seed=rank_seed(args.workload, rank), **kw)
    shape = sdb.shape_of(w)
    ws_topk = sdb.workspace_for(shape, sdb.SD_OP_TOPK, dev)
    ws_dec = sdb.workspace_for(shape, sdb.SD_OP_SPARSE, dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    idx = torch.full((w.B, w.Hq, w.k_max), -1, dtype=torch.int32, device=dev)
    out = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device=dev)
    flush = torch.zeros(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def flush_l2():
        # Reading a buffer larger than L2 evicts everything cached, leaving clean lines: unlike a write
        # flush, it leaves no dirty lines whose write-back would land inside the next timed step.
        flush.amax()

    stream = torch.cuda.current_stream(dev)

    def step():
        sdb.sd_topk_scores(shape, w.q, w.K, w.page_table, w.lens, w.k, ws_topk, status, stream)
        sdb.sd_topk_select(shape, w.lens, w.k, idx, ws_topk, status, stream)
        sdb.sd_sparse_decode(shape, w.q, w.K, w.V, w.page_table, w.lens, idx, out, ws_dec, status, stream)

    for _ in range(args.warmup):
        flush_l2()
        step()
    torch.cuda.synchronize()
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())}: {sdb.status_string(int(status.item()))}")
    req = required_bytes(w, idx)

    sampler = ClockSampler(local)
    sampler.start()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush_l2()
        e = ev[i]
        e[0].record(stream)
        sdb.sd_topk_scores(shape, w.q, w.K, w.page_table, w.lens, w.k, ws_topk, status, stream)
        e[1].record(stream)
        sdb.sd_topk_select(shape, w.lens, w.k, idx, ws_topk, status, stream)
        e[2].record(stream)
        sdb.sd_sparse_decode(shape, w.q, w.K, w.V, w.page_table, w.lens, idx, out, ws_dec, status, stream)
        e[3].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clocks = sampler.stop()
    t_scores = sum(e[0].elapsed_time(e[1]) for e in ev) / args.steps
    t_select = sum(e[1].elapsed_time(e[2]) for e in ev) / args.steps
    t_decode = sum(e[2].elapsed_time(e[3]) for e in ev) / args.steps
    t_step = sum(e[0].elapsed_time(e[3]) for e in ev) / args.steps
    t_step_max = max_over_ranks(world, t_step)

    # dense comparator at the same shape (not part of the step)
    dense_ms = None
    if not args.no_dense:
        dout = torch.empty_like(out)
        ws_dense = sdb.workspace_for(shape, sdb.SD_OP_DENSE, dev)
        dev_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(5)]
        for _ in range(2):
            flush_l2()
            sdb.sd_dense_decode(shape, w.q, w.K, w.V, w.page_table, w.lens, dout, ws_dense, status, stream)
        for a, b_ in dev_ev:
            flush_l2()
            a.record(stream)
            sdb.sd_dense_decode(shape, w.q, w.K, w.V, w.page_table, w.lens, dout, ws_dense, status, stream)
            b_.record(stream)
        torch.cuda.synchronize()
        dense_ms = statistics.mean(a.elapsed_time(b_) for a, b_ in dev_ev)

    # end to end through the public API: pinned host inputs in, host result out, every step
    q_h = w.q.cpu().pin_memory()
    lens_h = w.lens.cpu().pin_memory()
    k_h = w.k.cpu().pin_memory()
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    q_d, lens_d, k_d = torch.empty_like(w.q), torch.empty_like(w.lens), torch.empty_like(w.k)
    e2e_steps = max(3, min(args.steps, 50))
    e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(e2e_steps)]
    barrier(world)
    torch.cuda.synchronize()
    for a, b_ in e2e_ev:
        flush_l2()
        a.record(stream)
        q_d.copy_(q_h, non_blocking=True)
        lens_d.copy_(lens_h, non_blocking=True)
        k_d.copy_(k_h, non_blocking=True)
        sdb.sd_topk_index(shape, q_d, w.K, w.page_table, lens_d, k_d, idx, ws_topk, status, stream)
        sdb.sd_sparse_decode(shape, q_d, w.K, w.V, w.page_table, lens_d, idx, out, ws_dec, status, stream)
        out_h.copy_(out, non_blocking=True)
        b_.record(stream)
    torch.cuda.synchronize()
    t_e2e = max_over_ranks(world, statistics.mean(a.elapsed_time(b_) for a, b_ in e2e_ev))
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())}: {sdb.status_string(int(status.item()))}")

    if rank != 0:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    hbm, peak_kind = peaks()
    tokens = w.B * world
    value = job_tokens_per_s(world, w.B, t_step_max)

    def gbs(nbytes, ms):
        return nbytes / (ms / 1e3) / 1e9

    kernels = {
        "topk_scores": {"ms": t_scores, "bytes": req["topk_scores"], "gbs": gbs(req["topk_scores"], t_scores)},
        "topk_select": {"ms": t_select},
        "sparse_decode": {"ms": t_decode, "bytes": req["sparse_decode"], "gbs": gbs(req["sparse_decode"], t_decode)},
    }
    for kname in ("topk_scores", "sparse_decode"):
        kernels[kname]["frac"] = kernels[kname]["gbs"] / hbm
    if dense_ms is not None:
        kernels["dense_decode"] = {"ms": dense_ms, "bytes": req["dense_decode"],
                                   "gbs": gbs(req["dense_decode"], dense_ms),
                                   "frac": gbs(req["dense_decode"], dense_ms) / hbm}
    # dominant kernel of the step by time
    dom = "topk_scores" if t_scores >= t_decode else "sparse_decode"
    dom_kernel = {"topk_scores": "score_pass_kernel", "sparse_decode": "sparse_decode_kernel"}[dom]
    roofline = {"bound": "hbm", "kernel": dom_kernel, "achieved": kernels[dom]["gbs"], "peak": hbm, "unit": "GB/s",
                "frac": kernels[dom]["gbs"] / hbm, "peak_source": peak_kind,
                "traffic": traffic_from_profiles(dom_kernel, w.name),
                "algorithmic_bytes": kernels[dom]["bytes"]}
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t_step_max, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded bf16 N(0,1) q/K/V, structure per workload)",
        "config": config_of(w, args, world),
        "effective_hbm_gbs": gbs(req["step"], t_step_max), "effective_hbm_frac": gbs(req["step"], t_step_max) / hbm,
        "required_bytes_per_step": req["step"], "union_rows": req["union_rows"],
        "sparse_decode_frac": kernels["sparse_decode"]["frac"],
        "dense_vs_sparse_decode": (dense_ms / t_decode) if dense_ms else None,
        "dense_vs_step": (dense_ms / t_step_max) if dense_ms else None,
        "kernels": kernels, "roofline": roofline, "clocks": clocks,
        "e2e": {"value": tokens / (t_e2e / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": q_h.numel() * 2 + lens_h.numel() * 4 + k_h.numel() * 4,
                "d2h_bytes_per_step": out_h.numel() * 4},
        "gpu_launches": LAUNCHES_PER_STEP * args.steps,
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_study(args):
    """Indexer-inclusive end-to-end study: for each sparsity ratio of the sweep workload, the step time of
    exact index + decode and of Quest index + decode, against dense decode at the same shape.  Each
    point runs in its own process (this script, single GPU)."""
    import subprocess
    points = []
    for ratio in wl.SWEEP_RATIOS:
        for indexer in ("exact", "quest"):
            cmd = [sys.executable, os.path.abspath(__file__), "--workload", "sweep128k", "--ratio", str(ratio),
                   "--indexer", indexer, "--steps", str(args.steps), "--warmup", str(args.warmup),
                   "--no-cpu-baseline"] + (["--no-dense"] if indexer == "quest" else [])
            r = subprocess.run(cmd, capture_output=True, text=True, check=True)
            line = json.loads(r.stdout.strip().splitlines()[-1])
            point = {"ratio": ratio, "indexer": indexer, "ms_per_step": line["ms_per_step"],
                     "tokens_per_s": line["value"], "kernels": {k: v["ms"] for k, v in line["kernels"].items()}}
            if indexer == "exact":
                point["dense_decode_ms"] = line["kernels"].get("dense_decode", {}).get("ms")
            points.append(point)
            print(json.dumps(point), flush=True)
    dense = {p["ratio"]: p["dense_decode_ms"] for p in points if p["indexer"] == "exact"}
    summary = {"study": "index + decode vs dense decode, sweep128k (B=16, 32/8 heads, N=131072)",
               "speedup_vs_dense": {f"{p['indexer']}@N/{p['ratio']}": dense[p["ratio"]] / p["ms_per_step"]
                                    for p in points if dense.get(p["ratio"])}}
    print(json.dumps(summary), flush=True)


def quest_k_max(w) -> int:
    """Row length that holds every Quest selection of w (whole pages, or the whole context)."""
    need = 1
    for n, k in zip(w.lens.tolist(), w.k.tolist()):
        np_ = (n + w.P - 1) // w.P
        kp = min(np_, (k + w.P - 1) // w.P)
        need = max(need, n if kp >= np_ else kp * w.P)
    return need


def run_quest(args):
    """The step with the Quest page-level indexer in place of the exact one: refresh each request's
    last page box (what a decode loop does after appending), select pages, sparse decode."""
    world, rank, local = dist_setup()
    dev = torch.device("cuda", local)
    kw = {"ratio": args.ratio} if args.workload == "sweep128k" else {}
    w = wl.named(args.workload, device=dev, seed=rank_seed(args.workload, rank), **kw)
    k_max = quest_k_max(w)
    shape = sdb.make_shape(w.B, w.Hq, w.Hkv, w.max_pages, k_max, w.num_pages)
    boxes = sdb.quest_boxes_for(shape, dev)
    ws_q = sdb.workspace_for(shape, sdb.SD_OP_QUEST, dev)
    ws_dec = sdb.workspace_for(shape, sdb.SD_OP_SPARSE, dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    idx = torch.full((w.B, w.Hq, k_max), -1, dtype=torch.int32, device=dev)
    out = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device=dev)
    flush = torch.zeros(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    sdb.sd_quest_summarize(shape, w.K, w.page_table, w.lens, boxes, status, stream=stream)   # the prefill's part

    def index():
        sdb.sd_quest_summarize(shape, w.K, w.page_table, w.lens, boxes, status, last_page_only=True, stream=stream)
        sdb.sd_quest_index(shape, w.q, boxes, w.page_table, w.lens, w.k, idx, ws_q, status, stream)

    for _ in range(args.warmup):
        flush.amax()
        index()
        sdb.sd_sparse_decode(shape, w.q, w.K, w.V, w.page_table, w.lens, idx, out, ws_dec, status, stream)
    torch.cuda.synchronize()
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())}: {sdb.status_string(int(status.item()))}")
    sampler = ClockSampler(local)
    sampler.start()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.amax()
        e = ev[i]
        e[0].record(stream)
        index()
        e[1].record(stream)
        sdb.sd_sparse_decode(shape, w.q, w.K, w.V, w.page_table, w.lens, idx, out, ws_dec, status, stream)
        e[2].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clocks = sampler.stop()
    t_index = sum(e[0].elapsed_time(e[1]) for e in ev) / args.steps
    t_decode = sum(e[1].elapsed_time(e[2]) for e in ev) / args.steps
    t_step_max = max_over_ranks(world, sum(e[0].elapsed_time(e[2]) for e in ev) / args.steps)
    if rank != 0:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    hbm, peak_kind = peaks()
    lens = w.lens.long()
    pages = int(((lens + w.P - 1) // w.P).sum())
    q_bytes, out_bytes = w.B * w.Hq * w.d * 2, w.B * w.Hq * w.d * 4
    idx_bytes = int((idx >= 0).sum()) * 4
    U = union_rows(w, idx)
    # Eq. 10's page representation: min and max rows (2 x d bf16) per page and KV head, plus q
    index_bytes = pages * w.Hkv * 2 * w.d * 2 + q_bytes
    decode_bytes = U * 2 * w.d * 2 + q_bytes + idx_bytes + out_bytes

    def gbs(nbytes, ms):
        return nbytes / (ms / 1e3) / 1e9

    kernels = {"quest_index": {"ms": t_index, "bytes": index_bytes, "gbs": gbs(index_bytes, t_index),
                               "frac": gbs(index_bytes, t_index) / hbm},
               "sparse_decode": {"ms": t_decode, "bytes": decode_bytes, "gbs": gbs(decode_bytes, t_decode),
                                 "frac": gbs(decode_bytes, t_decode) / hbm}}
    cfg = config_of(w, args, world)
    cfg["indexer"] = "quest (page boxes, ceil(k/16) pages incl. the current one)"
    line = {
        "metric": METRIC, "value": job_tokens_per_s(world, w.B, t_step_max), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_step_max, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded bf16 N(0,1) q/K/V, structure per workload)", "config": cfg,
        "required_bytes_per_step": index_bytes + decode_bytes, "union_rows": U,
        "effective_hbm_gbs": gbs(index_bytes + decode_bytes, t_step_max),
        "effective_hbm_frac": gbs(index_bytes + decode_bytes, t_step_max) / hbm,
        "kernels": kernels,
        "roofline": {"bound": "hbm", "kernel": "sparse_decode_kernel", "achieved": kernels["sparse_decode"]["gbs"],
                     "peak": hbm, "unit": "GB/s", "frac": kernels["sparse_decode"]["frac"], "peak_source": peak_kind,
                     "traffic": None, "algorithmic_bytes": decode_bytes},
        "clocks": clocks, "gpu_launches": QUEST_LAUNCHES_PER_STEP * args.steps,
    }
    print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default="long128k", choices=sorted(wl.CONFIG_IDS))
    ap.add_argument("--ratio", type=int, default=50, help="sparsity ratio of the sweep128k workload")
    ap.add_argument("--indexer", choices=("exact", "quest"), default="exact",
                    help="exact top-k (the method) or the Quest page-level approximate indexer")
    ap.add_argument("--study", action="store_true",
                    help="index + decode against dense decode over the sparsity sweep (sweep128k: N/10, N/50, "
                         "N/100, N), exact and Quest indexers; one JSON line per point, then a summary line")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.study:
        run_study(args)
    elif args.impl == "reference":
        run_reference(args)
    elif args.indexer == "quest":
        run_quest(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
