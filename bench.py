#!/usr/bin/env python
"""Decode benchmark: tokens/s and effective HBM GB/s of exact top-k sparse decode attention.

One step = one pass of the whole hot path over one decode batch: the exact top-k indexer
(sd_topk_scores + sd_topk_select) followed by sparse decode over the selected rows
(sd_sparse_decode), for one attention layer.  Headline workload: 128K context at 50x sparsity
(B=4, 64 query / 8 KV heads, d=128, N=131072, k=2621, bf16, paged KV with page 16, attention
sinks), synthetic seeded inputs resident in HBM.  The same JSON line carries the other four
workloads (tiny, llama8b, the sparsity sweep against dense decode with both indexers, and the
ragged batch's 64-step append + index + decode loop) under "configs".

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
import re
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
NOMINAL_HBM_GBS = 8000.0   # HBM3e, nominal (context for the effective-bandwidth fractions)
# kernels of one step: threshold, score pass, select; rows, sparse decode
LAUNCHES_PER_STEP = 5
# kernels of one Quest step: page score, page select; rows, sparse decode
QUEST_LAUNCHES_PER_STEP = 4
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
    """Hash of the kernels' code: the sources with comments and blank lines removed, so that a capture
    stays keyed to its code when only comments change."""
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "sparse_attention_decode_sd_b200", "csrc", n), encoding="utf-8") as f:
            text = re.sub(r"/\*.*?\*/", "", f.read(), flags=re.S)
        lines = (re.sub(r"//.*", "", line).rstrip() for line in text.splitlines())
        h.update("\n".join(line for line in lines if line).encode())
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
    """The method's algorithmic bytes per step, leg by leg."""
    lens = w.lens.long()
    needs = (w.k.long() < lens) & (lens > 0)
    q_bytes = w.B * w.Hq * w.d * 2
    out_bytes = w.B * w.Hq * w.d * 4
    idx_bytes = int((idx >= 0).sum()) * 4
    U = union_rows(w, idx)
    k_bytes = int((lens * needs).sum()) * w.Hkv * w.d * 2
    return {
        "union_rows": U,
        "topk_scores": k_bytes + q_bytes,                       # K of every request that needs selection, q
        "sparse_decode": U * 2 * w.d * 2 + q_bytes + idx_bytes + out_bytes,
        "dense_decode": int(lens.sum()) * w.Hkv * w.d * 2 * 2 + q_bytes + out_bytes,
        "step": k_bytes + U * 2 * w.d * 2 + q_bytes + idx_bytes + out_bytes,
    }


def gbs(nbytes, ms):
    return nbytes / (ms / 1e3) / 1e9


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


def workload_desc(w) -> str:
    return (f"{w.name}: B={w.B}, Hq={w.Hq}, Hkv={w.Hkv}, d={w.d}, N={int(w.lens.max())}, k={int(w.k.max())}, "
            f"page={w.P}")


def config_of(w, args, world):
    return {"workload": workload_desc(w), "model": "one attention layer, synthetic bf16",
            "global_batch": w.B * world, "seq_len": int(w.lens.max()), "k": int(w.k.max()),
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": "flushed between steps by reading a 512 MiB buffer (untimed); the K/V cache exceeds L2 as well"}


class Flusher:
    """Reads a buffer larger than L2 between timed steps: everything cached is evicted and only
    clean lines are left (a write flush would leave dirty lines to be written back inside the next
    timed step)."""

    def __init__(self, dev):
        self.buf = torch.zeros(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def __call__(self):
        self.buf.amax()


class ExactStep:
    """Buffers and calls of one exact index + sparse decode step on a workload."""

    def __init__(self, w, dev, stream):
        self.w = w
        self.shape = sdb.shape_of(w)
        self.ws_topk = sdb.workspace_for(self.shape, sdb.SD_OP_TOPK, dev)
        self.ws_dec = sdb.workspace_for(self.shape, sdb.SD_OP_SPARSE, dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.idx = torch.full((w.B, w.Hq, w.k_max), -1, dtype=torch.int32, device=dev)
        self.out = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device=dev)
        self.stream = stream

    def scores(self):
        w = self.w
        sdb.sd_topk_scores(self.shape, w.q, w.K, w.page_table, w.lens, w.k, self.ws_topk, self.status, self.stream)

    def select(self):
        w = self.w
        sdb.sd_topk_select(self.shape, w.lens, w.k, self.idx, self.ws_topk, self.status, self.stream)

    def decode(self):
        w = self.w
        sdb.sd_sparse_decode(self.shape, w.q, w.K, w.V, w.page_table, w.lens, self.idx, self.out, self.ws_dec,
                             self.status, self.stream)

    def check(self):
        torch.cuda.synchronize()
        st = int(self.status.item())
        if st != 0:
            raise RuntimeError(f"device status {st}: {sdb.status_string(st)}")


def time_exact(step: ExactStep, flush, steps: int, warmup: int):
    """Mean per-leg times (ms) of `steps` exact steps, L2 flushed before each."""
    s = step.stream
    for _ in range(warmup):
        flush()
        step.scores()
        step.select()
        step.decode()
    step.check()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    torch.cuda.synchronize()
    for e in ev:
        flush()
        e[0].record(s)
        step.scores()
        e[1].record(s)
        step.select()
        e[2].record(s)
        step.decode()
        e[3].record(s)
    step.check()
    mean = lambda i, j: sum(e[i].elapsed_time(e[j]) for e in ev) / steps   # noqa: E731
    return {"scores": mean(0, 1), "select": mean(1, 2), "decode": mean(2, 3), "step": mean(0, 3)}


def time_dense(w, shape, flush, stream, reps: int = 5, warmup: int = 2):
    dev = w.q.device
    out = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device=dev)
    ws = sdb.workspace_for(shape, sdb.SD_OP_DENSE, dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    for _ in range(warmup):
        flush()
        sdb.sd_dense_decode(shape, w.q, w.K, w.V, w.page_table, w.lens, out, ws, st, stream)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for a, b_ in ev:
        flush()
        a.record(stream)
        sdb.sd_dense_decode(shape, w.q, w.K, w.V, w.page_table, w.lens, out, ws, st, stream)
        b_.record(stream)
    torch.cuda.synchronize()
    if int(st.item()) != 0:
        raise RuntimeError(f"dense decode status {int(st.item())}")
    return statistics.mean(a.elapsed_time(b_) for a, b_ in ev)


def quest_k_max(w) -> int:
    """Row length that holds every Quest selection of w (whole pages, or the whole context)."""
    need = 1
    for n, k in zip(w.lens.tolist(), w.k.tolist()):
        np_ = (n + w.P - 1) // w.P
        kp = min(np_, (k + w.P - 1) // w.P)
        need = max(need, n if kp >= np_ else kp * w.P)
    return need


def time_quest(w, flush, stream, steps: int, warmup: int):
    """Quest step: page index (the index leg), then sparse decode.  The page boxes are kept current by
    the append of each step (sd_quest_append_kv: the written page's box updated in the same pass), so
    the step itself reads them as they are; here K does not change between steps."""
    dev = w.q.device
    k_max = quest_k_max(w)
    shape = sdb.make_shape(w.B, w.Hq, w.Hkv, w.max_pages, k_max, w.num_pages)
    boxes = sdb.quest_boxes_for(shape, dev)
    ws_q = sdb.workspace_for(shape, sdb.SD_OP_QUEST, dev)
    ws_dec = sdb.workspace_for(shape, sdb.SD_OP_SPARSE, dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    idx = torch.full((w.B, w.Hq, k_max), -1, dtype=torch.int32, device=dev)
    out = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device=dev)
    sdb.sd_quest_summarize(shape, w.K, w.page_table, w.lens, boxes, status, stream=stream)   # the prefill's part

    def index():
        sdb.sd_quest_index(shape, w.q, boxes, w.page_table, w.lens, w.k, idx, ws_q, status, stream)

    def decode():
        sdb.sd_sparse_decode(shape, w.q, w.K, w.V, w.page_table, w.lens, idx, out, ws_dec, status, stream)

    for _ in range(warmup):
        flush()
        index()
        decode()
    torch.cuda.synchronize()
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())}: {sdb.status_string(int(status.item()))}")
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    for e in ev:
        flush()
        e[0].record(stream)
        index()
        e[1].record(stream)
        decode()
        e[2].record(stream)
    torch.cuda.synchronize()
    t_index = sum(e[0].elapsed_time(e[1]) for e in ev) / steps
    t_decode = sum(e[1].elapsed_time(e[2]) for e in ev) / steps
    lens = w.lens.long()
    pages = int(((lens + w.P - 1) // w.P).sum())
    q_bytes, out_bytes = w.B * w.Hq * w.d * 2, w.B * w.Hq * w.d * 4
    U = union_rows(w, idx)
    # Eq. 10's page representation: min and max rows (2 x d bf16) per page and KV head, plus q
    index_bytes = pages * w.Hkv * 2 * w.d * 2 + q_bytes
    decode_bytes = U * 2 * w.d * 2 + q_bytes + int((idx >= 0).sum()) * 4 + out_bytes
    return {"index_ms": t_index, "decode_ms": t_decode, "step_ms": t_index + t_decode, "union_rows": U,
            "index_bytes": index_bytes, "decode_bytes": decode_bytes, "idx": idx}


def exact_summary(w, t, req, hbm, dense_ms=None):
    d = {"tokens_per_s": w.B / (t["step"] / 1e3), "ms_per_step": t["step"],
         "legs_ms": {"topk_scores": t["scores"], "topk_select": t["select"], "sparse_decode": t["decode"]},
         "union_rows": req["union_rows"],
         "sparse_decode_gbs": gbs(req["sparse_decode"], t["decode"]),
         "sparse_decode_frac": gbs(req["sparse_decode"], t["decode"]) / hbm,
         "topk_scores_frac": gbs(req["topk_scores"], t["scores"]) / hbm}
    if dense_ms is not None:
        d["dense_decode_ms"] = dense_ms
        d["dense_decode_frac"] = gbs(req["dense_decode"], dense_ms) / hbm
        d["sparse_vs_dense_decode"] = dense_ms / t["decode"]
        d["step_vs_dense_decode"] = dense_ms / t["step"]
    return d


def extra_configs(dev, stream, flush, hbm, steps: int, warmup: int, seed_rank: int):
    """Throughput of the other four workloads at one GPU (short runs, same timing rules)."""
    res = {}
    for name in ("tiny", "llama8b"):
        w = wl.named(name, device=dev, seed=rank_seed(name, seed_rank))
        st = ExactStep(w, dev, stream)
        t = time_exact(st, flush, steps, warmup)
        req = required_bytes(w, st.idx)
        res[name] = {"workload": workload_desc(w),
                     **exact_summary(w, t, req, hbm, time_dense(w, st.shape, flush, stream))}
        del st, w
        torch.cuda.empty_cache()
    # sparsity sweep: one cache, k changed per ratio; exact and Quest indexers against dense decode
    base = wl.named("sweep128k", device=dev, seed=rank_seed("sweep128k", seed_rank), ratio=50)
    n = int(base.lens[0])
    dense_ms = time_dense(base, sdb.shape_of(base), flush, stream)
    sweep = {"workload": workload_desc(base).replace(f"k={int(base.k.max())}", "k=N/ratio"),
             "dense_decode_ms": dense_ms}
    for ratio in wl.SWEEP_RATIOS:
        k = wl.k_for_ratio(n, ratio)
        w = wl.Workload(name="sweep128k", B=base.B, Hq=base.Hq, Hkv=base.Hkv, d=base.d, P=base.P,
                        max_pages=base.max_pages, num_pages=base.num_pages, k_max=k, q=base.q, K=base.K, V=base.V,
                        page_table=base.page_table, lens=base.lens, k=torch.full_like(base.k, k))
        st = ExactStep(w, dev, stream)
        t = time_exact(st, flush, steps, warmup)
        req = required_bytes(w, st.idx)
        point = {"k": k, "exact": exact_summary(w, t, req, hbm, dense_ms)}
        del st
        torch.cuda.empty_cache()
        if ratio != 1:
            qt = time_quest(w, flush, stream, steps, warmup)
            point["quest"] = {"tokens_per_s": w.B / (qt["step_ms"] / 1e3), "ms_per_step": qt["step_ms"],
                              "index_ms": qt["index_ms"], "decode_ms": qt["decode_ms"],
                              "index_frac": gbs(qt["index_bytes"], qt["index_ms"]) / hbm,
                              "decode_frac": gbs(qt["decode_bytes"], qt["decode_ms"]) / hbm,
                              "step_vs_dense_decode": dense_ms / qt["step_ms"]}
            del qt
            torch.cuda.empty_cache()
        sweep[f"N/{ratio}" if ratio != 1 else "N"] = point
    res["sweep128k"] = sweep
    del base
    torch.cuda.empty_cache()
    res["ragged"] = ragged_loop(dev, stream, flush, hbm, warmup, seed_rank)
    return res


def ragged_loop(dev, stream, flush, hbm, warmup: int, seed_rank: int):
    """Ragged batch, 64 decode steps: each step appends one K/V row per request (sd_append_kv, which
    also sets k_b = round(N_b / 50)), indexes (sd_topk_index) and decodes (sd_sparse_decode).  Every
    step is timed on its own (L2 flushed before it); dense decode at the first and last lengths."""
    w = wl.named("ragged", device=dev, seed=rank_seed("ragged", seed_rank))
    steps, ratio = w.meta["steps"], w.meta["ratio"]
    shape = sdb.shape_of(w)
    ws_topk = sdb.workspace_for(shape, sdb.SD_OP_TOPK, dev)
    ws_dec = sdb.workspace_for(shape, sdb.SD_OP_SPARSE, dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    idx = torch.full((w.B, w.Hq, w.k_max), -1, dtype=torch.int32, device=dev)
    out = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device=dev)

    def index_decode():
        sdb.sd_topk_index(shape, w.q, w.K, w.page_table, w.lens, w.k, idx, ws_topk, status, stream)
        sdb.sd_sparse_decode(shape, w.q, w.K, w.V, w.page_table, w.lens, idx, out, ws_dec, status, stream)

    for _ in range(warmup):   # the initial state, nothing appended
        flush()
        index_decode()
    dense_first = time_dense(w, shape, flush, stream)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
    dec_bytes = []
    for t, e in enumerate(ev):
        w.q = w.meta["q_steps"][t].contiguous()
        flush()
        e[0].record(stream)
        sdb.sd_append_kv(shape, w.K, w.V, w.page_table, w.lens, w.meta["k_new"][t], w.meta["v_new"][t], w.k, ratio,
                         status, stream)
        index_decode()
        e[1].record(stream)
        if t in (0, steps // 2, steps - 1):   # required bytes of this step's decode (accounting, untimed)
            torch.cuda.synchronize()
            dec_bytes.append((t, required_bytes(w, idx)["sparse_decode"]))
    torch.cuda.synchronize()
    if int(status.item()) != 0:
        raise RuntimeError(f"ragged loop status {int(status.item())}")
    per_step = [e[0].elapsed_time(e[1]) for e in ev]
    dense_last = time_dense(w, shape, flush, stream)
    # the decode leg alone at the last step's lengths, for its effective bandwidth
    dts = []
    for _ in range(5):
        flush()
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        sdb.sd_sparse_decode(shape, w.q, w.K, w.V, w.page_table, w.lens, idx, out, ws_dec, status, stream)
        b_.record(stream)
        torch.cuda.synchronize()
        dts.append(a.elapsed_time(b_))
    t_dec = statistics.mean(dts)
    mean_ms = statistics.mean(per_step)
    return {"workload": workload_desc(w) + ", 64 steps of append + index + decode",
            "steps": steps, "mean_ms_per_step": mean_ms, "tokens_per_s": w.B / (mean_ms / 1e3),
            "first_step_ms": per_step[0], "last_step_ms": per_step[-1],
            "last_step_sparse_decode_ms": t_dec,
            "last_step_sparse_decode_frac": gbs(dec_bytes[-1][1], t_dec) / hbm,
            "dense_decode_ms_first": dense_first, "dense_decode_ms_last": dense_last,
            "launches_per_step": 1 + 3 + 2}


def run_reference(args):
    """The oracle as it stands, on the host cores: each timed step is one whole request of the
    workload (all its heads: exact top-k over all N positions + attention, fp64), i.e. one token;
    ms_per_step is that measured time."""
    world, rank, _ = dist_setup()
    if rank != 0:
        return
    w = wl.named(args.workload, device="cuda" if torch.cuda.is_available() else "cpu")
    import oracle
    oracle.build()
    samples = [request_sample(w, b) for b in range(min(w.B, 2))]
    for i in range(args.warmup):
        oracle_step(samples[i % len(samples)])
    times = []
    for i in range(args.steps):
        t0 = time.perf_counter()
        oracle_step(samples[i % len(samples)])
        times.append(time.perf_counter() - t0)
    per_step = statistics.mean(times)
    value = 1.0 / per_step
    cores = oracle.num_threads()
    sample = (f"each step: one request of {w.name} ({w.Hq} heads x {int(w.lens[0])} positions, exact "
              f"top-{int(w.k[0])} + attention in fp64) = 1 token; requests 0 and 1 alternate")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_step * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded)", "config": {**config_of(w, args, 1), "step": "one request (1 token)"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_ours(args):
    world, rank, local = dist_setup()
    dev = torch.device("cuda", local)
    kw = {"ratio": args.ratio} if args.workload == "sweep128k" else {}
    w = wl.named(args.workload, device=dev, seed=rank_seed(args.workload, rank), **kw)
    stream = torch.cuda.current_stream(dev)
    flush = Flusher(dev)
    step = ExactStep(w, dev, stream)
    shape = step.shape

    for _ in range(args.warmup):
        flush()
        step.scores()
        step.select()
        step.decode()
    step.check()
    req = required_bytes(w, step.idx)

    sampler = ClockSampler(local)
    sampler.start()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    for e in ev:
        flush()
        e[0].record(stream)
        step.scores()
        e[1].record(stream)
        step.select()
        e[2].record(stream)
        step.decode()
        e[3].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clocks = sampler.stop()
    step.check()
    t_scores = sum(e[0].elapsed_time(e[1]) for e in ev) / args.steps
    t_select = sum(e[1].elapsed_time(e[2]) for e in ev) / args.steps
    t_decode = sum(e[2].elapsed_time(e[3]) for e in ev) / args.steps
    t_step = sum(e[0].elapsed_time(e[3]) for e in ev) / args.steps
    t_step_max = max_over_ranks(world, t_step)

    # dense comparator at the same shape (not part of the step)
    dense_ms = None if args.no_dense else time_dense(w, shape, flush, stream)

    # end to end through the public API: pinned host inputs in, host result out, every step
    q_h = w.q.cpu().pin_memory()
    lens_h = w.lens.cpu().pin_memory()
    k_h = w.k.cpu().pin_memory()
    out_h = torch.empty(step.out.shape, dtype=step.out.dtype).pin_memory()
    q_d, lens_d, k_d = torch.empty_like(w.q), torch.empty_like(w.lens), torch.empty_like(w.k)
    e2e_steps = max(3, min(args.steps, 50))
    e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(e2e_steps)]
    barrier(world)
    torch.cuda.synchronize()
    for a, b_ in e2e_ev:
        flush()
        a.record(stream)
        q_d.copy_(q_h, non_blocking=True)
        lens_d.copy_(lens_h, non_blocking=True)
        k_d.copy_(k_h, non_blocking=True)
        sdb.sd_topk_index(shape, q_d, w.K, w.page_table, lens_d, k_d, step.idx, step.ws_topk, step.status, stream)
        sdb.sd_sparse_decode(shape, q_d, w.K, w.V, w.page_table, lens_d, step.idx, step.out, step.ws_dec,
                             step.status, stream)
        out_h.copy_(step.out, non_blocking=True)
        b_.record(stream)
    torch.cuda.synchronize()
    t_e2e = max_over_ranks(world, statistics.mean(a.elapsed_time(b_) for a, b_ in e2e_ev))
    step.check()

    hbm, peak_kind = peaks()
    extras = None
    if not args.no_extra and world == 1:
        del step
        torch.cuda.empty_cache()
        extras = extra_configs(dev, stream, flush, hbm, args.extra_steps, 3, rank)

    if rank != 0:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    tokens = w.B * world
    value = job_tokens_per_s(world, w.B, t_step_max)
    kernels = {
        "topk_scores": {"ms": t_scores, "bytes": req["topk_scores"], "gbs": gbs(req["topk_scores"], t_scores),
                        "kernels": "threshold_kernel + score_pass_kernel"},
        "topk_select": {"ms": t_select, "kernels": "select_kernel"},
        "sparse_decode": {"ms": t_decode, "bytes": req["sparse_decode"], "gbs": gbs(req["sparse_decode"], t_decode),
                          "kernels": "rows_kernel + sparse_decode_kernel"},
    }
    for kname in ("topk_scores", "sparse_decode"):
        kernels[kname]["frac"] = kernels[kname]["gbs"] / hbm
        kernels[kname]["frac_of_nominal_8tbs"] = kernels[kname]["gbs"] / NOMINAL_HBM_GBS
    if dense_ms is not None:
        kernels["dense_decode"] = {"ms": dense_ms, "bytes": req["dense_decode"],
                                   "gbs": gbs(req["dense_decode"], dense_ms),
                                   "frac": gbs(req["dense_decode"], dense_ms) / hbm,
                                   "kernels": "ranges_kernel + dense_decode_kernel + merge_kernel"}

    def roofline_of(leg, kernel_name, traffic_key):
        return {"bound": "hbm", "kernel": kernel_name, "achieved": kernels[leg]["gbs"], "peak": hbm, "unit": "GB/s",
                "frac": kernels[leg]["gbs"] / hbm, "peak_source": peak_kind,
                "traffic": traffic_from_profiles(traffic_key, w.name), "algorithmic_bytes": kernels[leg]["bytes"]}

    # the dominant leg of the step by time (the indexer's K stream), and the decode leg on its own
    dom = "topk_scores" if t_scores >= t_decode else "sparse_decode"
    legs = {"topk_scores": ("threshold_kernel + score_pass_kernel", "score_pass_kernel"),
            "sparse_decode": ("rows_kernel + sparse_decode_kernel", "sparse_decode_kernel")}
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t_step_max, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded bf16 N(0,1) q/K/V, structure per workload)",
        "config": config_of(w, args, world),
        # the metric's effective HBM figure: sd_sparse_decode on its required bytes (the union of the
        # selected K/V rows plus q, indices and output), against the measured and the nominal peak
        "effective_hbm_gbs": kernels["sparse_decode"]["gbs"],
        "effective_hbm_frac": kernels["sparse_decode"]["frac"],
        "effective_hbm_frac_of_nominal_8tbs": kernels["sparse_decode"]["frac_of_nominal_8tbs"],
        "sparse_decode_frac": kernels["sparse_decode"]["frac"],
        # the whole step (the indexer's read of all of K included) over its algorithmic bytes
        "step_bytes_gbs": gbs(req["step"], t_step_max), "step_bytes_frac": gbs(req["step"], t_step_max) / hbm,
        "required_bytes_per_step": req["step"], "union_rows": req["union_rows"],
        "dense_vs_sparse_decode": (dense_ms / t_decode) if dense_ms else None,
        "dense_vs_step": (dense_ms / t_step_max) if dense_ms else None,
        "kernels": kernels,
        "roofline": roofline_of(dom, *legs[dom]),
        "decode_roofline": roofline_of("sparse_decode", *legs["sparse_decode"]),
        "clocks": clocks,
        "e2e": {"value": tokens / (t_e2e / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": q_h.numel() * 2 + lens_h.numel() * 4 + k_h.numel() * 4,
                "d2h_bytes_per_step": out_h.numel() * 4},
        "gpu_launches": LAUNCHES_PER_STEP * args.steps,
    }
    if extras is not None:
        line["configs"] = extras
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_quest(args):
    """The step with the Quest page-level indexer in place of the exact one: select pages from the
    page boxes (kept current by the append of a decode loop, sd_quest_append_kv), sparse decode."""
    world, rank, local = dist_setup()
    dev = torch.device("cuda", local)
    kw = {"ratio": args.ratio} if args.workload == "sweep128k" else {}
    w = wl.named(args.workload, device=dev, seed=rank_seed(args.workload, rank), **kw)
    stream = torch.cuda.current_stream(dev)
    flush = Flusher(dev)
    sampler = ClockSampler(local)
    sampler.start()
    barrier(world)
    q = time_quest(w, flush, stream, args.steps, args.warmup)
    barrier(world)
    clocks = sampler.stop()
    t_step_max = max_over_ranks(world, q["step_ms"])
    if rank != 0:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    hbm, peak_kind = peaks()
    kernels = {"quest_index": {"ms": q["index_ms"], "bytes": q["index_bytes"], "gbs": gbs(q["index_bytes"], q["index_ms"]),
                               "frac": gbs(q["index_bytes"], q["index_ms"]) / hbm},
               "sparse_decode": {"ms": q["decode_ms"], "bytes": q["decode_bytes"],
                                 "gbs": gbs(q["decode_bytes"], q["decode_ms"]),
                                 "frac": gbs(q["decode_bytes"], q["decode_ms"]) / hbm}}
    cfg = config_of(w, args, world)
    cfg["indexer"] = "quest (page boxes, ceil(k/16) pages incl. the current one)"
    line = {
        "metric": METRIC, "value": job_tokens_per_s(world, w.B, t_step_max), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_step_max, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded bf16 N(0,1) q/K/V, structure per workload)", "config": cfg,
        "required_bytes_per_step": q["index_bytes"] + q["decode_bytes"], "union_rows": q["union_rows"],
        "effective_hbm_gbs": kernels["sparse_decode"]["gbs"], "effective_hbm_frac": kernels["sparse_decode"]["frac"],
        "step_bytes_frac": gbs(q["index_bytes"] + q["decode_bytes"], t_step_max) / hbm,
        "kernels": kernels,
        "roofline": {"bound": "hbm", "kernel": "rows_kernel + sparse_decode_kernel",
                     "achieved": kernels["sparse_decode"]["gbs"], "peak": hbm, "unit": "GB/s",
                     "frac": kernels["sparse_decode"]["frac"], "peak_source": peak_kind, "traffic": None,
                     "algorithmic_bytes": q["decode_bytes"]},
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
    ap.add_argument("--extra-steps", type=int, default=30,
                    help="timed steps for each of the other workloads reported under 'configs'")
    ap.add_argument("--no-extra", action="store_true", help="skip the other workloads")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    elif args.indexer == "quest":
        run_quest(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
