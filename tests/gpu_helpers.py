"""Helpers of the GPU parity tests: run the C-ABI entry points on a workload and compare them with
the CPU oracle under the stated rules.

Parity rules (exact top-k selection, "Technische Zusammenfassung: Kontextsparsitaet bei der
Inferenzzeit", sec. 2; SDPA over the selected rows, xllm survey sec. 1.1):
  * index sets: the GPU row holds exactly min(k_b, N_b) strictly ascending positions in [0, N_b)
    followed by -1; every position in the symmetric difference with the oracle's set has an
    oracle score within 1e-4 * max(|s_(k)|, 1) of the oracle's k-th score s_(k) (a score tie, which
    fp32 and fp64 accumulation may order differently);
  * outputs: max |gpu - oracle| <= 1e-2 and mean |gpu - oracle| <= 1e-3 against the fp64 oracle
    on the same rows.  Tighter bounds derived from the kernel's arithmetic (fp32 accumulation, P
    carried to ~16 significant bits) are checked as well: max-abs <= 2e-4, mean-abs <= 2e-5.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from sparse_attention_decode_sd_b200 import binding as sdb
from sparse_attention_decode_sd_b200 import workloads as wl

TIE_REL = 1e-4
MAX_ABS = 1e-2
MEAN_ABS = 1e-3
TIGHT_MAX_ABS = 2e-4
TIGHT_MEAN_ABS = 2e-5


class Runner:
    """Device buffers and calls for one workload (already on the GPU)."""

    def __init__(self, w: wl.Workload):
        self.w = w
        self.shape = sdb.shape_of(w)
        dev = w.q.device
        self.ws_topk = sdb.workspace_for(self.shape, sdb.SD_OP_TOPK, dev)
        self.ws_dec = sdb.workspace_for(self.shape, sdb.SD_OP_SPARSE, dev)
        self.ws_dense = sdb.workspace_for(self.shape, sdb.SD_OP_DENSE, dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)

    def topk(self, k=None) -> torch.Tensor:
        w = self.w
        idx = torch.full((w.B, w.Hq, w.k_max), -7, dtype=torch.int32, device=w.q.device)   # poisoned
        sdb.sd_topk_index(self.shape, w.q, w.K, w.page_table, w.lens, w.k if k is None else k, idx, self.ws_topk,
                          self.status)
        return idx

    def sparse(self, idx: torch.Tensor) -> torch.Tensor:
        w = self.w
        out = torch.full((w.B, w.Hq, w.d), float("nan"), dtype=torch.float32, device=w.q.device)
        sdb.sd_sparse_decode(self.shape, w.q, w.K, w.V, w.page_table, w.lens, idx, out, self.ws_dec, self.status)
        return out

    def dense(self) -> torch.Tensor:
        w = self.w
        out = torch.full((w.B, w.Hq, w.d), float("nan"), dtype=torch.float32, device=w.q.device)
        sdb.sd_dense_decode(self.shape, w.q, w.K, w.V, w.page_table, w.lens, out, self.ws_dense, self.status)
        return out

    def device_status(self) -> int:
        torch.cuda.synchronize()
        return int(self.status.item())


def check_index_rows(idx_gpu: np.ndarray, idx_orc: np.ndarray, lens, ks, score_fn, pairs):
    """Parity of index sets for the (b, h) pairs listed; score_fn(b, h) returns oracle fp64 scores."""
    n_diff = 0
    for (b, h) in pairs:
        n = int(lens[b])
        take = min(int(ks[b]), n)
        row = idx_gpu[b, h]
        sel = row[:take]
        assert (row[take:] == -1).all(), (b, h, "padding")
        if take:
            assert (np.diff(sel) > 0).all(), (b, h, "not strictly ascending")
            assert sel[0] >= 0 and sel[-1] < n, (b, h, "out of range")
        ref = idx_orc[b, h][:take]
        assert (idx_orc[b, h][take:] == -1).all()
        diff = set(sel.tolist()) ^ set(ref.tolist())
        if diff:
            s = score_fn(b, h)
            sk = float(s[ref].min())
            tol = TIE_REL * max(abs(sk), 1.0)
            for p in diff:
                assert abs(float(s[p]) - sk) <= tol, (b, h, p, float(s[p]), sk)
            n_diff += len(diff)
    return n_diff


def check_outputs(out_gpu: np.ndarray, out_orc: np.ndarray, tight: bool = True):
    d = np.abs(out_gpu.astype(np.float64) - out_orc)
    assert np.isfinite(out_gpu).all()
    mx, mean = float(d.max()), float(d.mean())
    assert mx <= MAX_ABS and mean <= MEAN_ABS, (mx, mean)
    if tight:
        assert mx <= TIGHT_MAX_ABS and mean <= TIGHT_MEAN_ABS, (mx, mean)
    return mx, mean


def full_parity(w_cpu: wl.Workload, r: Runner, check_dense: bool = True):
    """Every (b, h) of a small workload: top-k, sparse decode on the GPU's own indices, dense decode."""
    idx = r.topk()
    out = r.sparse(idx)
    dense = r.dense() if check_dense else None
    assert r.device_status() == 0
    idx_np = idx.cpu().numpy()
    shape = w_cpu.shape()
    idx_orc = oracle.topk(shape, w_cpu.q, w_cpu.K, w_cpu.page_table, w_cpu.lens, w_cpu.k)
    pairs = [(b, h) for b in range(w_cpu.B) for h in range(w_cpu.Hq)]
    check_index_rows(idx_np, idx_orc, w_cpu.lens, w_cpu.k,
                     lambda b, h: oracle.scores(shape, w_cpu.q, w_cpu.K, w_cpu.page_table, w_cpu.lens, b, h), pairs)
    orc_out = oracle.attend(shape, w_cpu.q, w_cpu.K, w_cpu.V, w_cpu.page_table, w_cpu.lens, idx_np)
    check_outputs(out.cpu().numpy(), orc_out)
    if check_dense:
        orc_dense = oracle.dense(shape, w_cpu.q, w_cpu.K, w_cpu.V, w_cpu.page_table, w_cpu.lens)
        check_outputs(dense.cpu().numpy(), orc_dense)
    return idx_np, out


def group_subproblem(w: wl.Workload, b: int, kvh: int):
    """The (b, kvh) group of a GPU workload as a one-request CPU workload with a contiguous cache
    (data movement only): q of the group's G heads, the group's K/V rows in logical order."""
    n = int(w.lens[b])
    P = w.P
    npages = max(1, (n + P - 1) // P)
    pages = w.page_table[b, :npages].long()
    Ks = w.K[pages, :, kvh:kvh + 1, :].contiguous().cpu()
    Vs = w.V[pages, :, kvh:kvh + 1, :].contiguous().cpu()
    G = w.G
    qs = w.q[b:b + 1, kvh * G:(kvh + 1) * G].contiguous().cpu()
    sub = wl.Workload(name=f"{w.name}[{b},{kvh}]", B=1, Hq=G, Hkv=1, d=w.d, P=P, max_pages=npages, num_pages=npages,
                      k_max=w.k_max, q=qs, K=Ks, V=Vs,
                      page_table=torch.arange(npages, dtype=torch.int32).view(1, npages),
                      lens=torch.tensor([n], dtype=torch.int32), k=w.k[b:b + 1].cpu())
    return sub


def request_subproblem(w: wl.Workload, b: int):
    """Request b of a GPU workload as a one-request CPU workload with a contiguous cache (data
    movement only): its q, all its KV heads' K/V rows in logical order, an identity page table."""
    n = int(w.lens[b])
    P = w.P
    npages = max(1, (n + P - 1) // P)
    pages = w.page_table[b, :npages].long()
    return wl.Workload(name=f"{w.name}[{b}]", B=1, Hq=w.Hq, Hkv=w.Hkv, d=w.d, P=P, max_pages=npages,
                       num_pages=npages, k_max=w.k_max, q=w.q[b:b + 1].contiguous().cpu(),
                       K=w.K[pages].contiguous().cpu(), V=w.V[pages].contiguous().cpu(),
                       page_table=torch.arange(npages, dtype=torch.int32).view(1, npages),
                       lens=torch.tensor([n], dtype=torch.int32), k=w.k[b:b + 1].cpu())


def all_requests_parity(w: wl.Workload, idx: torch.Tensor, out: torch.Tensor, dense: torch.Tensor | None = None,
                        requests=None):
    """Parity of every (request, query head) row of a full-size GPU workload, one request at a time:
    the oracle's index set and its attention over the GPU's own rows (and dense attention)."""
    idx_np = idx.cpu().numpy()
    out_np = out.cpu().numpy()
    dense_np = dense.cpu().numpy() if dense is not None else None
    stats, n_diff = [], 0
    for b in (range(w.B) if requests is None else requests):
        sub = request_subproblem(w, b)
        shape = sub.shape()
        rows = idx_np[b:b + 1]
        ref = oracle.topk(shape, sub.q, sub.K, sub.page_table, sub.lens, sub.k)
        n_diff += check_index_rows(rows, ref, sub.lens, sub.k,
                                   lambda bb, h: oracle.scores(shape, sub.q, sub.K, sub.page_table, sub.lens, bb, h),
                                   [(0, h) for h in range(w.Hq)])
        o = oracle.attend(shape, sub.q, sub.K, sub.V, sub.page_table, sub.lens, rows)
        stats.append(check_outputs(out_np[b:b + 1], o))
        if dense_np is not None:
            od = oracle.dense(shape, sub.q, sub.K, sub.V, sub.page_table, sub.lens)
            stats.append(check_outputs(dense_np[b:b + 1], od))
    return stats, n_diff
