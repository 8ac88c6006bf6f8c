"""GPU parity of stochastic index selection (the vAttention-style selection of "Technische
Zusammenfassung: Kontextsparsitaet bei der Inferenzzeit", sec. 2 "Stochastische Indexierung"; the
reading is stated at the top of oracle/oracle.c) through the C ABI: sd_stochastic_index against the
oracle's stochastic_topk (the same exact rows and the same drawn rows, bit for bit, on the same seed
and step), and sd_sparse_decode_sampled against the oracle's weighted attention on the GPU's rows.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from sparse_attention_decode_sd_b200 import binding as sdb
from sparse_attention_decode_sd_b200 import workloads as wl
from tests import gpu_helpers as gh

pytestmark = pytest.mark.gpu

DEV = "cuda"
FLAG = sdb.SD_SAMPLED_FLAG


class StochasticRunner:
    def __init__(self, w):
        self.w = w
        self.shape = sdb.shape_of(w)
        self.ws_topk = sdb.workspace_for(self.shape, sdb.SD_OP_TOPK, w.q.device)
        self.ws_dec = sdb.workspace_for(self.shape, sdb.SD_OP_SPARSE, w.q.device)
        self.status = torch.zeros(1, dtype=torch.int32, device=w.q.device)

    def index(self, k_det, k_samp, seed, step):
        w = self.w
        idx = torch.full((w.B, w.Hq, w.k_max), -7, dtype=torch.int32, device=w.q.device)
        kd = torch.as_tensor(k_det, dtype=torch.int32, device=w.q.device).expand(w.B).contiguous()
        ks = torch.as_tensor(k_samp, dtype=torch.int32, device=w.q.device).expand(w.B).contiguous()
        sdb.sd_stochastic_index(self.shape, w.q, w.K, w.page_table, w.lens, kd, ks, seed, step, idx, self.ws_topk,
                                self.status)
        return idx

    def decode(self, idx, sampled=True):
        w = self.w
        out = torch.full((w.B, w.Hq, w.d), float("nan"), dtype=torch.float32, device=w.q.device)
        f = sdb.sd_sparse_decode_sampled if sampled else sdb.sd_sparse_decode
        f(self.shape, w.q, w.K, w.V, w.page_table, w.lens, idx, out, self.ws_dec, self.status)
        return out

    def device_status(self):
        torch.cuda.synchronize()
        return int(self.status.item())


def _parity(w_cpu, k_det, k_samp, seed, step):
    w = w_cpu.to(DEV)
    r = StochasticRunner(w)
    idx = r.index(k_det, k_samp, seed, step)
    out = r.decode(idx)
    assert r.device_status() == 0
    shape = w_cpu.shape()
    kd = [k_det] * w_cpu.B if np.isscalar(k_det) else list(k_det)
    ks = [k_samp] * w_cpu.B if np.isscalar(k_samp) else list(k_samp)
    ref = oracle.stochastic_topk(shape, w_cpu.q, w_cpu.K, w_cpu.page_table, w_cpu.lens, kd, ks, seed, step)
    got = idx.cpu().numpy()
    assert np.array_equal(got, ref), int((got != ref).sum())
    ref_out = oracle.attend(shape, w_cpu.q, w_cpu.K, w_cpu.V, w_cpu.page_table, w_cpu.lens, got)
    gh.check_outputs(out.cpu().numpy(), ref_out)
    return got, out


@pytest.mark.parametrize("B,Hq,Hkv,lens,k_det,k_samp,seed,step", [
    (1, 8, 2, [4096], 41, 41, 1, 0),                         # the tiny shape, half of the budget drawn
    (2, 16, 4, [6000, 3100], 60, 90, 77, 5),                 # more drawn than exact rows
    (3, 8, 2, [1000, 40, 5000], 20, 30, 3, 9),               # the rest smaller than k_samp (N = 40)
    (2, 32, 2, [9000, 7000], 5, 200, 2 ** 63 + 11, 2 ** 31),  # G = 16, large seed and step
])
def test_small_shapes(B, Hq, Hkv, lens, k_det, k_samp, seed, step):
    w_cpu = wl.make_workload(B, Hq, Hkv, lens, k_det, seed=sum(lens) + Hq, page_order="shuffled",
                             k_max=k_det + k_samp)
    idx, _ = _parity(w_cpu, k_det, k_samp, seed, step)
    drawn = (idx >= 0) & ((idx & FLAG) != 0)
    for b in range(B):
        assert int(drawn[b].sum(axis=1).max()) == min(k_samp, lens[b] - min(k_det, lens[b]))


def test_no_draw_is_the_exact_path():
    """k_samp = 0: the rows are sd_topk_index's and the weighted decode equals sd_sparse_decode bit for bit."""
    w_cpu = wl.make_workload(2, 16, 4, [5000, 4000], 100, seed=31, k_max=100)
    w = w_cpu.to(DEV)
    r = StochasticRunner(w)
    idx = r.index(100, 0, seed=4, step=4)
    base = gh.Runner(w)
    idx_exact = base.topk()
    assert torch.equal(idx, idx_exact)
    assert torch.equal(r.decode(idx, sampled=True), r.decode(idx, sampled=False))
    assert r.device_status() == 0 and base.device_status() == 0


def test_steps_draw_different_rows():
    w_cpu = wl.make_workload(1, 8, 2, 8000, 50, seed=8, k_max=150)
    w = w_cpu.to(DEV)
    r = StochasticRunner(w)
    a, b = r.index(50, 100, seed=5, step=1), r.index(50, 100, seed=5, step=2)
    assert r.device_status() == 0
    a, b = a.cpu().numpy(), b.cpu().numpy()
    assert not np.array_equal(a, b)
    plain_a = np.where((a >= 0) & ((a & FLAG) == 0), a, -1)
    plain_b = np.where((b >= 0) & ((b & FLAG) == 0), b, -1)
    assert np.array_equal(np.sort(plain_a, axis=-1), np.sort(plain_b, axis=-1))   # the exact rows do not move


def test_row_capacity_is_checked():
    w_cpu = wl.make_workload(1, 4, 2, 3000, 10, seed=9, k_max=40)
    w = w_cpu.to(DEV)
    r = StochasticRunner(w)
    idx = r.index(10, 31, seed=1, step=1)   # 10 + 31 > k_max = 40
    assert r.device_status() == sdb.SD_ERR_INVALID_ARG
    assert (idx.cpu().numpy()[0, :, 10:] == -1).all()


def test_long_context_every_row():
    """The long-context shape (B = 4, 64/8 heads, N = 131072) with the 50x budget split evenly:
    k_det = 1311 exact rows and k_samp = 1310 drawn rows; every row against the oracle."""
    torch.cuda.empty_cache()
    n = 131072
    kd, ks = wl.k_for_ratio(n, 100), wl.k_for_ratio(n, 50) - wl.k_for_ratio(n, 100)
    w = wl.named("long128k", device=DEV)
    w.k_max = kd + ks
    r = StochasticRunner(w)
    idx = r.index(kd, ks, seed=2024, step=17)
    out = r.decode(idx)
    assert r.device_status() == 0
    idx_np = idx.cpu().numpy()
    out_np = out.cpu().numpy()
    for b in range(w.B):
        sub = gh.request_subproblem(w, b)
        shape = sub.shape()
        # the oracle's rows are numbered within the request: row b * Hq + h of the batch
        ref = _oracle_rows_of_request(sub, b, w.Hq, kd, ks, 2024, 17)
        assert np.array_equal(idx_np[b:b + 1], ref), int((idx_np[b:b + 1] != ref).sum())
        o = oracle.attend(shape, sub.q, sub.K, sub.V, sub.page_table, sub.lens, idx_np[b:b + 1])
        gh.check_outputs(out_np[b:b + 1], o)


def _oracle_rows_of_request(sub, b, Hq, kd, ks, seed, step):
    """The oracle's stochastic rows of request b of a batch, computed on the one-request workload
    `sub`: the batch's row number b * Hq + h enters the sampling key, so the request is placed at
    index b of a batch whose other requests are empty."""
    B = b + 1
    shape = dict(sub.shape(), B=B)
    q = torch.zeros((B, Hq, sub.d), dtype=torch.bfloat16)
    q[b] = sub.q[0]
    pt = torch.zeros((B, sub.max_pages), dtype=torch.int32)
    pt[b] = sub.page_table[0]
    lens = torch.zeros(B, dtype=torch.int32)
    lens[b] = sub.lens[0]
    idx = oracle.stochastic_topk(shape, q, sub.K, pt, lens, [kd] * B, [ks] * B, seed, step, k_max=kd + ks)
    return idx[b:b + 1]
