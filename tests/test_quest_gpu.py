"""GPU parity of the Quest page-level indexer ("The Sparse Frontier" review, sec. 7.1) through the C ABI.

Boxes (per page and KV head, the per-dimension min and max of the existing keys) are compared bit for
bit with a plain PyTorch reduction; kept pages are compared with the fp64 oracle (a page may differ
only inside the relevance tie window); the selection then feeds sd_sparse_decode, checked against the
oracle's attention on the same rows.
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
P = 16


def _kmax_quest(w):
    """Row length that holds every Quest selection of w (whole pages, or the whole context)."""
    need = 1
    for n, k in zip(w.lens.tolist(), w.k.tolist()):
        np_ = (n + P - 1) // P
        kp = min(np_, (k + P - 1) // P)
        need = max(need, n if kp >= np_ else kp * P)
    return need


def _quest(w_dev, k_max):
    shape = sdb.make_shape(w_dev.B, w_dev.Hq, w_dev.Hkv, w_dev.max_pages, k_max, w_dev.num_pages)
    boxes = sdb.quest_boxes_for(shape, DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    sdb.sd_quest_summarize(shape, w_dev.K, w_dev.page_table, w_dev.lens, boxes, status)
    ws = sdb.workspace_for(shape, sdb.SD_OP_QUEST, DEV)
    idx = torch.full((w_dev.B, w_dev.Hq, k_max), -7, dtype=torch.int32, device=DEV)
    sdb.sd_quest_index(shape, w_dev.q, boxes, w_dev.page_table, w_dev.lens, w_dev.k, idx, ws, status)
    torch.cuda.synchronize()
    return shape, boxes, idx, int(status.item())


def _boxes_reference(w):
    """Per (physical page, KV head): min and max over the page's positions < N_b (plain PyTorch)."""
    ref = {}
    for b in range(w.B):
        n = int(w.lens[b])
        for j in range((n + P - 1) // P):
            page = int(w.page_table[b, j])
            rows = w.K[page, : min(P, n - j * P)].float()      # [rows][Hkv][d]
            ref[page] = (rows.min(dim=0).values, rows.max(dim=0).values)
    return ref


def _check_pages(w_cpu, idx_gpu, k_max):
    shape = w_cpu.shape()
    idx_orc = oracle.quest_topk(shape, w_cpu.q, w_cpu.K, w_cpu.page_table, w_cpu.lens, w_cpu.k, k_max=k_max)
    n_diff = 0
    for b in range(w_cpu.B):
        n = int(w_cpu.lens[b])
        np_ = (n + P - 1) // P
        for h in range(w_cpu.Hq):
            row = idx_gpu[b, h]
            sel = [int(x) for x in row if x >= 0]
            assert sel == sorted(sel) and len(set(sel)) == len(sel), (b, h)
            assert (row[len(sel):] == -1).all(), (b, h)
            pages = sorted({p // P for p in sel})
            assert sel == [p for j in pages for p in range(j * P, min(n, j * P + P))], (b, h)
            ref_pages = sorted({int(p) // P for p in idx_orc[b, h] if p >= 0})
            if n:
                assert np_ - 1 in pages
            assert len(pages) == len(ref_pages), (b, h)
            diff = set(pages) ^ set(ref_pages)
            if diff:
                r = oracle.quest_scores(shape, w_cpu.q, w_cpu.K, w_cpu.page_table, w_cpu.lens, b, h)
                kept = [j for j in ref_pages if j != np_ - 1]
                rk = min(r[j] for j in kept)
                tol = gh.TIE_REL * max(abs(rk), 1.0)
                for j in diff:
                    assert abs(r[j] - rk) <= tol, (b, h, j, r[j], rk)
                n_diff += len(diff)
    return idx_orc, n_diff


SHAPES = [
    # B, Hq, Hkv, lens, k
    (1, 4, 4, [777], [90]),                       # G = 1, partial last page
    (2, 8, 2, [1000, 5000], [100, 700]),          # G = 4
    (2, 64, 8, [4096, 3000], [82, 60]),           # G = 8
    (2, 32, 2, [3333, 1500], [67, 30]),           # G = 16
    (4, 8, 2, [0, 15, 16, 17], [3, 20, 1, 5]),    # empty, single page, exact page, budget covers all
    (1, 8, 1, [20000], [1]),                      # one page: the current one only
]


@pytest.mark.parametrize("B,Hq,Hkv,lens,k", SHAPES)
def test_quest_matches_oracle_and_decodes(B, Hq, Hkv, lens, k):
    w_cpu = wl.make_workload(B, Hq, Hkv, lens, k, seed=sum(lens) + 7 * Hq)
    k_max = _kmax_quest(w_cpu)
    w = w_cpu.to(DEV)
    shape, boxes, idx, status = _quest(w, k_max)
    assert status == 0
    # boxes: exact bf16 min / max of the existing rows
    ref = _boxes_reference(w_cpu)
    bx = boxes.float().cpu()
    for page, (mn, mx) in ref.items():
        assert torch.equal(bx[page, :, 0], mn) and torch.equal(bx[page, :, 1], mx), page
    idx_np = idx.cpu().numpy()
    _check_pages(w_cpu, idx_np, k_max)
    # the Quest rows through the sparse decode
    dshape = sdb.make_shape(w.B, w.Hq, w.Hkv, w.max_pages, k_max, w.num_pages)
    ws = sdb.workspace_for(dshape, sdb.SD_OP_SPARSE, DEV)
    out = torch.empty((B, Hq, 128), dtype=torch.float32, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    sdb.sd_sparse_decode(dshape, w.q, w.K, w.V, w.page_table, w.lens, idx, out, ws, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref_out = oracle.attend(w_cpu.shape(), w_cpu.q, w_cpu.K, w_cpu.V, w_cpu.page_table, w_cpu.lens, idx_np)
    gh.check_outputs(out.cpu().numpy(), ref_out)


def test_quest_last_page_update_after_append():
    """Appending a row and refreshing only each request's last page gives the boxes a full pass gives."""
    w_cpu = wl.make_workload(3, 8, 2, [40, 47, 48], [16, 16, 16], seed=77, extra_pages=2)
    k_max = 64
    w = w_cpu.to(DEV)
    shape = sdb.make_shape(w.B, w.Hq, w.Hkv, w.max_pages, k_max, w.num_pages)
    boxes = sdb.quest_boxes_for(shape, DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    sdb.sd_quest_summarize(shape, w.K, w.page_table, w.lens, boxes, st)
    g = torch.Generator().manual_seed(3)
    for _ in range(3):
        kn = torch.randn(w.B, w.Hkv, 128, generator=g).to(torch.bfloat16).to(DEV)
        vn = torch.randn(w.B, w.Hkv, 128, generator=g).to(torch.bfloat16).to(DEV)
        sdb.sd_append_kv(shape, w.K, w.V, w.page_table, w.lens, kn, vn, None, 50, st)
        sdb.sd_quest_summarize(shape, w.K, w.page_table, w.lens, boxes, st, last_page_only=True)
    full = sdb.quest_boxes_for(shape, DEV)
    sdb.sd_quest_summarize(shape, w.K, w.page_table, w.lens, full, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for b in range(w.B):
        n = int(w.lens[b])
        for j in range((n + P - 1) // P):
            page = int(w.page_table[b, j])
            assert torch.equal(boxes[page], full[page]), (b, j)


def test_quest_append_keeps_boxes_current():
    """sd_quest_append_kv over 20 steps (rows that open new pages and rows that extend them): every box
    equals the one a full summary of the grown cache writes, bit for bit; K, V and lens as sd_append_kv."""
    w_cpu = wl.make_workload(3, 8, 2, [40, 47, 48], [16, 16, 16], seed=78, extra_pages=3)
    k_max = 96
    w = w_cpu.to(DEV)
    w2 = w_cpu.to(DEV)
    shape = sdb.make_shape(w.B, w.Hq, w.Hkv, w.max_pages, k_max, w.num_pages)
    boxes = sdb.quest_boxes_for(shape, DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    sdb.sd_quest_summarize(shape, w.K, w.page_table, w.lens, boxes, st)
    g = torch.Generator().manual_seed(4)
    ks = torch.zeros(w.B, dtype=torch.int32, device=DEV)
    ks2 = torch.zeros(w.B, dtype=torch.int32, device=DEV)
    for _ in range(20):
        kn = torch.randn(w.B, w.Hkv, 128, generator=g).to(torch.bfloat16).to(DEV)
        vn = torch.randn(w.B, w.Hkv, 128, generator=g).to(torch.bfloat16).to(DEV)
        sdb.sd_quest_append_kv(shape, w.K, w.V, w.page_table, w.lens, kn, vn, ks, 50, boxes, st)
        sdb.sd_append_kv(shape, w2.K, w2.V, w2.page_table, w2.lens, kn, vn, ks2, 50, st)
    full = sdb.quest_boxes_for(shape, DEV)
    sdb.sd_quest_summarize(shape, w.K, w.page_table, w.lens, full, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert torch.equal(w.K, w2.K) and torch.equal(w.V, w2.V) and torch.equal(w.lens, w2.lens) and torch.equal(ks, ks2)
    assert [int(x) for x in w.lens] == [60, 67, 68]
    for b in range(w.B):
        n = int(w.lens[b])
        for j in range((n + P - 1) // P):
            page = int(w.page_table[b, j])
            assert torch.equal(boxes[page], full[page]), (b, j)


def test_quest_append_rejects_missing_boxes():
    w = wl.make_workload(1, 8, 2, [40], [16], seed=79, extra_pages=1).to(DEV)
    shape = sdb.make_shape(w.B, w.Hq, w.Hkv, w.max_pages, 64, w.num_pages)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    kn = torch.zeros(w.B, w.Hkv, 128, dtype=torch.bfloat16, device=DEV)
    assert sdb.sd_quest_append_kv(shape, w.K, w.V, w.page_table, w.lens, kn, kn, None, 50, None, st,
                                  check=False) == sdb.SD_ERR_INVALID_ARG


def test_quest_long128k_sampled():
    """The benchmark's workload (4 x 64/8 heads, N = 131072, k = 2621): Quest pages on sampled groups."""
    w = wl.named("long128k", device=DEV)
    k_max = _kmax_quest(w)
    shape, boxes, idx, status = _quest(w, k_max)
    assert status == 0
    idx_np = idx.cpu().numpy()
    for b, kvh in ((0, 0), (3, 7)):
        sub = gh.group_subproblem(w, b, kvh)
        _check_pages(sub, idx_np[b:b + 1, kvh * w.G:(kvh + 1) * w.G], k_max)
