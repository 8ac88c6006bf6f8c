"""Pins for the oracle's Quest page-level indexer (CPU only).

Quest ("The Sparse Frontier" review (xllm), sec. 7.1 and Table 1; Eq. 10): pages of P positions,
each represented per KV head by the per-dimension minimum and maximum of its keys; the most relevant
pages are kept, always including the page of the current position.  Relevance is read as the largest
q.k any key inside the page's [min, max] box can reach.  These tests check the oracle against things
other than its own formula: brute force over the box's corners, the exact per-row scores the box must
bound, hand-built pages with known rankings, and the budget and tie rules.
"""
from __future__ import annotations

import itertools

import numpy as np
import torch

import oracle
from sparse_attention_decode_sd_b200 import workloads as wl


def _int_workload(n, P=4, d=4, seed=0, Hq=1, Hkv=1, stale=1000.0):
    """One request with small-integer bf16 q and K (every product and sum is exact), stored through a
    reversed page table; slots past N in the last page hold a huge `stale` value that must be ignored."""
    g = torch.Generator().manual_seed(seed)
    pages = (n + P - 1) // P
    pt = torch.arange(pages - 1, -1, -1, dtype=torch.int32).view(1, pages)
    K = torch.full((pages, P, Hkv, d), stale, dtype=torch.float64)
    Kl = torch.randint(-8, 9, (n, Hkv, d), generator=g).double()
    for i in range(n):
        K[pt[0, i // P], i % P] = Kl[i]
    q = torch.randint(-4, 5, (1, Hq, d), generator=g).double()
    shape = dict(B=1, Hq=Hq, Hkv=Hkv, d=d, P=P, max_pages=pages)
    return shape, q.to(torch.bfloat16), K.to(torch.bfloat16), pt, torch.tensor([n], dtype=torch.int32), Kl


def test_relevance_is_max_over_box_corners():
    """r_j = max over the 2^d corners of the page's box of q.corner, the box taken over the page's
    existing rows only (the stale slots of the last page hold 1000 and must not count)."""
    for n, seed in ((13, 1), (16, 2), (9, 3)):
        P, d = 4, 4
        shape, q, K, pt, lens, Kl = _int_workload(n, P=P, d=d, seed=seed)
        r = oracle.quest_scores(shape, q, K, pt, lens, 0, 0)
        qd = q[0, 0].double().numpy()
        assert len(r) == (n + P - 1) // P
        for j in range(len(r)):
            rows = Kl[j * P: min(n, (j + 1) * P), 0].numpy()
            lo, hi = rows.min(axis=0), rows.max(axis=0)
            best = max(float(np.dot(qd, np.where(np.array(c), hi, lo))) for c in itertools.product((0, 1), repeat=d))
            assert r[j] == best, (n, j, r[j], best)


def test_relevance_bounds_every_row_of_its_page():
    """On random bf16 data (d = 128, GQA, shuffled pages) no row of a page scores above the page's
    relevance, and a page with a single existing row scores exactly that row's q.k."""
    w = wl.make_workload(1, 4, 2, 16 * 9 + 1, 5, seed=31)
    shape = w.shape()
    for h in range(4):
        s = oracle.scores(shape, w.q, w.K, w.page_table, w.lens, 0, h)
        r = oracle.quest_scores(shape, w.q, w.K, w.page_table, w.lens, 0, h)
        for j in range(len(r)):
            rows = s[j * 16: (j + 1) * 16]
            assert rows.max() <= r[j] + 1e-9 * max(1.0, abs(r[j]))
        assert r[-1] == s[-1]   # the last page holds one row


def _ranked_pages_workload(page_values, P=4, d=4):
    """One request whose page j holds P copies of the key v_j * e_0, with q = e_0: page j's relevance is
    exactly v_j (and so is every row's score)."""
    n = len(page_values) * P
    K = torch.zeros(len(page_values), P, 1, d, dtype=torch.float64)
    for j, v in enumerate(page_values):
        K[j, :, 0, 0] = v
    q = torch.zeros(1, 1, d, dtype=torch.float64)
    q[0, 0, 0] = 1.0
    pt = torch.arange(len(page_values), dtype=torch.int32).view(1, -1)
    shape = dict(B=1, Hq=1, Hkv=1, d=d, P=P, max_pages=len(page_values))
    return shape, q.to(torch.bfloat16), K.to(torch.bfloat16), pt, torch.tensor([n], dtype=torch.int32)


def _pages_of(idx_row, P):
    sel = [int(x) for x in idx_row if x >= 0]
    assert sel == sorted(sel) and len(set(sel)) == len(sel)
    return sorted({p // P for p in sel}), sel


def test_current_page_always_kept():
    """The last page has the lowest relevance but is kept; the budget of 2 pages adds the best other."""
    shape, q, K, pt, lens = _ranked_pages_workload([3, 7, 5, 1, -9])
    idx = oracle.quest_topk(shape, q, K, pt, lens, [8], k_max=8)
    pages, sel = _pages_of(idx[0, 0], 4)
    assert pages == [1, 4]
    assert sel == [4, 5, 6, 7, 16, 17, 18, 19]


def test_ties_go_to_lower_page_and_budget_rounds_up():
    """Equal relevance everywhere: k = 9 positions -> ceil(9/4) = 3 pages = the last page plus pages
    0 and 1 (the lower of the tied pages)."""
    shape, q, K, pt, lens = _ranked_pages_workload([2, 2, 2, 2, 2, 2])
    idx = oracle.quest_topk(shape, q, K, pt, lens, [9], k_max=12)
    pages, sel = _pages_of(idx[0, 0], 4)
    assert pages == [0, 1, 5]
    assert len(sel) == 12 and (idx[0, 0] >= 0).all()


def test_partial_last_page_and_whole_cache_budget():
    """A budget covering every page returns every position 0..N-1 (the last page holds 2 of 4 slots)."""
    shape, q, K, pt, lens, _ = _int_workload(14, P=4, d=4, seed=5)
    idx = oracle.quest_topk(shape, q, K, pt, lens, [100], k_max=16)
    assert [int(x) for x in idx[0, 0] if x >= 0] == list(range(14))
    assert (idx[0, 0, 14:] == -1).all()


def test_selection_is_the_most_relevant_pages():
    """Random data, several heads: the kept pages other than the current one are exactly the
    ceil(k/P) - 1 most relevant ones (every kept page at least as relevant as every dropped one, a
    tie only ever won by the lower page)."""
    w = wl.make_workload(2, 8, 2, [16 * 40 + 7, 16 * 23], [16 * 6 + 3, 16 * 4], seed=32, k_max=16 * 8)
    shape = w.shape()
    idx = oracle.quest_topk(shape, w.q, w.K, w.page_table, w.lens, w.k, k_max=16 * 8)
    for b in range(2):
        n, kb = int(w.lens[b]), int(w.k[b])
        np_ = (n + 15) // 16
        kp = (kb + 15) // 16
        for h in range(8):
            r = oracle.quest_scores(shape, w.q, w.K, w.page_table, w.lens, b, h)
            pages, sel = _pages_of(idx[b, h], 16)
            assert np_ - 1 in pages and len(pages) == kp
            assert sel == [p for j in pages for p in range(j * 16, min(n, j * 16 + 16))]
            kept = [j for j in pages if j != np_ - 1]
            dropped = [j for j in range(np_ - 1) if j not in kept]
            for i in kept:
                for o in dropped:
                    assert r[i] > r[o] or (r[i] == r[o] and i < o), (b, h, i, o)
