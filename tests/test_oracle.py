"""Pins for the fp64 CPU oracle (CPU only).

The oracle is checked against things other than itself: hand-worked fixtures (tests/golden),
closed forms, brute force on tiny inputs, the library SDPA routine in float64, and invariants the
definition forces.  Sources of the definition: SDPA ("Sparse Attention inference survey" (xllm),
sec. 1.1), exact top-k ("Technische Zusammenfassung: Kontextsparsitaet bei der Inferenzzeit",
sec. 2, Oracle Top-K), selected-rows attention ("Inference-time context sparsity: illusion or
opportunity?", Fig. 1(a)).
"""
from __future__ import annotations

import itertools
import math
import os

import numpy as np
import pytest
import torch

import oracle
from sparse_attention_decode_sd_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
D = 128


def _bf16_exact(x) -> torch.Tensor:
    t = torch.as_tensor(x, dtype=torch.float64)
    b = t.to(torch.bfloat16)
    assert torch.equal(b.double(), t), "fixture value is not exactly representable in bf16"
    return b


def _line_workload(scores, v=None, P=4, vdim=5):
    """One request, one head: q = e_0, K row i = scores[i] * e_0, V row i = v[i] * e_vdim,
    stored through a reversed page table so that paging is exercised."""
    n = len(scores)
    pages = max(1, (n + P - 1) // P)
    q = torch.zeros(1, 1, D, dtype=torch.float64)
    q[0, 0, 0] = 1.0
    Kl = torch.zeros(n, D, dtype=torch.float64)
    Kl[:, 0] = torch.tensor(scores, dtype=torch.float64)
    Vl = torch.zeros(n, D, dtype=torch.float64)
    if v is not None:
        Vl[:, vdim] = torch.tensor(v, dtype=torch.float64)
    pt = torch.arange(pages - 1, -1, -1, dtype=torch.int32).view(1, pages)
    K = torch.zeros(pages, P, 1, D, dtype=torch.float64)
    V = torch.zeros(pages, P, 1, D, dtype=torch.float64)
    for i in range(n):
        K[pt[0, i // P], i % P, 0] = Kl[i]
        V[pt[0, i // P], i % P, 0] = Vl[i]
    shape = dict(B=1, Hq=1, Hkv=1, d=D, P=P, max_pages=pages)
    return shape, _bf16_exact(q), _bf16_exact(K), _bf16_exact(V), pt, torch.tensor([n], dtype=torch.int32)


def _read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            rows.append([part.split() for part in line.split("|")])
    return rows


# ----------------------------------------------------------------------------------------------
# selection
# ----------------------------------------------------------------------------------------------

def test_golden_topk_ties():
    cases = _read_golden("topk_ties.txt")
    assert len(cases) >= 10
    for scores, k, expected in cases:
        scores = [float(x) for x in scores]
        k = int(k[0])
        expected = [int(x) for x in expected]
        shape, q, K, V, pt, lens = _line_workload(scores)
        idx = oracle.topk(shape, q, K, pt, lens, [k], k_max=k)
        got = [int(x) for x in idx[0, 0] if x >= 0]
        assert got == expected, (scores, k)
        assert all(x == -1 for x in idx[0, 0, len(expected):])


def _brute_topk(s, k):
    """Exhaustive: the size-min(k,n) subset with the largest score sum; among equal sums, the one
    whose ascending positions are lexicographically smallest (= ties to the lower position)."""
    n = len(s)
    m = min(k, n)
    best, best_key = None, None
    for sub in itertools.combinations(range(n), m):
        key = (-sum(s[i] for i in sub), sub)
        if best_key is None or key < best_key:
            best, best_key = sub, key
    return list(best)


def test_topk_brute_force_tiny():
    rng = np.random.default_rng(7)
    checked = 0
    for trial in range(300):
        n = int(rng.integers(1, 13))
        k = int(rng.integers(1, n + 2))
        # small integers: many exact ties; exactly representable; sums exact in double
        scores = rng.integers(-4, 5, size=n).astype(float).tolist()
        shape, q, K, V, pt, lens = _line_workload(scores)
        idx = oracle.topk(shape, q, K, pt, lens, [k], k_max=max(k, 1))
        got = [int(x) for x in idx[0, 0] if x >= 0]
        assert got == _brute_topk(scores, k), (scores, k)
        checked += 1
    assert checked == 300


def test_topk_brute_force_random_real_scores():
    """Brute force against real-valued scores from random bf16 q/K, several heads and a GQA group,
    through a shuffled page table, ragged lengths."""
    for seed in range(4):
        w = wl.make_workload(2, 4, 2, [11, 7], [3, 5], seed=seed, P=4)
        idx = oracle.topk(w.shape(), w.q, w.K, w.page_table, w.lens, w.k)
        for b in range(w.B):
            for h in range(w.Hq):
                s = oracle.scores(w.shape(), w.q, w.K, w.page_table, w.lens, b, h).tolist()
                got = [int(x) for x in idx[b, h] if x >= 0]
                assert got == _brute_topk(s, int(w.k[b])), (seed, b, h)


def test_scores_closed_form_paging_and_gqa():
    """q[b,h] = (h+1) * ones, K row of (b, kvh, i) = v(b,kvh,i) * e_{(5i+kvh) % d}, so the score is
    exactly (h+1) * v(b, h//G, i).  A wrong page, slot, KV-head mapping or dropped term changes it."""
    B, Hq, Hkv, P = 2, 6, 3, 4
    G = Hq // Hkv
    lens = [13, 9]
    pages = [(n + P - 1) // P for n in lens]
    total = sum(pages)
    perm = torch.randperm(total, generator=torch.Generator().manual_seed(3)).to(torch.int32)
    max_pages = max(pages)
    pt = torch.full((B, max_pages), -1, dtype=torch.int32)
    off = 0
    for b in range(B):
        pt[b, :pages[b]] = perm[off:off + pages[b]]
        off += pages[b]
    K = torch.zeros(total, P, Hkv, D, dtype=torch.float64)
    expect = {}
    for b in range(B):
        for kvh in range(Hkv):
            for i in range(lens[b]):
                v = float(((i + 3 * kvh + 7 * b) % 17) - 8)
                K[pt[b, i // P], i % P, kvh, (5 * i + kvh) % D] = v
                expect[(b, kvh, i)] = v
    q = torch.zeros(B, Hq, D, dtype=torch.float64)
    for h in range(Hq):
        q[:, h, :] = h + 1
    shape = dict(B=B, Hq=Hq, Hkv=Hkv, d=D, P=P, max_pages=max_pages)
    qb, Kb = _bf16_exact(q), _bf16_exact(K)
    L = torch.tensor(lens, dtype=torch.int32)
    for b in range(B):
        for h in range(Hq):
            s = oracle.scores(shape, qb, Kb, pt, L, b, h)
            want = [(h + 1) * expect[(b, h // G, i)] for i in range(lens[b])]
            assert s.tolist() == want, (b, h)


def test_topk_edge_cases():
    w = wl.make_workload(3, 4, 2, [0, 5, 20], [3, 9, 20], seed=1, P=4, k_max=20)
    idx = oracle.topk(w.shape(), w.q, w.K, w.page_table, w.lens, w.k)
    assert (idx[0] == -1).all()                              # empty context
    assert (idx[1, :, :5] == np.arange(5)).all() and (idx[1, :, 5:] == -1).all()   # k > N: all rows
    assert (idx[2] == np.arange(20)).all()                   # k == N: all rows


def test_planted_keys_are_selected():
    """tiny workload: each head's 16 planted keys score ~4*|q_h|^2 ~ 512, far above the k-th
    score (~2 sigma ~ 23), so all 16 must be in the head's top-82."""
    w = wl.named("tiny")
    idx = oracle.topk(w.shape(), w.q, w.K, w.page_table, w.lens, w.k)
    assert int(w.k[0]) == 82
    for (b, h), pos in w.meta["planted"].items():
        sel = set(int(x) for x in idx[b, h] if x >= 0)
        assert len(sel) == 82
        assert set(pos.tolist()) <= sel, h


# ----------------------------------------------------------------------------------------------
# attention
# ----------------------------------------------------------------------------------------------

def _gather_rows(w, cache, b, kvh):
    n = int(w.lens[b])
    pos = torch.arange(n)
    pages = w.page_table[b].long()[pos // w.P]
    return cache[pages, pos % w.P, kvh].double()          # [n, d]


def _library_sdpa(w, b, h, mask=None):
    """torch's scaled_dot_product_attention in float64 on the gathered rows."""
    kvh = h // w.G
    Kr = _gather_rows(w, w.K, b, kvh)
    Vr = _gather_rows(w, w.V, b, kvh)
    qh = w.q[b, h].double().view(1, 1, 1, -1)
    am = None
    if mask is not None:
        am = torch.full((1, 1, 1, Kr.shape[0]), float("-inf"), dtype=torch.float64)
        am[..., mask] = 0.0
    o = torch.nn.functional.scaled_dot_product_attention(qh, Kr.view(1, 1, *Kr.shape), Vr.view(1, 1, *Vr.shape),
                                                         attn_mask=am)
    return o.view(-1).numpy()


def test_dense_equals_library_sdpa():
    w = wl.make_workload(2, 8, 2, [37, 50], 50, seed=11, P=16)
    out = oracle.dense(w.shape(), w.q, w.K, w.V, w.page_table, w.lens)
    for b in range(w.B):
        for h in range(w.Hq):
            np.testing.assert_allclose(out[b, h], _library_sdpa(w, b, h), rtol=0, atol=1e-12)


def test_k_equals_n_is_dense():
    w = wl.make_workload(2, 4, 1, [33, 64], [33, 64], seed=5, P=16)
    idx = oracle.topk(w.shape(), w.q, w.K, w.page_table, w.lens, w.k)
    sparse = oracle.attend(w.shape(), w.q, w.K, w.V, w.page_table, w.lens, idx)
    dense = oracle.dense(w.shape(), w.q, w.K, w.V, w.page_table, w.lens)
    np.testing.assert_allclose(sparse, dense, rtol=0, atol=1e-12)
    for b in range(w.B):
        for h in range(w.Hq):
            np.testing.assert_allclose(sparse[b, h], _library_sdpa(w, b, h), rtol=0, atol=1e-12)


def test_any_k_equals_masked_library_sdpa():
    w = wl.make_workload(3, 8, 2, [40, 61, 17], [5, 12, 17], seed=9, P=16)
    idx = oracle.topk(w.shape(), w.q, w.K, w.page_table, w.lens, w.k)
    out = oracle.attend(w.shape(), w.q, w.K, w.V, w.page_table, w.lens, idx)
    for b in range(w.B):
        for h in range(w.Hq):
            sel = [int(x) for x in idx[b, h] if x >= 0]
            np.testing.assert_allclose(out[b, h], _library_sdpa(w, b, h, mask=sel), rtol=0, atol=1e-12)


def test_k1_returns_argmax_row():
    w = wl.make_workload(2, 8, 4, [29, 70], 1, seed=13, P=16)
    idx = oracle.topk(w.shape(), w.q, w.K, w.page_table, w.lens, w.k)
    out = oracle.attend(w.shape(), w.q, w.K, w.V, w.page_table, w.lens, idx)
    for b in range(w.B):
        for h in range(w.Hq):
            s = oracle.scores(w.shape(), w.q, w.K, w.page_table, w.lens, b, h)
            am = int(np.argmax(s))                           # first maximum = lower position
            assert idx[b, h, 0] == am
            row = _gather_rows(w, w.V, b, h // w.G)[am].numpy()
            assert np.array_equal(out[b, h], row)            # softmax over one row is exactly 1


def test_two_rows_logistic_closed_form():
    """Two selected rows: out = sigmoid(dz) V1 + sigmoid(-dz) V2 with dz = (s1 - s2)/sqrt(d)."""
    w = wl.make_workload(1, 2, 1, 45, 2, seed=17, P=16)
    idx = oracle.topk(w.shape(), w.q, w.K, w.page_table, w.lens, w.k)
    out = oracle.attend(w.shape(), w.q, w.K, w.V, w.page_table, w.lens, idx)
    Vr = _gather_rows(w, w.V, 0, 0).numpy()
    for h in range(2):
        s = oracle.scores(w.shape(), w.q, w.K, w.page_table, w.lens, 0, h)
        i1, i2 = [int(x) for x in idx[0, h]]
        dz = (s[i1] - s[i2]) / math.sqrt(D)
        sig = 1.0 / (1.0 + math.exp(-dz))
        np.testing.assert_allclose(out[0, h], sig * Vr[i1] + (1.0 - sig) * Vr[i2], rtol=0, atol=1e-13)


def test_golden_uniform_average():
    for scores, v, sel, expected in _read_golden("uniform_average.txt"):
        scores = [float(x) for x in scores]
        v = [float(x) for x in v]
        sel = [int(x) for x in sel]
        shape, q, K, V, pt, lens = _line_workload(scores, v)
        out = oracle.attend(shape, q, K, V, pt, lens, np.array(sel, dtype=np.int32).reshape(1, 1, -1))
        assert out[0, 0, 5] == pytest.approx(float(expected[0]), abs=1e-14)
        assert np.count_nonzero(out[0, 0]) <= 1


def test_unselected_rows_do_not_matter():
    """Rewriting every unselected K/V row leaves the output bit-identical."""
    w = wl.make_workload(2, 4, 1, [48, 33], [6, 4], seed=21, P=16)
    idx = oracle.topk(w.shape(), w.q, w.K, w.page_table, w.lens, w.k)
    out = oracle.attend(w.shape(), w.q, w.K, w.V, w.page_table, w.lens, idx)
    K2, V2 = w.K.clone(), w.V.clone()
    g = torch.Generator().manual_seed(99)
    for b in range(w.B):
        selected = set(int(x) for x in idx[b].reshape(-1) if x >= 0)
        others = [i for i in range(int(w.lens[b])) if i not in selected]
        perm = torch.tensor(others)[torch.randperm(len(others), generator=g)]
        src_p = w.page_table[b].long()[torch.tensor(others) // w.P]
        dst_p = w.page_table[b].long()[perm // w.P]
        K2[dst_p, perm % w.P] = w.K[src_p, torch.tensor(others) % w.P]
        V2[dst_p, perm % w.P] = w.V[src_p, torch.tensor(others) % w.P]
    out2 = oracle.attend(w.shape(), w.q, K2, V2, w.page_table, w.lens, idx)
    assert np.array_equal(out, out2)


def test_physical_page_placement_does_not_matter():
    w = wl.make_workload(2, 8, 2, [70, 45], [9, 45], seed=23, P=16, page_order="identity")
    perm = torch.randperm(w.num_pages, generator=torch.Generator().manual_seed(4))
    K2 = torch.empty_like(w.K)
    V2 = torch.empty_like(w.V)
    K2[perm] = w.K
    V2[perm] = w.V
    pt2 = w.page_table.clone()
    valid = pt2 >= 0
    pt2[valid] = perm[pt2[valid].long()].to(torch.int32)
    idx1 = oracle.topk(w.shape(), w.q, w.K, w.page_table, w.lens, w.k)
    idx2 = oracle.topk(w.shape(), w.q, K2, pt2, w.lens, w.k)
    assert np.array_equal(idx1, idx2)
    o1 = oracle.attend(w.shape(), w.q, w.K, w.V, w.page_table, w.lens, idx1)
    o2 = oracle.attend(w.shape(), w.q, K2, V2, pt2, w.lens, idx2)
    assert np.array_equal(o1, o2)


def test_v_scaling_is_linear():
    w = wl.make_workload(1, 4, 2, 50, 7, seed=29, P=16)
    idx = oracle.topk(w.shape(), w.q, w.K, w.page_table, w.lens, w.k)
    o1 = oracle.attend(w.shape(), w.q, w.K, w.V, w.page_table, w.lens, idx)
    o2 = oracle.attend(w.shape(), w.q, w.K, (w.V.double() * 4).to(torch.bfloat16), w.page_table, w.lens, idx)
    assert np.array_equal(o2, 4 * o1)


def test_empty_selection_and_empty_context_give_zero():
    w = wl.make_workload(2, 2, 1, [0, 10], 3, seed=31, P=16)
    idx = oracle.topk(w.shape(), w.q, w.K, w.page_table, w.lens, w.k)
    out = oracle.attend(w.shape(), w.q, w.K, w.V, w.page_table, w.lens, idx)
    assert (out[0] == 0).all()
    none = np.full_like(idx, -1)
    assert (oracle.attend(w.shape(), w.q, w.K, w.V, w.page_table, w.lens, none) == 0).all()
    assert (oracle.dense(w.shape(), w.q, w.K, w.V, w.page_table, w.lens)[0] == 0).all()


def test_rejects_out_of_range_arguments():
    w = wl.make_workload(1, 2, 1, 20, 3, seed=1, P=16)
    bad = np.array([[[0, 25, -1]] * 2], dtype=np.int32)     # position beyond N_b
    with pytest.raises(ValueError):
        oracle.attend(w.shape(), w.q, w.K, w.V, w.page_table, w.lens, bad)
    with pytest.raises(ValueError):
        oracle.topk(w.shape(), w.q, w.K, w.page_table, w.lens, [0])     # k < 1
    pt = w.page_table.clone()
    pt[0, 0] = w.num_pages + 5
    with pytest.raises(ValueError):
        oracle.topk(w.shape(), w.q, w.K, pt, w.lens, w.k)


def test_k_rounding_matches_printed_values():
    assert [wl.k_for_ratio(n, 50) for n in (4096, 32768, 131072)] == [82, 655, 2621]
    assert wl.k_for_ratio(131072, 10) == 13107 and wl.k_for_ratio(131072, 100) == 1311
    assert wl.k_for_ratio(131072, 1) == 131072 and wl.k_for_ratio(10, 50) == 1
