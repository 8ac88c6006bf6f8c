"""Pins of the oracle's stochastic index selection (vAttention-style; "Technische
Zusammenfassung: Kontextsparsitaet bei der Inferenzzeit", sec. 2 "Stochastische Indexierung" and
sec. 3A; the estimator is the reading stated at the top of oracle/oracle.c): exact top-k_det
rows plus m rows drawn uniformly without replacement from the rest, each sampled row weighted by
|rest| / m in the softmax's numerator and denominator.

Each check is against something other than the oracle itself: the generator's published outputs,
the oracle's own exact and dense paths (k_samp = 0 and k_samp = |rest| reduce to them), brute force
over every possible sample (unbiasedness of both sums, an exact identity), and the binomial law of
how often each row is drawn.  CPU only.
"""
from __future__ import annotations

import itertools
import math
import os

import numpy as np
import torch

import oracle
from sparse_attention_decode_sd_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "splitmix64_seed0.txt")
FLAG = oracle.SAMPLED_FLAG
MASK = FLAG - 1


def _golden_vectors():
    out = []
    for line in open(GOLDEN):
        line = line.split("#")[0].strip()
        if line:
            i, v = (x.strip() for x in line.split("|"))
            out.append((int(i), int(v, 16)))
    return out


def test_splitmix64_published_outputs():
    golden = 0x9E3779B97F4A7C15
    for i, v in _golden_vectors():
        assert oracle.splitmix64((i - 1) * golden) == v, i


def _case(n, H=4, Hkv=2, seed=21, k_max=None):
    w = wl.make_workload(1, H, Hkv, n, 1, seed=seed, page_order="shuffled", k_max=k_max or n)
    return w


def test_zero_samples_is_exact_topk():
    w = _case(300, k_max=300)
    shape = w.shape()
    for kd in (1, 7, 40):
        ref = oracle.topk(shape, w.q, w.K, w.page_table, w.lens, torch.tensor([kd], dtype=torch.int32))
        got = oracle.stochastic_topk(shape, w.q, w.K, w.page_table, w.lens, [kd], [0], seed=5, step=3)
        assert np.array_equal(got, ref)
        assert not (got[got >= 0] & FLAG).any()


def test_sampling_all_the_rest_is_dense_attention():
    n = 200
    w = _case(n, k_max=n)
    shape = w.shape()
    idx = oracle.stochastic_topk(shape, w.q, w.K, w.page_table, w.lens, [13], [n], seed=9, step=0)
    for h in range(w.Hq):
        row = idx[0, h]
        assert (row >= 0).all()
        assert sorted((row & MASK).tolist()) == list(range(n))
        assert int(((row & FLAG) == 0).sum()) == 13
    got = oracle.attend(shape, w.q, w.K, w.V, w.page_table, w.lens, idx)
    ref = oracle.dense(shape, w.q, w.K, w.V, w.page_table, w.lens)
    assert np.allclose(got, ref, rtol=0, atol=1e-12)


def test_weighted_sums_are_unbiased_over_every_sample():
    """E over all C(|R|, m) equally likely samples of the weighted numerator and denominator equals
    the sums over every row (an exact identity of the inverse-inclusion-probability weight)."""
    n, kd, m = 9, 2, 3
    w = _case(n, H=2, Hkv=1, k_max=n)
    shape = w.shape()
    det = oracle.topk(shape, w.q, w.K, w.page_table, w.lens, torch.tensor([kd], dtype=torch.int32))[0]
    num_all, den_all = oracle.attend_parts(shape, w.q, w.K, w.V, w.page_table, w.lens,
                                           np.arange(n, dtype=np.int32).reshape(1, 1, n).repeat(2, 1))
    for h in range(2):
        d_set = set(det[h][:kd].tolist())
        rest = [p for p in range(n) if p not in d_set]
        nums, dens = [], []
        for sub in itertools.combinations(rest, m):
            row = sorted([(p, 0) for p in d_set] + [(p, FLAG) for p in sub])
            idx = np.full((1, 2, n), -1, dtype=np.int32)
            idx[0, h, :len(row)] = [p | f for p, f in row]
            num, den = oracle.attend_parts(shape, w.q, w.K, w.V, w.page_table, w.lens, idx)
            nums.append(num[0, h])
            dens.append(den[0, h])
        assert len(nums) == math.comb(n - kd, m)
        assert np.allclose(np.mean(nums, axis=0), num_all[0, h], rtol=1e-12, atol=1e-12)
        assert abs(np.mean(dens) - den_all[0, h]) <= 1e-12 * abs(den_all[0, h])


def test_sample_is_distinct_outside_the_deterministic_rows_and_reproducible():
    n, kd, m = 500, 20, 60
    w = _case(n, k_max=kd + m)
    shape = w.shape()
    a = oracle.stochastic_topk(shape, w.q, w.K, w.page_table, w.lens, [kd], [m], seed=1, step=7)
    b = oracle.stochastic_topk(shape, w.q, w.K, w.page_table, w.lens, [kd], [m], seed=1, step=7)
    c = oracle.stochastic_topk(shape, w.q, w.K, w.page_table, w.lens, [kd], [m], seed=1, step=8)
    det = oracle.topk(shape, w.q, w.K, w.page_table, w.lens, torch.tensor([kd], dtype=torch.int32))
    assert np.array_equal(a, b)
    assert not np.array_equal(a, c)
    for h in range(w.Hq):
        row = a[0, h]
        pos = row & MASK
        assert (np.diff(pos) > 0).all()
        samp = set(pos[(row & FLAG) != 0].tolist())
        plain = set(pos[(row & FLAG) == 0].tolist())
        assert plain == set(det[0, h][:kd].tolist())
        assert len(samp) == m and not (samp & plain)
    # rows of different heads draw different samples
    s0 = set((a[0, 0] & MASK)[(a[0, 0] & FLAG) != 0].tolist())
    s1 = set((a[0, 1] & MASK)[(a[0, 1] & FLAG) != 0].tolist())
    assert s0 != s1


def test_each_rest_row_is_drawn_with_probability_m_over_rest():
    """Over many seeds every row of the rest is drawn m / |R| of the time (binomial, 6 sigma)."""
    n, kd, m, trials = 12, 2, 3, 3000
    w = _case(n, H=1, Hkv=1, k_max=n)
    shape = w.shape()
    counts = np.zeros(n)
    det = None
    for s in range(trials):
        row = oracle.stochastic_topk(shape, w.q, w.K, w.page_table, w.lens, [kd], [m], seed=1000 + s, step=0)[0, 0]
        row = row[row >= 0]
        samp = (row & MASK)[(row & FLAG) != 0]
        assert len(samp) == m and len(set(samp.tolist())) == m
        counts[samp] += 1
        det = set((row & MASK)[(row & FLAG) == 0].tolist())
    p = m / (n - kd)
    sigma = math.sqrt(trials * p * (1 - p))
    for pos in range(n):
        if pos in det:
            assert counts[pos] == 0
        else:
            assert abs(counts[pos] - trials * p) <= 6 * sigma, (pos, counts[pos])


def test_sample_fewer_rows_than_asked_when_the_rest_is_small():
    n = 30
    w = _case(n, k_max=n)
    shape = w.shape()
    idx = oracle.stochastic_topk(shape, w.q, w.K, w.page_table, w.lens, [25], [100], seed=3, step=1)
    for h in range(w.Hq):
        row = idx[0, h]
        assert int((row >= 0).sum()) == n
        row = row[row >= 0]
        assert int(((row & FLAG) != 0).sum()) == 5
        assert sorted((row & MASK).tolist()) == list(range(n))


def _key(seed, step, r, p):
    """The documented sampling key, composed from the generator pinned above."""
    M = 0xFFFFFFFFFFFFFFFF
    c = oracle.splitmix64(oracle.splitmix64(oracle.splitmix64((seed + step) & M) + r & M) + p & M)
    return c >> 32


def test_sample_is_the_rows_with_the_smallest_keys():
    """The drawn rows are exactly the m rows of the rest with the smallest (key, position): the
    selection the GPU has to reproduce bit for bit."""
    n, kd, m, seed, step = 40, 5, 7, 123456789, 42
    w = _case(n, H=4, Hkv=2, k_max=kd + m)
    shape = w.shape()
    idx = oracle.stochastic_topk(shape, w.q, w.K, w.page_table, w.lens, [kd], [m], seed=seed, step=step)
    for h in range(w.Hq):
        row = idx[0, h]
        det = set((row & MASK)[(row & FLAG) == 0].tolist())
        rest = sorted((p for p in range(n) if p not in det), key=lambda p: (_key(seed, step, h, p), p))
        assert set((row & MASK)[(row & FLAG) != 0].tolist()) == set(rest[:m])
