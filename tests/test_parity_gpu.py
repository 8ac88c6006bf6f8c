"""GPU parity: the CUDA path through the C ABI against the fp64 CPU oracle on the same seeded inputs.

Small cases and the full-size workloads (the five named configurations, in the launch
configuration the benchmark times) are compared element by element on every (b, h) row; the
full-size ones one request at a time.  Rules and tolerances: tests/gpu_helpers.py.
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


def _run_small(w_cpu, check_dense=True):
    w = w_cpu.to(DEV)
    r = gh.Runner(w)
    return gh.full_parity(w_cpu, r, check_dense=check_dense)


def test_tiny_planted_keys():
    w_cpu = wl.named("tiny")
    idx, _ = _run_small(w_cpu)
    for (b, h), pos in w_cpu.meta["planted"].items():
        assert set(pos.tolist()) <= set(idx[b, h].tolist())


SMALL = [
    # B, Hq, Hkv, lens, k, page_order
    (1, 4, 4, [777], [9], "shuffled"),                      # G = 1
    (2, 8, 4, [300, 1], [17, 1], "shuffled"),               # G = 2, N = 1
    (3, 8, 2, [1000, 5000, 37], [20, 700, 37], "shuffled"),  # ragged tails; k == N
    (2, 28, 4, [2500, 1999], [50, 40], "shuffled"),         # G = 7 (Qwen2.5-7B heads)
    (2, 64, 8, [4096, 3000], [82, 60], "identity"),         # G = 8
    (2, 32, 2, [3333, 1500], [67, 30], "shuffled"),         # G = 16
    (4, 8, 2, [0, 15, 16, 17], [3, 20, 1, 5], "shuffled"),  # empty context, k > N, N < 16
    (1, 8, 1, [20000], [1], "shuffled"),                    # k = 1
    (1, 8, 2, [9000], [9000 // 3], "shuffled"),             # dense-ish selection (k = N/3)
    (1, 256, 16, [700], [30], "shuffled"),                  # the most heads supported: Hkv = 16, G = 16
]


@pytest.mark.parametrize("B,Hq,Hkv,lens,k,order", SMALL)
def test_small_shapes(B, Hq, Hkv, lens, k, order):
    w_cpu = wl.make_workload(B, Hq, Hkv, lens, k, seed=sum(lens) + Hq, page_order=order)
    _run_small(w_cpu)


def test_decode_on_oracle_indices():
    """Feeds the oracle's own index sets to the GPU decode: isolates the decode kernel."""
    w_cpu = wl.make_workload(2, 16, 4, [6000, 4100], [120, 90], seed=3)
    w = w_cpu.to(DEV)
    r = gh.Runner(w)
    idx = oracle.topk(w_cpu.shape(), w_cpu.q, w_cpu.K, w_cpu.page_table, w_cpu.lens, w_cpu.k)
    out = r.sparse(torch.from_numpy(idx).to(DEV))
    assert r.device_status() == 0
    ref = oracle.attend(w_cpu.shape(), w_cpu.q, w_cpu.K, w_cpu.V, w_cpu.page_table, w_cpu.lens, idx)
    gh.check_outputs(out.cpu().numpy(), ref)


def test_decode_arbitrary_index_sets():
    """Per-head random subsets (no relation to the scores), different sizes per head, -1 padding."""
    w_cpu = wl.make_workload(2, 16, 2, [5000, 3000], 1, seed=4, k_max=400)
    g = torch.Generator().manual_seed(5)
    idx = torch.full((2, 16, 400), -1, dtype=torch.int32)
    for b in range(2):
        for h in range(16):
            cnt = int(torch.randint(0, 401, (1,), generator=g))
            cnt = min(cnt, int(w_cpu.lens[b]))
            sel = torch.randperm(int(w_cpu.lens[b]), generator=g)[:cnt].sort().values
            idx[b, h, :cnt] = sel.to(torch.int32)
    w = w_cpu.to(DEV)
    r = gh.Runner(w)
    out = r.sparse(idx.to(DEV))
    assert r.device_status() == 0
    ref = oracle.attend(w_cpu.shape(), w_cpu.q, w_cpu.K, w_cpu.V, w_cpu.page_table, w_cpu.lens, idx)
    gh.check_outputs(out.cpu().numpy(), ref)


def test_decode_rows_spanning_many_warps():
    """Few long rows: every row is cut across ~64 decode warps (the segment limit per row), whose
    partials the last warp to finish merges; one row is empty and one holds a single entry."""
    w_cpu = wl.make_workload(1, 4, 1, 9000, 1, seed=12, k_max=6300)
    g = torch.Generator().manual_seed(13)
    idx = torch.full((1, 4, 6300), -1, dtype=torch.int32)
    for h, cnt in enumerate([6300, 0, 1, 5000]):
        idx[0, h, :cnt] = torch.randperm(9000, generator=g)[:cnt].sort().values.to(torch.int32)
    w = w_cpu.to(DEV)
    r = gh.Runner(w)
    out = r.sparse(idx.to(DEV))
    assert r.device_status() == 0
    ref = oracle.attend(w_cpu.shape(), w_cpu.q, w_cpu.K, w_cpu.V, w_cpu.page_table, w_cpu.lens, idx)
    gh.check_outputs(out.cpu().numpy(), ref)
    assert (out[0, 1] == 0).all()


def test_decode_repeated_calls_reuse_the_workspace():
    """The per-row arrival counters are reset by every call: two calls with different index sets on
    one workspace give each call's own result."""
    w_cpu = wl.make_workload(2, 8, 2, [3000, 2000], 1, seed=14, k_max=500)
    g = torch.Generator().manual_seed(15)
    w = w_cpu.to(DEV)
    r = gh.Runner(w)
    for _ in range(2):
        idx = torch.full((2, 8, 500), -1, dtype=torch.int32)
        for b in range(2):
            for h in range(8):
                cnt = int(torch.randint(1, 501, (1,), generator=g))
                idx[b, h, :cnt] = torch.randperm(int(w_cpu.lens[b]), generator=g)[:cnt].sort().values.to(torch.int32)
        out = r.sparse(idx.to(DEV))
        assert r.device_status() == 0
        ref = oracle.attend(w_cpu.shape(), w_cpu.q, w_cpu.K, w_cpu.V, w_cpu.page_table, w_cpu.lens, idx)
        gh.check_outputs(out.cpu().numpy(), ref)


GROUP_WALK = [
    # B, Hq, Hkv, lens, k_max, per-head fraction selected: heads of a group that share many rows
    # (expected duplication G f / (1 - (1 - f)^G) >= 1.4 with f = k_max / capacity) make the decode
    # walk groups (one gathered row serves every head that selected it).  Where the union is expected
    # to cover >= 90% of the positions the walk takes whole tiles with head masks, else only the
    # selected positions.
    (2, 16, 4, [20000, 7000], 12000, 0.6),    # whole tiles: two 16384-position ranges, ragged
    (1, 32, 2, [40000], 30000, 0.7),          # whole tiles, G = 16 (16-bit head masks)
    (3, 8, 2, [50000, 0, 333], 25000, 0.5),   # whole tiles: an empty request and a short one
    (2, 8, 4, [17000, 16384], 16384, 1.0),    # whole tiles, G = 2, k = N: every row, range edges
    (2, 16, 2, [30000, 9000], 4500, 0.15),    # selected positions only (coverage 0.73), G = 8
    (1, 8, 2, [20000], 7000, 0.35),           # selected positions only (coverage 0.82), G = 4
    (1, 32, 2, [40000], 4000, 0.1),           # selected positions only, G = 16 (16-bit masks)
]


@pytest.mark.parametrize("B,Hq,Hkv,lens,k_max,frac", GROUP_WALK)
def test_group_walk_arbitrary_rows(B, Hq, Hkv, lens, k_max, frac):
    """Per-head random subsets of a large fraction of the rows (some heads empty, one with a single
    row), decoded through the group walk, against the oracle on the same rows."""
    w_cpu = wl.make_workload(B, Hq, Hkv, lens, 1, seed=sum(lens) + Hq, k_max=k_max)
    g = torch.Generator().manual_seed(B * 1000 + Hq)
    idx = torch.full((B, Hq, k_max), -1, dtype=torch.int32)
    for b in range(B):
        n = int(w_cpu.lens[b])
        for h in range(Hq):
            cnt = min(k_max, n, int(frac * n))
            if h == 1:
                cnt = 0
            elif h == 2:
                cnt = min(1, n)
            idx[b, h, :cnt] = torch.randperm(n, generator=g)[:cnt].sort().values.to(torch.int32)
    w = w_cpu.to(DEV)
    r = gh.Runner(w)
    out = r.sparse(idx.to(DEV))
    assert r.device_status() == 0
    ref = oracle.attend(w_cpu.shape(), w_cpu.q, w_cpu.K, w_cpu.V, w_cpu.page_table, w_cpu.lens, idx)
    gh.check_outputs(out.cpu().numpy(), ref)
    assert (out[:, 1] == 0).all()


@pytest.mark.parametrize("defect,code", [("swap", sdb.SD_ERR_ORDER), ("past_end", sdb.SD_ERR_INDEX_OOB),
                                         ("after_padding", sdb.SD_ERR_ORDER)])
def test_group_walk_reports_bad_rows(defect, code):
    """Rows checked on the group walk's path (k close to N, where it is taken): a swapped pair, a
    position at N_b and a position after the padding are each reported."""
    B, Hq, Hkv, n = 2, 8, 4, 16384
    w_cpu = wl.make_workload(B, Hq, Hkv, n, 1, seed=5, k_max=n)
    idx = torch.arange(n, dtype=torch.int32).repeat(B, Hq, 1)
    if defect == "swap":
        idx[1, 5, 7000], idx[1, 5, 7001] = 7001, 7000
    elif defect == "past_end":
        idx[0, 2, n - 1] = n
    else:
        idx[1, 6, 9000:] = -1
        idx[1, 6, 12000] = 12000
    w = w_cpu.to(DEV)
    r = gh.Runner(w)
    r.sparse(idx.to(DEV))
    assert r.device_status() == code


@pytest.mark.parametrize("n,k", [(3000, 100), (40000, 100), (40000, 39999)])
def test_exact_ties_go_to_lower_positions(n, k):
    """Identical K rows: every score ties, so the selection is exactly positions 0..k-1.  With N
    large every position passes the candidate threshold, the score pass's candidate segments
    overflow, and the row is recomputed and selected in full."""
    w_cpu = wl.make_workload(1, 4, 1, n, k, seed=7)
    w_cpu.K[:] = w_cpu.K[0, 0, 0]
    w = w_cpu.to(DEV)
    r = gh.Runner(w)
    idx = r.topk().cpu().numpy()
    assert r.device_status() == 0
    assert (idx[0, :, :k] == np.arange(k)).all()
    assert (idx[0, :, k:] == -1).all()


def test_partial_ties_resolved_among_candidates():
    """K rows drawn from 50 distinct vectors: each score value is shared by about 800 positions, so
    the k-th score ties many times over while the candidates still fit their segments.  The
    selection is unique (lowest positions among the tied) and must equal the oracle's exactly."""
    n, k = 40000, 100
    w_cpu = wl.make_workload(2, 8, 2, [n, n - 4321], k, seed=14, page_order="shuffled")
    g = torch.Generator().manual_seed(15)
    for b in range(2):
        nb = int(w_cpu.lens[b])
        pos = torch.arange(nb)
        pages = w_cpu.page_table[b].long()[pos // w_cpu.P]
        slots = pos % w_cpu.P
        src = torch.randint(0, 50, (nb,), generator=g)
        K0 = w_cpu.K[pages[:50], slots[:50]].clone()   # [50][Hkv][128]
        w_cpu.K[pages, slots] = K0[src]
    w = w_cpu.to(DEV)
    r = gh.Runner(w)
    idx = r.topk().cpu().numpy()
    assert r.device_status() == 0
    ref = oracle.topk(w_cpu.shape(), w_cpu.q, w_cpu.K, w_cpu.page_table, w_cpu.lens, w_cpu.k)
    assert np.array_equal(idx, ref)


def test_many_requests_per_score_cta():
    """512 requests alternating between thresholded rows (N = 4200 > 3 k + 4096) and rows whose every
    position is a candidate (N = 1000): each score-pass CTA spans four or five requests, so every
    consumer warp's candidate stream crosses request boundaries."""
    B = 512
    lens = [4200 if b % 2 == 0 else 1000 for b in range(B)]
    lens[5] = 4199
    w_cpu = wl.make_workload(B, 2, 1, lens, 3, seed=16, page_order="shuffled")
    _run_small(w_cpu, check_dense=False)


def test_sampled_threshold_misplaced_falls_back():
    """Every 32nd position scores high and all others score exactly 0.  The selector's strided sample
    sees only the high positions, so its candidate threshold admits fewer rows than k; the exact
    fallback must still return the 2048 high rows plus the lowest-position zeros."""
    n, k = 65536, 3000
    w_cpu = wl.make_workload(1, 1, 1, n, k, seed=12, page_order="shuffled")
    q = w_cpu.q[0, 0]
    high = torch.zeros(n, dtype=torch.bool)
    high[::32] = True
    pos = torch.arange(n)
    pages = w_cpu.page_table[0].long()[pos // w_cpu.P]
    slots = pos % w_cpu.P
    K = w_cpu.K
    K[pages, slots, 0] = 0
    K[pages[high], slots[high], 0] = q
    w = w_cpu.to(DEV)
    r = gh.Runner(w)
    idx = r.topk().cpu().numpy()
    assert r.device_status() == 0
    expect = sorted(set(range(0, n, 32)) | set([p for p in range(n) if p % 32][: k - 2048]))
    assert idx[0, 0, :k].tolist() == expect


def test_zero_scores_are_ties():
    """K = 0 gives +0/-0 scores, which compare equal: the lowest positions win."""
    w_cpu = wl.make_workload(1, 4, 2, 2000, 10, seed=8)
    w_cpu.K.zero_()
    w_cpu.q[0, 1] = -w_cpu.q[0, 1].abs()
    w = w_cpu.to(DEV)
    r = gh.Runner(w)
    idx = r.topk().cpu().numpy()
    assert r.device_status() == 0
    assert (idx[0, :, :10] == np.arange(10)).all()


def test_deterministic_and_placement_invariant():
    """Two runs are bit-identical; moving pages to other physical slots changes nothing."""
    w_cpu = wl.make_workload(2, 16, 4, [7000, 5000], [140, 100], seed=9, page_order="identity")
    w = w_cpu.to(DEV)
    r = gh.Runner(w)
    i1, o1 = r.topk(), None
    o1 = r.sparse(i1)
    d1 = r.dense()
    i2 = r.topk()
    o2 = r.sparse(i2)
    assert torch.equal(i1, i2) and torch.equal(o1, o2)
    perm = torch.randperm(w_cpu.num_pages, generator=torch.Generator().manual_seed(1))
    w2 = w_cpu.to("cpu")
    K2 = torch.empty_like(w2.K)
    V2 = torch.empty_like(w2.V)
    K2[perm] = w2.K
    V2[perm] = w2.V
    pt2 = w2.page_table.clone()
    valid = pt2 >= 0
    pt2[valid] = perm[pt2[valid].long()].to(torch.int32)
    w2.K, w2.V, w2.page_table = K2, V2, pt2
    r2 = gh.Runner(w2.to(DEV))
    i3 = r2.topk()
    o3 = r2.sparse(i3)
    d3 = r2.dense()
    assert r.device_status() == 0 and r2.device_status() == 0
    assert torch.equal(i1, i3) and torch.equal(o1, o3) and torch.equal(d1, d3)


def test_llama8b_full():
    w_cpu = wl.named("llama8b")
    _run_small(w_cpu, check_dense=True)


def _big(name, **kw):
    torch.cuda.empty_cache()
    w = wl.named(name, device=DEV, **kw)
    return w, gh.Runner(w)


def test_long128k_all_groups():
    """Long-context workload (B = 4, 64/8 heads, N = 131072, k = 2621), in the launch configuration
    the benchmark times: every (request, head) row against the oracle, sparse and dense decode."""
    w, r = _big("long128k")
    idx = r.topk()
    out = r.sparse(idx)
    dense = r.dense()
    assert r.device_status() == 0
    gh.all_requests_parity(w, idx, out, dense=dense)
    # attention sinks: K rows 0-3 are scaled by 3; every index row is full
    assert (idx[:, :, :2621] >= 0).all()


@pytest.mark.parametrize("ratio", [10, 50, 100, 1])
def test_sweep128k_all_groups(ratio):
    """Sparsity sweep (B = 16, 32/8 heads, N = 131072, k = N/10, N/50, N/100, N): every row."""
    w, r = _big("sweep128k", ratio=ratio)
    idx = r.topk()
    out = r.sparse(idx)
    dense = r.dense() if ratio == 1 else None
    assert r.device_status() == 0
    gh.all_requests_parity(w, idx, out, dense=dense)
    if ratio == 1:
        # k = N: both read every row; the sparse decode sums per head and the dense one per GQA
        # group, in different segment orders, so only fp32 rounding (and the bf16 hi + lo split of
        # the weights) differs
        assert torch.allclose(out, dense, rtol=1e-3, atol=1e-5)


def test_ragged_steps_with_append():
    """Ragged agentic batch (32 requests, N_b in [8192, 163840], k_b = N_b / 50) over 64 decode steps
    with one K/V row appended per request per step: every row checked at steps 0, 32 and 63."""
    w, r = _big("ragged")
    steps = w.meta["steps"]
    ratio = w.meta["ratio"]
    checks = {0, steps // 2, steps - 1}
    for t in range(steps):
        w.q = w.meta["q_steps"][t].contiguous()
        sdb.sd_append_kv(r.shape, w.K, w.V, w.page_table, w.lens, w.meta["k_new"][t], w.meta["v_new"][t], w.k, ratio,
                         r.status)
        idx = r.topk()
        out = r.sparse(idx)
        if t in checks:
            assert r.device_status() == 0
            lens = w.lens.cpu()
            assert int(w.k[0]) == wl.k_for_ratio(int(lens[0]), ratio)
            gh.all_requests_parity(w, idx, out)
    assert r.device_status() == 0


# ----------------------------------------------------------------------------------------------
# device-side error reporting (every bad value below is caught by the kernels' own checks)
# ----------------------------------------------------------------------------------------------

def _err_setup():
    w_cpu = wl.make_workload(2, 8, 2, [500, 300], [10, 10], seed=11)
    return w_cpu.to(DEV)


def test_index_out_of_range_is_reported():
    w = _err_setup()
    r = gh.Runner(w)
    idx = r.topk()
    assert r.device_status() == 0
    idx[1, 3, 9] = 400          # >= N_1 = 300, still ascending
    r.sparse(idx)
    assert r.device_status() == sdb.SD_ERR_INDEX_OOB


def test_unsorted_indices_are_reported():
    w = _err_setup()
    r = gh.Runner(w)
    idx = r.topk()
    row = idx[0, 2, :10].flip(0).clone()
    idx[0, 2, :10] = row
    r.sparse(idx)
    assert r.device_status() == sdb.SD_ERR_ORDER


def test_entry_after_padding_is_reported():
    w = _err_setup()
    r = gh.Runner(w)
    idx = r.topk()
    assert r.device_status() == 0
    idx[0, 5, 4] = -1           # padding inside the row, selected entries after it
    r.sparse(idx)
    assert r.device_status() == sdb.SD_ERR_ORDER


def test_bad_page_entry_is_reported():
    w = _err_setup()
    w.page_table[0, 3] = w.num_pages + 10
    r = gh.Runner(w)
    r.topk()
    assert r.device_status() == sdb.SD_ERR_INDEX_OOB
    r.status.zero_()
    r.dense()
    assert r.device_status() == sdb.SD_ERR_INDEX_OOB


def test_bad_k_and_length_are_reported():
    w = _err_setup()
    r = gh.Runner(w)
    k = torch.tensor([0, 10], dtype=torch.int32, device=DEV)
    idx = r.topk(k=k)
    assert r.device_status() == sdb.SD_ERR_INVALID_ARG
    assert (idx[0] == -1).all()
    r.status.zero_()
    w.lens[1] = w.max_pages * w.P + 1
    r.dense()
    assert r.device_status() == sdb.SD_ERR_INVALID_ARG


def test_bounded_wait_gives_up_and_the_context_survives():
    """Failure detection without a fault: a device-side wait on a barrier nothing completes gives up after
    its limit and records SD_ERR_TIMEOUT; the context then still runs the indexer and decode correctly."""
    import time
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    sdb.sd_selftest_wait_timeout(50, st)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert int(st.item()) == sdb.SD_ERR_TIMEOUT
    assert 0.045 <= dt < 5.0, dt
    w_cpu = wl.make_workload(1, 8, 2, 3000, 50, seed=91)
    _run_small(w_cpu)
