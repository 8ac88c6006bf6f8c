"""The C-ABI library loads, exports every entry point its header declares, and validates arguments on
the host before any launch.  CPU only: no call here reaches a kernel."""
from __future__ import annotations

import ctypes
import os
import re
import subprocess

import pytest

from sparse_attention_decode_sd_b200 import binding as sdb
from sparse_attention_decode_sd_b200 import build as sdbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sparsedecode.h")


@pytest.fixture(scope="module")
def lib():
    sdbuild.build()
    return sdb.load()


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"SD_API\s+[\w\s\*]+?\b(sd_\w+)\s*\(", text)))


def test_header_declares_the_binding_names():
    assert _declared() == sorted(sdb.EXPORTED)


def test_every_declared_symbol_is_exported(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", sdb.library_path()], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\sT\s(sd_\w+)$", out, flags=re.M))
    for name in _declared():
        assert name in exported, name
        assert hasattr(lib, name)


def test_header_compiles_as_c():
    src = '#include "sparsedecode.h"\nint main(void){ sd_shape s; (void)s; return SD_OK; }\n'
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-fsyntax-only", "-I", os.path.dirname(HEADER), "-x",
                        "c", "-"], input=src, text=True, capture_output=True)
    assert r.returncode == 0, r.stderr


def test_status_strings_and_version(lib):
    assert sdb.status_string(sdb.SD_OK) == "ok"
    for code in range(1, 8):
        assert sdb.status_string(code) not in ("ok", "unknown status")
    assert sdb.status_string(99) == "unknown status"
    assert sdb.version() >= 100


def test_last_cuda_error_starts_clear(lib):
    assert sdb.last_cuda_error() == (0, "cudaSuccess")


def _shape(**kw):
    base = dict(B=4, Hq=64, Hkv=8, max_pages=8192, k_max=2621, num_pages=32768)
    base.update(kw)
    return sdb.make_shape(base["B"], base["Hq"], base["Hkv"], base["max_pages"], base["k_max"], base["num_pages"],
                          base.get("head_dim", 128), base.get("page_size", 16))


def test_workspace_sizes(lib):
    s = _shape()
    topk = sdb.sd_workspace_size(s, sdb.SD_OP_TOPK)
    rows = 4 * 64
    scores = rows * 8192 * 16 * 4                          # fp32 candidate streams, B*Hq*n_cap
    small = rows * 8192 * 8 + rows * 4 + 3 * 8             # (head, page) records, thresholds, pointers
    assert scores + small <= topk <= scores + small + 4 * 256
    # sparse decode: 64 segment partials per (b, h) row (fp32 output + max and sum), per row its
    # length and arrival counter, one length sum per CTA of the row pass (1 row per CTA at k_max
    # 2621), and per row the weight of drawn rows (stochastic selection)
    sparse = sdb.sd_workspace_size(s, sdb.SD_OP_SPARSE)
    need = rows * 64 * (128 * 4 + 8) + rows * 4 * 2 + rows * 4 + rows * 4
    assert need <= sparse <= need + 6 * 256
    # dense decode: min(N, 1280) + 1 segment partials per (b, h) and one row count per 16384 positions
    # of every (b, KV head) group
    dense = sdb.sd_workspace_size(s, sdb.SD_OP_DENSE)
    slots = rows * (1280 + 1)
    need = slots * (128 * 4 + 8) + 4 * 8 * 8 * 4
    assert need <= dense <= need + 3 * 256
    assert sparse % 256 == 0 and dense % 256 == 0 and topk % 256 == 0


def test_workspace_size_of_the_group_walk(lib):
    """A shape whose heads are expected to share most rows (k = N, G = 4) takes the group walk: its
    workspace holds the per-head walk's part (which a stochastic selection, decoded per head, uses),
    the dense decode's partials and range counts, and one head-mask byte per position of each group."""
    B, Hq, Hkv, max_pages, k_max = 4, 32, 8, 1024, 16384
    s = _shape(B=B, Hq=Hq, Hkv=Hkv, max_pages=max_pages, k_max=k_max, num_pages=B * max_pages)
    got = sdb.sd_workspace_size(s, sdb.SD_OP_SPARSE)
    rows = B * Hq
    per_head = rows * 64 * (128 * 4 + 8) + rows * 4 * 3 + rows * 4   # partials, lengths/counters/weights, sums
    slots = rows * (1280 + 1)
    dense = slots * (128 * 4 + 8) + B * Hkv * 1 * 4                    # one 16384-position range per group
    masks = B * Hkv * max_pages * 16
    need = per_head + dense + masks
    assert need <= got <= need + 10 * 256
    # the same shape at 50x sparsity keeps the per-head walk's workspace alone
    s50 = _shape(B=B, Hq=Hq, Hkv=Hkv, max_pages=max_pages, k_max=328, num_pages=B * max_pages)
    assert sdb.sd_workspace_size(s50, sdb.SD_OP_SPARSE) < per_head


def test_sparse_workspace_rejects_entry_count_overflow(lib):
    # B * Hq * k_max entries are counted in int32
    n = ctypes.c_size_t(0)
    st = lib.sd_workspace_size(ctypes.byref(_shape(B=64, Hq=128, Hkv=8, k_max=1 << 18, max_pages=1 << 14)),
                               sdb.SD_OP_SPARSE, ctypes.byref(n))
    assert st == sdb.SD_ERR_UNSUPPORTED


@pytest.mark.parametrize("kw,code", [
    (dict(B=0), sdb.SD_ERR_INVALID_ARG),
    (dict(Hq=60, Hkv=8), sdb.SD_ERR_INVALID_ARG),
    (dict(k_max=0), sdb.SD_ERR_INVALID_ARG),
    (dict(num_pages=0), sdb.SD_ERR_INVALID_ARG),
    (dict(head_dim=64), sdb.SD_ERR_UNSUPPORTED),
    (dict(page_size=32), sdb.SD_ERR_UNSUPPORTED),
    (dict(Hq=136, Hkv=4), sdb.SD_ERR_UNSUPPORTED),   # G = 34 > 16
    (dict(Hkv=32, Hq=64), sdb.SD_ERR_UNSUPPORTED),   # more than 16 KV heads
])
def test_shape_validation(lib, kw, code):
    n = ctypes.c_size_t(0)
    st = lib.sd_workspace_size(ctypes.byref(_shape(**kw)), sdb.SD_OP_SPARSE, ctypes.byref(n))
    assert st == code


def test_bad_op_and_null_shape(lib):
    n = ctypes.c_size_t(0)
    assert lib.sd_workspace_size(None, sdb.SD_OP_TOPK, ctypes.byref(n)) == sdb.SD_ERR_INVALID_ARG
    assert lib.sd_workspace_size(ctypes.byref(_shape()), 9, ctypes.byref(n)) == sdb.SD_ERR_INVALID_ARG
    assert lib.sd_workspace_size(ctypes.byref(_shape()), sdb.SD_OP_TOPK, None) == sdb.SD_ERR_INVALID_ARG


def test_null_and_misaligned_pointers_rejected_before_launch(lib):
    s = ctypes.byref(_shape())
    fake = ctypes.c_void_p(1 << 20)       # never dereferenced: validation fails first
    odd = ctypes.c_void_p((1 << 20) + 2)
    N = None
    ws = ctypes.c_size_t(1 << 40)
    assert lib.sd_topk_index(s, N, fake, fake, fake, fake, fake, fake, ws, fake, N) == sdb.SD_ERR_INVALID_ARG
    assert lib.sd_topk_index(s, odd, fake, fake, fake, fake, fake, fake, ws, fake, N) == sdb.SD_ERR_INVALID_ARG
    assert lib.sd_sparse_decode(s, fake, fake, fake, fake, fake, N, fake, fake, ws, fake, N) == sdb.SD_ERR_INVALID_ARG
    assert lib.sd_sparse_decode(s, fake, fake, odd, fake, fake, fake, fake, fake, ws, fake, N) == sdb.SD_ERR_INVALID_ARG
    assert lib.sd_dense_decode(s, fake, fake, fake, fake, fake, fake, N, ws, fake, N) == sdb.SD_ERR_INVALID_ARG
    assert lib.sd_append_kv(s, fake, fake, fake, fake, fake, fake, N, 0, fake, N) == sdb.SD_ERR_INVALID_ARG
    assert lib.sd_append_kv(s, fake, fake, fake, fake, N, fake, N, 50, fake, N) == sdb.SD_ERR_INVALID_ARG
    # the append that keeps Quest boxes: boxes required and 16-byte aligned, then the append's own checks
    assert lib.sd_quest_append_kv(s, fake, fake, fake, fake, fake, fake, N, 50, N, fake, N) == sdb.SD_ERR_INVALID_ARG
    assert lib.sd_quest_append_kv(s, fake, fake, fake, fake, fake, fake, N, 50, odd, fake, N) == sdb.SD_ERR_INVALID_ARG
    assert lib.sd_quest_append_kv(s, fake, fake, fake, fake, N, fake, N, 50, fake, fake, N) == sdb.SD_ERR_INVALID_ARG
    # stochastic selection: k_samp required, then the exact indexer's checks (idx null)
    assert lib.sd_stochastic_index(s, fake, fake, fake, fake, fake, N, 1, 0, fake, fake, ws, fake, N) == \
        sdb.SD_ERR_INVALID_ARG
    assert lib.sd_stochastic_index(s, fake, fake, fake, fake, fake, fake, 1, 0, N, fake, ws, fake, N) == \
        sdb.SD_ERR_INVALID_ARG
    assert lib.sd_sparse_decode_sampled(s, fake, fake, fake, fake, fake, N, fake, fake, ws, fake, N) == \
        sdb.SD_ERR_INVALID_ARG


def test_small_workspace_rejected_before_launch(lib):
    s = ctypes.byref(_shape())
    fake = ctypes.c_void_p(1 << 20)
    small = ctypes.c_size_t(1024)
    assert lib.sd_topk_index(s, fake, fake, fake, fake, fake, fake, fake, small, fake, None) == sdb.SD_ERR_WORKSPACE
    assert lib.sd_sparse_decode(s, fake, fake, fake, fake, fake, fake, fake, fake, small, fake, None) == \
        sdb.SD_ERR_WORKSPACE
    assert lib.sd_dense_decode(s, fake, fake, fake, fake, fake, fake, fake, small, fake, None) == sdb.SD_ERR_WORKSPACE


def test_library_does_not_link_the_oracle():
    out = subprocess.run(["nm", "-D", sdb.library_path()], capture_output=True, text=True, check=True).stdout
    assert "oracle_" not in out
    ldd = subprocess.run(["ldd", sdb.library_path()], capture_output=True, text=True).stdout
    assert "oracle" not in ldd
