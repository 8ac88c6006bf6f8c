"""sd_topk_index_static: the top-k indexer for callers that cannot allocate device memory (a plugin
handed only its inputs and outputs, a service with a fixed device-memory plan).  It keeps its
workspace (score rows, candidate counts) in a 48 MiB array inside the library instead of a caller
workspace.

Checked through the C ABI against sd_topk_index with an ordinary workspace, on calls in a row with
different shapes in both orders (a small call after a large one reuses an array whose candidate
records and thresholds the large call left behind, and the reverse), and the size limit is rejected
before any launch.  This file is collected last on purpose."""
from __future__ import annotations

import ctypes

import pytest
import torch

from sparse_attention_decode_sd_b200 import binding as sdb
from sparse_attention_decode_sd_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _both(w):
    shape = sdb.shape_of(w)
    ws = sdb.workspace_for(shape, sdb.SD_OP_TOPK, w.q.device)
    st_ref = torch.zeros(1, dtype=torch.int32, device=w.q.device)
    st_static = torch.zeros(1, dtype=torch.int32, device=w.q.device)
    ref = torch.full((w.B, w.Hq, w.k_max), -7, dtype=torch.int32, device=w.q.device)
    got = torch.full_like(ref, -7)
    sdb.sd_topk_index(shape, w.q, w.K, w.page_table, w.lens, w.k, ref, ws, st_ref)
    lib = sdb.load()
    status = lib.sd_topk_index_static(ctypes.byref(shape), ctypes.c_void_p(w.q.data_ptr()),
                                      ctypes.c_void_p(w.K.data_ptr()), ctypes.c_void_p(w.page_table.data_ptr()),
                                      ctypes.c_void_p(w.lens.data_ptr()), ctypes.c_void_p(w.k.data_ptr()),
                                      ctypes.c_void_p(got.data_ptr()), ctypes.c_void_p(st_static.data_ptr()),
                                      ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert status == sdb.SD_OK
    torch.cuda.synchronize()
    assert int(st_ref.item()) == 0 and int(st_static.item()) == 0
    return ref, got


def test_static_scratch_matches_workspace_version_twice():
    small = wl.make_workload(2, 16, 4, [9000, 5000], [180, 100], seed=41, device="cuda")
    # one long-context request: about 33 MiB of the 48 MiB array
    large = wl.make_workload(1, 64, 8, 131072, 2621, seed=42, structure="sinks3", device="cuda")
    for w in (small, large, small, large):
        ref, got = _both(w)
        assert torch.equal(ref, got)   # integer output: identical


def test_static_scratch_rejects_shapes_beyond_its_size():
    shape = sdb.make_shape(2, 64, 8, 8192, 2621, 16384)   # 2 * 64 * 131072 scores alone = 64 MiB
    fake = ctypes.c_void_p(1 << 20)
    status = sdb.load().sd_topk_index_static(ctypes.byref(shape), fake, fake, fake, fake, fake, fake, fake, None)
    assert status == sdb.SD_ERR_WORKSPACE
