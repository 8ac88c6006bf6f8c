"""ctypes binding of libsparsedecode (include/sparsedecode.h): argument marshalling only.

Every function takes torch tensors that already live on the current CUDA device, passes their
device pointers to the C entry point of the same name on the current stream (or `stream`), and
returns the host status.  No computation happens here and there is no fallback: if the shared
library is missing, loading raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsparsedecode.so")
_lib = None

SD_OK = 0
SD_ERR_INVALID_ARG = 1
SD_ERR_UNSUPPORTED = 2
SD_ERR_CUDA = 3
SD_ERR_INDEX_OOB = 4
SD_ERR_TIMEOUT = 5
SD_ERR_WORKSPACE = 6
SD_ERR_ORDER = 7

SD_OP_TOPK = 1
SD_OP_SPARSE = 2
SD_OP_DENSE = 3
SD_OP_QUEST = 4

SD_SAMPLED_FLAG = 1 << 30   # idx entry of a row drawn by sd_stochastic_index (position in the low 30 bits)

EXPORTED = ("sd_workspace_size", "sd_topk_index", "sd_topk_scores", "sd_topk_select", "sd_topk_index_static",
            "sd_sparse_decode", "sd_stochastic_index", "sd_sparse_decode_sampled", "sd_dense_decode", "sd_append_kv",
            "sd_quest_summarize", "sd_quest_append_kv", "sd_quest_index", "sd_selftest_wait_timeout", "sd_status_string",
            "sd_last_cuda_error", "sd_version")


class SdShape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("num_q_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("page_size", ctypes.c_int32), ("max_pages_per_req", ctypes.c_int32),
                ("k_max", ctypes.c_int32), ("num_pages", ctypes.c_int32)]


class SdError(RuntimeError):
    def __init__(self, status: int, what: str):
        msg = f"{what}: {status_string(status)} (status {status})"
        if status == SD_ERR_CUDA:
            code, name = last_cuda_error()
            msg += f": {name} ({code})"
        super().__init__(msg)
        self.status = status


def library_path() -> str:
    return _LIB_PATH


def load():
    """Loads libsparsedecode.so (built by sparse_attention_decode_sd_b200.build)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(f"libsparsedecode.so not found at {_LIB_PATH}; run "
                           "`python -m sparse_attention_decode_sd_b200.build` first")
    lib = ctypes.CDLL(_LIB_PATH)
    P, I32, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    SH = ctypes.POINTER(SdShape)
    lib.sd_workspace_size.argtypes = [SH, I32, ctypes.POINTER(SZ)]
    lib.sd_topk_index.argtypes = [SH, P, P, P, P, P, P, P, SZ, P, P]
    lib.sd_topk_scores.argtypes = [SH, P, P, P, P, P, P, SZ, P, P]
    lib.sd_topk_select.argtypes = [SH, P, P, P, P, SZ, P, P]
    lib.sd_topk_index_static.argtypes = [SH, P, P, P, P, P, P, P, P]
    lib.sd_topk_index_static.restype = I32
    lib.sd_sparse_decode.argtypes = [SH, P, P, P, P, P, P, P, P, SZ, P, P]
    lib.sd_sparse_decode_sampled.argtypes = [SH, P, P, P, P, P, P, P, P, SZ, P, P]
    lib.sd_stochastic_index.argtypes = [SH, P, P, P, P, P, P, ctypes.c_uint64, ctypes.c_uint32, P, P, SZ, P, P]
    lib.sd_dense_decode.argtypes = [SH, P, P, P, P, P, P, P, SZ, P, P]
    lib.sd_append_kv.argtypes = [SH, P, P, P, P, P, P, P, I32, P, P]
    lib.sd_quest_append_kv.argtypes = [SH, P, P, P, P, P, P, P, I32, P, P, P]
    lib.sd_quest_summarize.argtypes = [SH, P, P, P, P, I32, P, P]
    lib.sd_quest_index.argtypes = [SH, P, P, P, P, P, P, P, SZ, P, P]
    lib.sd_selftest_wait_timeout.argtypes = [ctypes.c_uint32, P, P]
    lib.sd_selftest_wait_timeout.restype = I32
    for f in (lib.sd_workspace_size, lib.sd_topk_index, lib.sd_topk_scores, lib.sd_topk_select, lib.sd_sparse_decode,
              lib.sd_sparse_decode_sampled, lib.sd_stochastic_index, lib.sd_dense_decode, lib.sd_append_kv,
              lib.sd_quest_summarize, lib.sd_quest_append_kv, lib.sd_quest_index):
        f.restype = I32
    lib.sd_status_string.argtypes = [I32]
    lib.sd_status_string.restype = ctypes.c_char_p
    lib.sd_last_cuda_error.argtypes = [ctypes.POINTER(ctypes.c_char_p)]
    lib.sd_last_cuda_error.restype = I32
    lib.sd_version.argtypes = []
    lib.sd_version.restype = I32
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().sd_status_string(int(status)).decode()


def last_cuda_error() -> tuple[int, str]:
    """(cudaError_t value, its name) behind the last SD_ERR_CUDA on this thread."""
    name = ctypes.c_char_p()
    code = load().sd_last_cuda_error(ctypes.byref(name))
    return int(code), (name.value or b"").decode()


def version() -> int:
    return int(load().sd_version())


def make_shape(B, Hq, Hkv, max_pages, k_max, num_pages, head_dim=128, page_size=16) -> SdShape:
    return SdShape(int(B), int(Hq), int(Hkv), int(head_dim), int(page_size), int(max_pages), int(k_max), int(num_pages))


def shape_of(w) -> SdShape:
    """SdShape of a workloads.Workload."""
    return make_shape(w.B, w.Hq, w.Hkv, w.max_pages, w.k_max, w.num_pages, w.d, w.P)


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _check(status: int, what: str, check: bool) -> int:
    if check and status != SD_OK:
        raise SdError(status, what)
    return status


def sd_workspace_size(shape: SdShape, op: int) -> int:
    n = ctypes.c_size_t(0)
    st = load().sd_workspace_size(ctypes.byref(shape), int(op), ctypes.byref(n))
    _check(st, "sd_workspace_size", True)
    return int(n.value)


def _ws_bytes(workspace):
    return 0 if workspace is None else workspace.numel() * workspace.element_size()


def sd_topk_index(shape, q, K, page_table, lens, k, idx, workspace, dev_status, stream=None, check=True) -> int:
    st = load().sd_topk_index(ctypes.byref(shape), _ptr(q), _ptr(K), _ptr(page_table), _ptr(lens), _ptr(k), _ptr(idx),
                              _ptr(workspace), _ws_bytes(workspace), _ptr(dev_status), _stream(stream))
    return _check(st, "sd_topk_index", check)


def sd_topk_scores(shape, q, K, page_table, lens, k, workspace, dev_status, stream=None, check=True) -> int:
    st = load().sd_topk_scores(ctypes.byref(shape), _ptr(q), _ptr(K), _ptr(page_table), _ptr(lens), _ptr(k),
                               _ptr(workspace), _ws_bytes(workspace), _ptr(dev_status), _stream(stream))
    return _check(st, "sd_topk_scores", check)


def sd_topk_select(shape, lens, k, idx, workspace, dev_status, stream=None, check=True) -> int:
    st = load().sd_topk_select(ctypes.byref(shape), _ptr(lens), _ptr(k), _ptr(idx), _ptr(workspace),
                               _ws_bytes(workspace), _ptr(dev_status), _stream(stream))
    return _check(st, "sd_topk_select", check)


def sd_topk_index_static(shape, q, K, page_table, lens, k, idx, dev_status, stream=None, check=True) -> int:
    """sd_topk_index with the library's own static 48 MiB scratch (no workspace argument)."""
    st = load().sd_topk_index_static(ctypes.byref(shape), _ptr(q), _ptr(K), _ptr(page_table), _ptr(lens), _ptr(k),
                                     _ptr(idx), _ptr(dev_status), _stream(stream))
    return _check(st, "sd_topk_index_static", check)


def sd_sparse_decode(shape, q, K, V, page_table, lens, idx, out, workspace, dev_status, stream=None,
                     check=True) -> int:
    st = load().sd_sparse_decode(ctypes.byref(shape), _ptr(q), _ptr(K), _ptr(V), _ptr(page_table), _ptr(lens),
                                 _ptr(idx), _ptr(out), _ptr(workspace), _ws_bytes(workspace), _ptr(dev_status),
                                 _stream(stream))
    return _check(st, "sd_sparse_decode", check)


def sd_stochastic_index(shape, q, K, page_table, lens, k_det, k_samp, seed, step, idx, workspace, dev_status,
                        stream=None, check=True) -> int:
    st = load().sd_stochastic_index(ctypes.byref(shape), _ptr(q), _ptr(K), _ptr(page_table), _ptr(lens), _ptr(k_det),
                                    _ptr(k_samp), ctypes.c_uint64(int(seed) & 0xFFFFFFFFFFFFFFFF),
                                    ctypes.c_uint32(int(step) & 0xFFFFFFFF), _ptr(idx), _ptr(workspace),
                                    _ws_bytes(workspace), _ptr(dev_status), _stream(stream))
    return _check(st, "sd_stochastic_index", check)


def sd_sparse_decode_sampled(shape, q, K, V, page_table, lens, idx, out, workspace, dev_status, stream=None,
                             check=True) -> int:
    st = load().sd_sparse_decode_sampled(ctypes.byref(shape), _ptr(q), _ptr(K), _ptr(V), _ptr(page_table),
                                         _ptr(lens), _ptr(idx), _ptr(out), _ptr(workspace), _ws_bytes(workspace),
                                         _ptr(dev_status), _stream(stream))
    return _check(st, "sd_sparse_decode_sampled", check)


def sd_dense_decode(shape, q, K, V, page_table, lens, out, workspace, dev_status, stream=None, check=True) -> int:
    st = load().sd_dense_decode(ctypes.byref(shape), _ptr(q), _ptr(K), _ptr(V), _ptr(page_table), _ptr(lens),
                                _ptr(out), _ptr(workspace), _ws_bytes(workspace), _ptr(dev_status), _stream(stream))
    return _check(st, "sd_dense_decode", check)


def sd_quest_summarize(shape, K, page_table, lens, boxes, dev_status, last_page_only=False, stream=None,
                       check=True) -> int:
    st = load().sd_quest_summarize(ctypes.byref(shape), _ptr(K), _ptr(page_table), _ptr(lens), _ptr(boxes),
                                   int(bool(last_page_only)), _ptr(dev_status), _stream(stream))
    return _check(st, "sd_quest_summarize", check)


def sd_quest_index(shape, q, boxes, page_table, lens, k, idx, workspace, dev_status, stream=None, check=True) -> int:
    st = load().sd_quest_index(ctypes.byref(shape), _ptr(q), _ptr(boxes), _ptr(page_table), _ptr(lens), _ptr(k),
                               _ptr(idx), _ptr(workspace), ctypes.c_size_t(workspace.numel()), _ptr(dev_status),
                               _stream(stream))
    return _check(st, "sd_quest_index", check)


def sd_selftest_wait_timeout(wait_ms: int, dev_status, stream=None, check=True) -> int:
    st = load().sd_selftest_wait_timeout(int(wait_ms), _ptr(dev_status), _stream(stream))
    return _check(st, "sd_selftest_wait_timeout", check)


def quest_boxes_for(shape: SdShape, device=None) -> torch.Tensor:
    """A caller-side buffer for the Quest page boxes: bf16 [num_pages][Hkv][2][head_dim]."""
    return torch.empty((shape.num_pages, shape.num_kv_heads, 2, shape.head_dim), dtype=torch.bfloat16,
                       device=device or "cuda")


def sd_append_kv(shape, K, V, page_table, lens, k_new, v_new, k_sel, ratio, dev_status, stream=None,
                 check=True) -> int:
    st = load().sd_append_kv(ctypes.byref(shape), _ptr(K), _ptr(V), _ptr(page_table), _ptr(lens), _ptr(k_new),
                             _ptr(v_new), _ptr(k_sel), int(ratio), _ptr(dev_status), _stream(stream))
    return _check(st, "sd_append_kv", check)


def sd_quest_append_kv(shape, K, V, page_table, lens, k_new, v_new, k_sel, ratio, boxes, dev_status, stream=None,
                       check=True) -> int:
    """sd_append_kv that also brings the Quest box of each written page up to date."""
    st = load().sd_quest_append_kv(ctypes.byref(shape), _ptr(K), _ptr(V), _ptr(page_table), _ptr(lens), _ptr(k_new),
                                   _ptr(v_new), _ptr(k_sel), int(ratio), _ptr(boxes), _ptr(dev_status),
                                   _stream(stream))
    return _check(st, "sd_quest_append_kv", check)


def workspace_for(shape: SdShape, op: int, device=None) -> torch.Tensor:
    """A caller-side workspace buffer of the size the library asks for (uint8, 256-byte aligned)."""
    n = sd_workspace_size(shape, op)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device or "cuda")


def read_status(dev_status: torch.Tensor) -> int:
    """Synchronises dev_status's stream and returns the device-side status word."""
    return int(dev_status.item())
