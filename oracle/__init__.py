"""fp64 CPU oracle for exact top-k sparse decode attention.

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg
of ``bench.py`` may use this package; the product library never does.  It is independent of
the CUDA path: it imports nothing from ``sparse_attention_decode_sd_b200`` and shares no code
with it.  The arithmetic lives in ``oracle.c`` (plain loops in double precision); this module
only compiles it with gcc and marshals tensors.

Functions (all inputs are CPU tensors; bf16 tensors are read as their raw 16-bit patterns):

* ``scores(shape, q, K, page_table, lens, b, h)``  -> float64 [N_b]
      s_i = q[b,h] . K[b, h/G, i]  (the QK^T term of SDPA, "Sparse Attention inference
      survey" (xllm), sec. 1.1).
* ``topk(shape, q, K, page_table, lens, k)``        -> int32 [B, Hq, k_max]
      exact top-k per (b, h), ties to the lower position, ascending, -1 padded
      ("Technische Zusammenfassung: Kontextsparsitaet bei der Inferenzzeit", sec. 2,
      "Oracle Top-K").
* ``attend(shape, q, K, V, page_table, lens, idx)`` -> float64 [B, Hq, d]
      softmax(s/sqrt(d)) V over the listed rows only (SDPA restricted to the selected set;
      "Inference-time context sparsity: illusion or opportunity?", Fig. 1(a) "Sparse").
* ``dense(shape, q, K, V, page_table, lens)``       -> float64 [B, Hq, d]
      the same over all N_b rows (Fig. 1(a) "Dense").

Parity status: every function above is pinned by tests/test_oracle.py (closed forms, brute
force, library SDPA, invariants); none is "parity unpinned".
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import subprocess
import threading

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def compile_source(src: str, out: str) -> str:
    """gcc -O2 with OpenMP: one C file to one shared library."""
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-Wall", "-Wextra",
           "-o", tmp, src, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it."""
    if not force and os.path.exists(_LIB_PATH) and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC):
        return _LIB_PATH
    return compile_source(_SRC, _LIB_PATH)


def _configure(lib):
    P = ctypes.c_void_p
    I = ctypes.c_int
    lib.oracle_scores.argtypes = [I] * 7 + [P, P, P, P, I, I, P]
    lib.oracle_topk.argtypes = [I] * 8 + [P, P, P, P, P, P]
    lib.oracle_attend.argtypes = [I] * 8 + [P, P, P, P, P, P, P]
    lib.oracle_dense.argtypes = [I] * 7 + [P, P, P, P, P, P]
    lib.oracle_quest_scores.argtypes = [I] * 7 + [P, P, P, P, I, I, P]
    lib.oracle_quest_topk.argtypes = [I] * 8 + [P, P, P, P, P, P]
    lib.oracle_attend_parts.argtypes = [I] * 8 + [P, P, P, P, P, P, P, P]
    lib.oracle_stochastic_topk.argtypes = [I] * 8 + [P, P, P, P, P, P, ctypes.c_uint64, ctypes.c_uint32, P]
    lib.oracle_splitmix64.argtypes = [ctypes.c_uint64]
    lib.oracle_splitmix64.restype = ctypes.c_uint64
    for f in (lib.oracle_scores, lib.oracle_topk, lib.oracle_attend, lib.oracle_dense, lib.oracle_quest_scores,
              lib.oracle_quest_topk, lib.oracle_attend_parts, lib.oracle_stochastic_topk):
        f.restype = ctypes.c_int
    lib.oracle_num_threads.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = _configure(ctypes.CDLL(build()))
    return _lib


@contextlib.contextmanager
def use_library(path: str):
    """Route this module's functions through another build of oracle.c (the pin tests use it to
    show that deliberately broken copies of the oracle fail them)."""
    global _lib
    prev = _load()
    with _lock:
        _lib = _configure(ctypes.CDLL(path))
    try:
        yield
    finally:
        with _lock:
            _lib = prev


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def _u16(t: torch.Tensor) -> np.ndarray:
    if t.dtype != torch.bfloat16:
        raise TypeError(f"expected a bfloat16 tensor, got {t.dtype}")
    return np.ascontiguousarray(t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def _i32(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        t = t.detach().cpu().numpy()
    return np.ascontiguousarray(np.asarray(t, dtype=np.int32))


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _dims(shape: dict):
    return (int(shape["B"]), int(shape["Hq"]), int(shape["Hkv"]), int(shape["d"]), int(shape["P"]),
            int(shape["max_pages"]))


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle {what} rejected its arguments (code {rc})")


def scores(shape: dict, q, K, page_table, lens, b: int, h: int) -> np.ndarray:
    B, Hq, Hkv, d, P, max_pages = _dims(shape)
    qa, Ka, pt, ln = _u16(q), _u16(K), _i32(page_table), _i32(lens)
    num_pages = Ka.size // (P * Hkv * d)
    out = np.zeros(max(int(ln[b]), 1), dtype=np.float64)
    _check(_load().oracle_scores(B, Hq, Hkv, d, P, max_pages, num_pages, _p(qa), _p(Ka), _p(pt), _p(ln),
                                 int(b), int(h), _p(out)), "scores")
    return out[: int(ln[b])]


def topk(shape: dict, q, K, page_table, lens, k, k_max: int | None = None) -> np.ndarray:
    B, Hq, Hkv, d, P, max_pages = _dims(shape)
    k_max = int(shape["k_max"] if k_max is None else k_max)
    qa, Ka, pt, ln, ka = _u16(q), _u16(K), _i32(page_table), _i32(lens), _i32(k)
    num_pages = Ka.size // (P * Hkv * d)
    idx = np.full((B, Hq, max(k_max, 0)), -1, dtype=np.int32)
    _check(_load().oracle_topk(B, Hq, Hkv, d, P, max_pages, num_pages, k_max, _p(qa), _p(Ka), _p(pt), _p(ln),
                               _p(ka), _p(idx)), "topk")
    return idx


def attend(shape: dict, q, K, V, page_table, lens, idx) -> np.ndarray:
    B, Hq, Hkv, d, P, max_pages = _dims(shape)
    qa, Ka, Va, pt, ln = _u16(q), _u16(K), _u16(V), _i32(page_table), _i32(lens)
    ix = _i32(idx)
    k_max = ix.shape[-1]
    num_pages = Ka.size // (P * Hkv * d)
    out = np.zeros((B, Hq, d), dtype=np.float64)
    _check(_load().oracle_attend(B, Hq, Hkv, d, P, max_pages, num_pages, k_max, _p(qa), _p(Ka), _p(Va), _p(pt),
                                 _p(ln), _p(ix), _p(out)), "attend")
    return out


def dense(shape: dict, q, K, V, page_table, lens) -> np.ndarray:
    B, Hq, Hkv, d, P, max_pages = _dims(shape)
    qa, Ka, Va, pt, ln = _u16(q), _u16(K), _u16(V), _i32(page_table), _i32(lens)
    num_pages = Ka.size // (P * Hkv * d)
    out = np.zeros((B, Hq, d), dtype=np.float64)
    _check(_load().oracle_dense(B, Hq, Hkv, d, P, max_pages, num_pages, _p(qa), _p(Ka), _p(Va), _p(pt), _p(ln),
                                _p(out)), "dense")
    return out


def quest_scores(shape: dict, q, K, page_table, lens, b: int, h: int) -> np.ndarray:
    """Quest page relevance r_j = sum_d max(q_d min_d, q_d max_d) of every page of (b, h)."""
    B, Hq, Hkv, d, P, max_pages = _dims(shape)
    qa, Ka, pt, ln = _u16(q), _u16(K), _i32(page_table), _i32(lens)
    num_pages = Ka.size // (P * Hkv * d)
    np_ = (int(ln[b]) + P - 1) // P
    out = np.zeros(max(np_, 1), dtype=np.float64)
    _check(_load().oracle_quest_scores(B, Hq, Hkv, d, P, max_pages, num_pages, _p(qa), _p(Ka), _p(pt), _p(ln),
                                       int(b), int(h), _p(out)), "quest_scores")
    return out[:np_]


def quest_topk(shape: dict, q, K, page_table, lens, k, k_max: int | None = None) -> np.ndarray:
    """Quest selection: positions of the current page plus the ceil(k_b / P) - 1 most relevant others."""
    B, Hq, Hkv, d, P, max_pages = _dims(shape)
    k_max = int(shape["k_max"] if k_max is None else k_max)
    qa, Ka, pt, ln, ka = _u16(q), _u16(K), _i32(page_table), _i32(lens), _i32(k)
    num_pages = Ka.size // (P * Hkv * d)
    idx = np.full((B, Hq, max(k_max, 0)), -1, dtype=np.int32)
    _check(_load().oracle_quest_topk(B, Hq, Hkv, d, P, max_pages, num_pages, k_max, _p(qa), _p(Ka), _p(pt),
                                     _p(ln), _p(ka), _p(idx)), "quest_topk")
    return idx


SAMPLED_FLAG = 1 << 30   # idx entry of a row drawn by the stochastic selection (position in the low 30 bits)


def splitmix64(x: int) -> int:
    """One output of the SplitMix64 generator from state x (the oracle's sampling hash)."""
    return int(_load().oracle_splitmix64(ctypes.c_uint64(x & 0xFFFFFFFFFFFFFFFF)))


def stochastic_topk(shape: dict, q, K, page_table, lens, k_det, k_samp, seed: int, step: int,
                    k_max: int | None = None) -> np.ndarray:
    """Stochastic selection: exact top-k_det plus min(k_samp, |rest|) rows drawn uniformly without
    replacement from the rest (smallest sampling keys), ascending, sampled rows flagged."""
    B, Hq, Hkv, d, P, max_pages = _dims(shape)
    k_max = int(shape["k_max"] if k_max is None else k_max)
    qa, Ka, pt, ln, kd, ks = _u16(q), _u16(K), _i32(page_table), _i32(lens), _i32(k_det), _i32(k_samp)
    num_pages = Ka.size // (P * Hkv * d)
    idx = np.full((B, Hq, max(k_max, 0)), -1, dtype=np.int32)
    _check(_load().oracle_stochastic_topk(B, Hq, Hkv, d, P, max_pages, num_pages, k_max, _p(qa), _p(Ka), _p(pt),
                                          _p(ln), _p(kd), _p(ks), ctypes.c_uint64(seed & 0xFFFFFFFFFFFFFFFF),
                                          ctypes.c_uint32(step & 0xFFFFFFFF), _p(idx)), "stochastic_topk")
    return idx


def attend_parts(shape: dict, q, K, V, page_table, lens, idx):
    """Unnormalised numerator [B, Hq, d] and denominator [B, Hq] of attend (exps relative to 0)."""
    B, Hq, Hkv, d, P, max_pages = _dims(shape)
    qa, Ka, Va, pt, ln = _u16(q), _u16(K), _u16(V), _i32(page_table), _i32(lens)
    ix = _i32(idx)
    k_max = ix.shape[-1]
    num_pages = Ka.size // (P * Hkv * d)
    num = np.zeros((B, Hq, d), dtype=np.float64)
    den = np.zeros((B, Hq), dtype=np.float64)
    _check(_load().oracle_attend_parts(B, Hq, Hkv, d, P, max_pages, num_pages, k_max, _p(qa), _p(Ka), _p(Va),
                                       _p(pt), _p(ln), _p(ix), _p(num), _p(den)), "attend_parts")
    return num, den

