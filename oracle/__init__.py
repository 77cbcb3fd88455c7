"""fp64 CPU oracle for MLA decoding over a paged latent KV cache.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's
CPU-baseline leg are its only callers.  It shares no code with the CUDA path
and imports nothing from it.

`decode` / `decode_rows` run the plain definition in `mla_oracle.c` (softmax of
scaled dot products over the visible cached rows, value = first 512 dims of the
same row; see that file's header for the passages it follows).
`combine` states the split merge by log-sum-exp, and `scheduler` restates the
split-KV work partition rule.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mla_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "liboracle.so")
_lock = threading.Lock()
_lib = None

PAGE = 64
D_QK = 576
D_V = 512


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (OpenMP) if it is missing or stale."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-Wall", "-o", tmp, _SRC, "-lm"],
                   check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def load_library(path: str):
    """Open a compiled oracle library and declare its entry points."""
    lib = ctypes.CDLL(path)
    p = ctypes.c_void_p
    i32, i64, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_double
    lib.mla_oracle_decode.argtypes = [p, p, p, i64, p, i32, i32, i32, f64, i32, p, p, i32]
    lib.mla_oracle_decode.restype = i32
    lib.mla_oracle_decode_rows.argtypes = [p, p, p, i64, p, i32, i32, i32, f64, i32, p, i64,
                                           p, p, i32]
    lib.mla_oracle_decode_rows.restype = i32
    lib.mla_oracle_threads.argtypes = []
    lib.mla_oracle_threads.restype = i32
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = load_library(build())
    return _lib


def _bits(t) -> np.ndarray:
    """bf16 tensor -> contiguous uint16 bit patterns (exact)."""
    import torch
    assert t.dtype == torch.bfloat16
    return np.ascontiguousarray(t.detach().cpu().contiguous().view(torch.int16).numpy()).view(np.uint16)


def _i32(t) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(t.detach().cpu() if hasattr(t, "detach") else t,
                                           dtype=np.int32))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def decode(q, kcache, block_table, cache_seqlens, scale: float, causal: bool,
           nthreads: int = 0, lib=None):
    """Exact attention for every (sequence, query position, head).

    Returns (out [b, s_q, h_q, 512] float64, lse [b, h_q, s_q] float64).
    `lib` selects another compiled copy of the oracle (the mutation tests use it).
    """
    lib = lib or _load()
    b, s_q, h_q, d = q.shape
    assert d == D_QK and kcache.shape[1:] == (PAGE, D_QK)
    qb, kb = _bits(q), _bits(kcache)
    bt, sl = _i32(block_table), _i32(cache_seqlens)
    out = np.zeros((b, s_q, h_q, D_V), dtype=np.float64)
    lse = np.zeros((b, h_q, s_q), dtype=np.float64)
    rc = lib.mla_oracle_decode(_ptr(qb), _ptr(kb), _ptr(bt), bt.shape[1], _ptr(sl), b, s_q, h_q,
                               float(scale), int(bool(causal)), _ptr(out), _ptr(lse), nthreads)
    if rc != 0:
        raise RuntimeError(f"oracle failed ({rc})")
    return out, lse


def decode_rows(q, kcache, block_table, cache_seqlens, scale: float, causal: bool, rows,
                nthreads: int = 0):
    """Selected rows.  `rows`: iterable of (i, j, h) or (i, j, h, t_begin, t_end).

    A row with a token range attends only over its visible tokens inside
    [t_begin, t_end), normalised over that range.  Returns (out [n, 512], lse [n]).
    """
    lib = _load()
    b, s_q, h_q, _ = q.shape
    lens = _i32(cache_seqlens)
    sel = []
    for r in rows:
        r = tuple(int(v) for v in r)
        if len(r) == 3:
            r = r + (0, int(lens[r[0]]))
        sel.append(r)
    sel = np.ascontiguousarray(np.asarray(sel, dtype=np.int32).reshape(-1, 5))
    qb, kb = _bits(q), _bits(kcache)
    bt = _i32(block_table)
    out = np.zeros((sel.shape[0], D_V), dtype=np.float64)
    lse = np.zeros((sel.shape[0],), dtype=np.float64)
    rc = lib.mla_oracle_decode_rows(_ptr(qb), _ptr(kb), _ptr(bt), bt.shape[1], _ptr(lens), b, s_q,
                                    h_q, float(scale), int(bool(causal)), _ptr(sel), sel.shape[0],
                                    _ptr(out), _ptr(lse), nthreads)
    if rc != 0:
        raise RuntimeError(f"oracle failed ({rc})")
    return out, lse


def combine(outs, lses):
    """Merge partial results of one row computed over disjoint token ranges.

    outs: [k, 512] (each normalised over its own range), lses: [k].
    lse = ln sum_s exp(lse_s);  out = sum_s exp(lse_s - lse) * out_s.
    A range with lse = -inf (no visible tokens) has weight 0; if every range
    is empty the result is out = 0, lse = -inf.
    """
    outs = np.asarray(outs, dtype=np.float64)
    lses = np.asarray(lses, dtype=np.float64)
    m = np.max(lses)
    if m == -np.inf:
        return np.zeros(outs.shape[1:]), -np.inf
    w = np.exp(lses - m)
    total = np.sum(w)
    lse = m + np.log(total)
    out = np.tensordot(w / total, outs, axes=(0, 0))
    return out, lse


def threads() -> int:
    """Threads the oracle's OpenMP regions use on this host."""
    return int(_load().mla_oracle_threads())
