"""ctypes front end of the plain C oracle (pa_oracle.c) -- test infrastructure only."""

from __future__ import annotations

import ctypes
import os

import numpy as np

from .build import build

_DT = {"f32": 0, "f16": 1, "bf16": 2}
_lib = None


def _load():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        p, i, d = ctypes.c_void_p, ctypes.c_int, ctypes.c_double
        _lib.oracle_decode.argtypes = [p, p, p, p, i, p, i, p, i, i, i, i, i, i, d, i]
        _lib.oracle_decode.restype = i
        _lib.oracle_decode_pairs.argtypes = [p, p, i, p, p, p, i, p, i, p, i, i, i, i, i, d, i]
        _lib.oracle_decode_pairs.restype = i
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def decode(q, key_cache, value_cache, block_tables, context_lens, scale, dtype, num_kv_heads,
           num_threads: int = 0) -> np.ndarray:
    """fp64 [B, Hq, D] decode output for every (b, h); raises on out-of-pool block ids."""
    lib = _load()
    q = np.ascontiguousarray(q)
    kc = np.ascontiguousarray(key_cache)
    vc = np.ascontiguousarray(value_cache)
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    cl = np.ascontiguousarray(context_lens, dtype=np.int32)
    B, Hq, D = q.shape
    out = np.empty((B, Hq, D), dtype=np.float64)
    rc = lib.oracle_decode(_ptr(out), _ptr(q), _ptr(kc), _ptr(vc), _DT[dtype], _ptr(bt), bt.shape[1],
                           _ptr(cl), B, Hq, num_kv_heads, D, kc.shape[2], kc.shape[0], float(scale),
                           int(num_threads or os.cpu_count() or 1))
    if rc != 0:
        raise IndexError(f"C oracle status {rc}")
    return out


def decode_pairs(pairs, q, key_cache, value_cache, block_tables, context_lens, scale, dtype,
                 num_kv_heads, num_threads: int = 0) -> np.ndarray:
    """fp64 [len(pairs), D] decode output for the given (b, h) pairs only."""
    lib = _load()
    pr = np.ascontiguousarray(np.asarray(pairs, dtype=np.int32).reshape(-1, 2))
    q = np.ascontiguousarray(q)
    kc = np.ascontiguousarray(key_cache)
    vc = np.ascontiguousarray(value_cache)
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    cl = np.ascontiguousarray(context_lens, dtype=np.int32)
    Hq, D = q.shape[1], q.shape[2]
    out = np.empty((pr.shape[0], D), dtype=np.float64)
    rc = lib.oracle_decode_pairs(_ptr(out), _ptr(pr), pr.shape[0], _ptr(q), _ptr(kc), _ptr(vc), _DT[dtype],
                                 _ptr(bt), bt.shape[1], _ptr(cl), Hq, num_kv_heads, D, kc.shape[2],
                                 kc.shape[0], float(scale), int(num_threads or os.cpu_count() or 1))
    if rc != 0:
        raise IndexError(f"C oracle status {rc}")
    return out


def prefill(q, key_cache, value_cache, block_tables, query_start, context_lens, scale, dtype, num_kv_heads,
            num_threads: int = 0) -> np.ndarray:
    """fp64 [T, Hq, D] causal prefill: row at position p attends to positions 0 .. p (a decode of p + 1 tokens)."""
    from .reference import prefill_rows

    seqs, pos = prefill_rows(np.asarray(query_start), np.asarray(context_lens))
    bt = np.ascontiguousarray(np.asarray(block_tables)[seqs], dtype=np.int32)
    return decode(q, key_cache, value_cache, bt, (pos + 1).astype(np.int32), scale, dtype, num_kv_heads,
                  num_threads=num_threads)
