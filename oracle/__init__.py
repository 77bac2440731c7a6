"""CPU oracle for the DSA decode/verify step (fp64, plain C, see dsa_oracle.c).

TEST INFRASTRUCTURE.  Only the tests, the smoke check and the benchmark's CPU
baseline may import this package.  It is independent of the CUDA path: it
neither imports nor is imported by ``sparse_attention_decode_relu_b200`` (the
shared, arithmetic-free input generator is the only common module).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dsa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (OpenMP, -O2, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        cmd = ["gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-fopenmp", "-fno-fast-math",
               "-ffp-contract=off", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_LIB)
            P = ctypes.c_void_p
            i32, i64 = ctypes.c_int32, ctypes.c_int64
            L.dsa_oracle_bf16.restype = ctypes.c_double
            L.dsa_oracle_bf16.argtypes = [ctypes.c_uint16]
            L.dsa_oracle_e4m3.restype = ctypes.c_double
            L.dsa_oracle_e4m3.argtypes = [ctypes.c_uint8]
            for f in (L.dsa_oracle_index_scores, L.dsa_oracle_index_magnitude):
                f.restype = None
                f.argtypes = [i32, i64, P, P, P, i32, i64, P, P, P]
            L.dsa_oracle_topk.restype = i32
            L.dsa_oracle_topk.argtypes = [i32, i64, P, i64, P, i32, P]
            L.dsa_oracle_sparse_attn.restype = i32
            L.dsa_oracle_sparse_attn.argtypes = [i32, i64, P, P, i64, P, i32, P, P]
            L.dsa_oracle_decode.restype = i32
            L.dsa_oracle_decode.argtypes = [i32, i64, P, P, P, P, i32, i64, P, P, i64, P, i32, P, P, P]
            L.dsa_oracle_threads.restype = i32
            L.dsa_oracle_set_threads.argtypes = [i32]
            _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def bf16(bits) -> float:
    return lib().dsa_oracle_bf16(int(bits))


def e4m3(code) -> float:
    return lib().dsa_oracle_e4m3(int(code))


def _keys(k_idx):
    k = np.ascontiguousarray(k_idx)
    if k.dtype == np.uint8:
        return k, 1
    if k.dtype == np.uint16:
        return k, 0
    raise TypeError("k_idx must be bf16 bits (uint16) or E4M3 codes (uint8)")


def index_scores(q_idx, w_idx, k_idx, k_scale, pos) -> np.ndarray:
    """fp64 indexer scores [T][L]; -inf where s > pos[t]."""
    q_idx = _c(q_idx, np.uint16)
    w = _c(w_idx, np.float32)
    k, fp8 = _keys(k_idx)
    sc = _c(k_scale, np.float32)
    pos = _c(pos, np.int32)
    T, L = q_idx.shape[0], k.shape[0]
    out = np.empty((T, L), np.float64)
    lib().dsa_oracle_index_scores(T, L, _p(q_idx), _p(w), _p(k), fp8, k.shape[1], _p(sc), _p(pos), _p(out))
    return out


def index_magnitude(q_idx, w_idx, k_idx, k_scale, pos) -> np.ndarray:
    q_idx = _c(q_idx, np.uint16)
    w = _c(w_idx, np.float32)
    k, fp8 = _keys(k_idx)
    sc = _c(k_scale, np.float32)
    pos = _c(pos, np.int32)
    T, L = q_idx.shape[0], k.shape[0]
    out = np.empty((T, L), np.float64)
    lib().dsa_oracle_index_magnitude(T, L, _p(q_idx), _p(w), _p(k), fp8, k.shape[1], _p(sc), _p(pos), _p(out))
    return out


def topk(scores, pos, k) -> np.ndarray:
    """Causal top-k of a [T][L] score array: [T][k] int32, ascending, -1 padded."""
    scores = _c(scores, np.float64)
    pos = _c(pos, np.int32)
    T, L = scores.shape
    sel = np.empty((T, k), np.int32)
    rc = lib().dsa_oracle_topk(T, L, _p(scores), L, _p(pos), k, _p(sel))
    if rc != 0:
        raise ValueError("oracle top-k rejected its input (rc=%d)" % rc)
    return sel


def sparse_attn(q, kv, sel, sink=None) -> np.ndarray:
    """fp64 attention over the selected rows: [T][64][128]."""
    q = _c(q, np.uint16)
    kv = np.ascontiguousarray(kv, dtype=np.uint16)
    sel = _c(sel, np.int32)
    sink = _c(sink, np.float32)
    T, k = sel.shape
    L = kv.shape[0]
    out = np.empty((T, 64, 128), np.float64)
    rc = lib().dsa_oracle_sparse_attn(T, L, _p(q), _p(kv), kv.reshape(L, -1).shape[1], _p(sel), k,
                                      _p(sink), _p(out))
    if rc != 0:
        raise ValueError("oracle attention rejected a selected index")
    return out


def window_select(pos, window) -> np.ndarray:
    """Sliding-window selection (NaiveAI research page, "Hybrid SWA-DSA
    Architecture": SWA layers attend over a 128-token window): query t takes the
    last min(pos[t] + 1, window) positions, ascending, padded with -1 to window."""
    pos = np.asarray(pos, np.int64)
    sel = np.full((pos.shape[0], window), -1, np.int32)
    for t, p in enumerate(pos):
        n = min(int(p) + 1, window)
        sel[t, :n] = np.arange(int(p) + 1 - n, int(p) + 1)
    return sel


def swa_decode(q, kv, pos, window, sink=None) -> np.ndarray:
    """fp64 sliding-window attention: attention over window_select(pos, window)."""
    return sparse_attn(q, kv, window_select(pos, window), sink=sink)


def decode(q, q_idx, w_idx, k_idx, k_scale, kv, pos, k, want_scores=False):
    """The whole step.  Returns (out fp64 [T][64][128], sel int32 [T][k][, scores])."""
    q = _c(q, np.uint16)
    q_idx = _c(q_idx, np.uint16)
    w = _c(w_idx, np.float32)
    kk, fp8 = _keys(k_idx)
    sc = _c(k_scale, np.float32)
    kv = np.ascontiguousarray(kv, dtype=np.uint16)
    pos = _c(pos, np.int32)
    T, L = q_idx.shape[0], kk.shape[0]
    out = np.empty((T, 64, 128), np.float64)
    sel = np.empty((T, k), np.int32)
    scores = np.empty((T, L), np.float64) if want_scores else None
    rc = lib().dsa_oracle_decode(T, L, _p(q), _p(q_idx), _p(w), _p(kk), fp8, kk.shape[1], _p(sc),
                                 _p(kv), kv.reshape(L, -1).shape[1], _p(pos), k, _p(out), _p(sel),
                                 _p(scores))
    if rc != 0:
        raise ValueError("oracle decode failed (rc=%d)" % rc)
    return (out, sel, scores) if want_scores else (out, sel)


def threads() -> int:
    return lib().dsa_oracle_threads()


def set_threads(n: int) -> None:
    lib().dsa_oracle_set_threads(int(n))
