"""CPU oracle for the DSA forward path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
legs of ``bench.py`` may import this package. The product (the CUDA library
under ``learned_sparse_attention_dsa_b200`` and its binding) never imports it,
and it imports nothing from the product.

The arithmetic of the forward path lives in ``dsa_oracle.c`` (plain C, fp64,
one query row at a time; see that file's header for the page passages each
function follows and the readings taken where the pages are silent). This
module compiles it with gcc, and marshals numpy arrays into it. The indexer's
training loss and its backward pass are in ``kl.py`` (numpy, fp64; its header
lists its sources, readings and pins).

Inputs are numpy arrays: ``float32`` for fp32 data, ``uint16`` holding raw
bf16 bit patterns for bf16 data, or ``uint8`` holding e4m3 codes (indexer
inputs only). Every function takes the rows to evaluate as
``(row_b, row_t)`` arrays so that a full-size problem can be checked on a
sample of query rows.

Parity status per function (what pins it, independently of this code):
  indexer_rows : hand-traced t=10 example ("Learned Token Selection" §2.3-2.5), ReLU(q.k)
                 against numpy matmul for H=1, exact integer arithmetic.
  topk_rows    : the page's S_10 = {3, 8, 9} and rank order ("Learned Token Selection" §3.2),
                 Python's sort on tiny rows, the closed-form count of
                 selected entries ("Learned Token Selection" §7.2-7.3);
                 with include_self (§3.4): S_10 = {3, 9, 10} from the
                 page's trace, t always kept, the rest equal to Python's
                 sort of positions 0..t-1.
  kl.kl_rows, kl.indexer_backward_* : see kl.py (the warm-up target example
                 of "Learned Token Selection" §5.3, KL closed forms, torch's
                 kl_div and autograd, central differences).
  attn_rows    : torch's dense causal scaled_dot_product_attention when the
                 budget covers every candidate ("Learned Token Selection" §7.6 note, §9.3),
                 |S|=1 and equal-score special cases, permutation invariance.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import sys

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dsa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

F32 = 0
BF16 = 1
E4M3 = 2

_lib = None


def build(force: bool = False) -> str:
    """Compile dsa_oracle.c into liboracle.so (gcc, OpenMP, no fast-math)."""
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
               "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    i32p = ctypes.POINTER(ctypes.c_int32)
    f32p = ctypes.POINTER(ctypes.c_float)
    f64p = ctypes.POINTER(ctypes.c_double)
    vp = ctypes.c_void_p
    ci, i64 = ctypes.c_int, ctypes.c_int64
    lib.oracle_indexer_rows.argtypes = [ci, i32p, i32p, vp, f32p, vp, ci, ci, ci, ci, f32p, ci]
    lib.oracle_indexer_rows.restype = None
    lib.oracle_topk_rows.argtypes = [ci, i32p, f32p, ci, ci, i32p, ci]
    lib.oracle_topk_rows.restype = None
    lib.oracle_topk_self_rows.argtypes = [ci, i32p, f32p, ci, ci, i32p, ci]
    lib.oracle_topk_self_rows.restype = None
    lib.oracle_attn_rows.argtypes = [ci, i32p, vp, vp, vp, ci,
                                     i64, i64, i64, i64, i64, i64,
                                     i32p, ci, ci, ci, ci, ci, ctypes.c_double,
                                     f64p, f64p, ci]
    lib.oracle_attn_rows.restype = None
    lib.oracle_max_threads.argtypes = []
    lib.oracle_max_threads.restype = ci
    lib.oracle_e4m3_decode.argtypes = [ci, ctypes.POINTER(ctypes.c_uint8), ctypes.POINTER(ctypes.c_double)]
    lib.oracle_e4m3_decode.restype = None
    _lib = lib
    return lib


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.float32:
        return F32
    if a.dtype == np.uint16:
        return BF16
    if a.dtype == np.uint8:
        return E4M3
    raise TypeError(f"oracle inputs must be float32, uint16 (bf16 bits) or uint8 (e4m3 codes), got {a.dtype}")


def e4m3_decode(codes) -> np.ndarray:
    """float64 values of e4m3 codes (uint8), as the oracle reads them."""
    lib = _load()
    codes = np.ascontiguousarray(codes, dtype=np.uint8).ravel()
    out = np.empty(codes.shape, dtype=np.float64)
    lib.oracle_e4m3_decode(codes.size, _ptr(codes, ctypes.c_uint8), _ptr(out, ctypes.c_double))
    return out


def _ptr(a: np.ndarray, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _rows(row_b, row_t):
    row_b = np.ascontiguousarray(row_b, dtype=np.int32)
    row_t = np.ascontiguousarray(row_t, dtype=np.int32)
    if row_b.shape != row_t.shape or row_b.ndim != 1:
        raise ValueError("row_b and row_t must be 1-D arrays of equal length")
    return row_b, row_t


def indexer_rows(q_rows, w_rows, k_cache, row_b, row_t, nthreads: int = 0):
    """I[t, s] for each requested row ("Learned Token Selection" §2.1).

    q_rows [n, H, d], w_rows [n, H] float32, k_cache [B, L, d].
    Returns float32 [n, L] with -inf at s > t.
    """
    lib = _load()
    row_b, row_t = _rows(row_b, row_t)
    q_rows = np.ascontiguousarray(q_rows)
    k_cache = np.ascontiguousarray(k_cache)
    w_rows = np.ascontiguousarray(w_rows, dtype=np.float32)
    dt = _dtype_code(q_rows)
    if _dtype_code(k_cache) != dt:
        raise TypeError("q_rows and k_cache must share a dtype")
    n, H, d = q_rows.shape
    B, L, dk = k_cache.shape
    if dk != d or w_rows.shape != (n, H) or len(row_b) != n:
        raise ValueError("indexer_rows: inconsistent shapes")
    if n and (row_b.min() < 0 or row_b.max() >= B or row_t.min() < 0 or row_t.max() >= L):
        raise ValueError("indexer_rows: row out of range")
    out = np.empty((n, L), dtype=np.float32)
    lib.oracle_indexer_rows(n, _ptr(row_b, ctypes.c_int32), _ptr(row_t, ctypes.c_int32),
                            q_rows.ctypes.data, _ptr(w_rows, ctypes.c_float),
                            k_cache.ctypes.data, dt, L, H, d,
                            _ptr(out, ctypes.c_float), nthreads)
    return out


def topk_rows(scores, row_t, k: int, nthreads: int = 0, include_self: bool = False):
    """S_t for each row ("Learned Token Selection" §3.1): ascending positions, -1 padded.

    scores [n, L] float32; only entries 0..row_t[r] are read. With
    include_self, S_t = {t} plus the k-1 best of positions 0..t-1 (§3.4:
    the current token is always included).
    """
    lib = _load()
    scores = np.ascontiguousarray(scores, dtype=np.float32)
    row_t = np.ascontiguousarray(row_t, dtype=np.int32)
    n, L = scores.shape
    if row_t.shape != (n,) or k < 1 or (n and (row_t.min() < 0 or row_t.max() >= L)):
        raise ValueError("topk_rows: bad arguments")
    idx = np.empty((n, k), dtype=np.int32)
    fn = lib.oracle_topk_self_rows if include_self else lib.oracle_topk_rows
    fn(n, _ptr(row_t, ctypes.c_int32), _ptr(scores, ctypes.c_float), L, k, _ptr(idx, ctypes.c_int32), nthreads)
    return idx


def attn_rows(q_rows, k_cache, v_cache, idx, row_b, scale: float,
              k_strides=None, v_strides=None, Hkv: int | None = None,
              Dv: int | None = None, nthreads: int = 0, want_lse: bool = False):
    """u[t, h] for each row ("Learned Token Selection" §3.3, §10.1), fp64.

    q_rows [n, Hq, Dqk]. k_cache / v_cache are either 4-D [B, L, Hkv, D]
    contiguous arrays, or flat buffers with explicit element strides
    (b, s, g) given in k_strides / v_strides (then Hkv and Dv are required).
    idx [n, k] int32 with -1 padding.
    """
    lib = _load()
    q_rows = np.ascontiguousarray(q_rows)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    row_b = np.ascontiguousarray(row_b, dtype=np.int32)
    n, Hq, Dqk = q_rows.shape
    k = idx.shape[1]
    if k_strides is None:
        k_cache = np.ascontiguousarray(k_cache)
        _, _, Hkv_k, Dk = k_cache.shape
        if Dk != Dqk:
            raise ValueError("attn_rows: key dim mismatch")
        k_strides = (k_cache.shape[1] * Hkv_k * Dk, Hkv_k * Dk, Dk)
        Hkv = Hkv_k if Hkv is None else Hkv
    if v_strides is None:
        v_cache = np.ascontiguousarray(v_cache)
        _, _, Hkv_v, Dv_v = v_cache.shape
        v_strides = (v_cache.shape[1] * Hkv_v * Dv_v, Hkv_v * Dv_v, Dv_v)
        Dv = Dv_v if Dv is None else Dv
    if Hkv is None or Dv is None or Hq % Hkv != 0:
        raise ValueError("attn_rows: need Hkv dividing Hq and Dv")
    dt = _dtype_code(q_rows)
    if _dtype_code(k_cache) != dt or _dtype_code(v_cache) != dt:
        raise TypeError("attn_rows: q, k and v must share a dtype")
    out = np.empty((n, Hq, Dv), dtype=np.float64)
    lse = np.empty((n, Hq), dtype=np.float64) if want_lse else None
    lib.oracle_attn_rows(n, _ptr(row_b, ctypes.c_int32), q_rows.ctypes.data,
                         k_cache.ctypes.data, v_cache.ctypes.data, dt,
                         int(k_strides[0]), int(k_strides[1]), int(k_strides[2]),
                         int(v_strides[0]), int(v_strides[1]), int(v_strides[2]),
                         _ptr(idx, ctypes.c_int32), k, Hq, Hkv, Dqk, Dv, float(scale),
                         _ptr(out, ctypes.c_double),
                         _ptr(lse, ctypes.c_double) if want_lse else None, nthreads)
    return (out, lse) if want_lse else out


def forward_rows(q_idx_rows, w_rows, k_idx_cache, q_rows, k_cache, v_cache,
                 row_b, row_t, k: int, scale: float, k_strides=None, v_strides=None,
                 Hkv=None, Dv=None, nthreads: int = 0, include_self: bool = False):
    """The three stages back to back for the requested rows.

    Returns (scores [n, L] float32, idx [n, k] int32, out [n, Hq, Dv] fp64).
    """
    scores = indexer_rows(q_idx_rows, w_rows, k_idx_cache, row_b, row_t, nthreads)
    idx = topk_rows(scores, row_t, k, nthreads, include_self)
    out = attn_rows(q_rows, k_cache, v_cache, idx, row_b, scale, k_strides, v_strides,
                    Hkv, Dv, nthreads)
    return scores, idx, out


if __name__ == "__main__":  # pragma: no cover
    print(build(force="--force" in sys.argv))
