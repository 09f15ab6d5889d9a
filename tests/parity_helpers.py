"""Shared plumbing for the parity tests: feed the same seeded inputs to the
CUDA path (through the C ABI binding) and to the CPU oracle, row by row.

Nothing here computes any part of the method; it converts tensors to the
oracle's numpy inputs and compares results.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

# Attention tolerance: max absolute error and norm-wise relative error of the
# bf16/fp32 outputs against the fp64 oracle.
ATOL = 2e-2
RTOL = 1e-2
# log-sum-exp: fp32 logits of bf16 inputs against fp64
LSE_ATOL = 2e-3


def bits(t: torch.Tensor) -> np.ndarray:
    """A CPU tensor as the oracle's numpy input (fp32, raw bf16 bits, or e4m3 codes)."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.float32:
        return t.numpy()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float8_e4m3fn:
        return t.view(torch.uint8).numpy()
    raise TypeError(t.dtype)


def rows_of(wl, flat_rows):
    """(row_b, row_i, row_t) arrays for flat row ids b*Tq + i."""
    flat_rows = np.asarray(flat_rows, dtype=np.int64)
    row_b = flat_rows // wl.Tq
    row_i = flat_rows % wl.Tq
    return row_b.astype(np.int32), row_i.astype(np.int32), (row_i + wl.q_pos0).astype(np.int32)


def cache_strides(t: torch.Tensor):
    return t.stride(0), t.stride(1), t.stride(2)


def oracle_forward(wl, inp, flat_rows, nthreads=0, idx_override=None, want_lse=False, include_self=False):
    """Run the oracle on the given rows of a make_inputs() dict (CPU tensors).

    Returns (scores, idx, out), plus the log-sum-exp per (row, head) when
    want_lse is set."""
    row_b, row_i, row_t = rows_of(wl, flat_rows)
    q_idx = inp["q_idx"][row_b, row_i]
    w = inp["w"][row_b, row_i]
    q = inp["q"][row_b, row_i]
    scores = oracle.indexer_rows(bits(q_idx), w.numpy(), bits(inp["k_idx"]), row_b, row_t, nthreads)
    idx = oracle.topk_rows(scores, row_t, wl.k, nthreads, include_self) if idx_override is None else idx_override
    kc = inp["k_cache"]
    vc = inp["v_cache"]
    kbuf = bits(kc)
    if vc.data_ptr() == kc.data_ptr():
        vbuf = kbuf
    else:
        vbuf = bits(vc)
    # the caches are passed as flat buffers with the element strides of the
    # contiguous K array (V may be a view of it)
    ks = (kc.shape[1] * kc.shape[2] * kc.shape[3], kc.shape[2] * kc.shape[3], kc.shape[3])
    if vc.data_ptr() == kc.data_ptr():
        vs = ks
    else:
        vs = (vc.shape[1] * vc.shape[2] * vc.shape[3], vc.shape[2] * vc.shape[3], vc.shape[3])
    res = oracle.attn_rows(bits(q), kbuf, vbuf, idx, row_b, wl.scale, k_strides=ks, v_strides=vs,
                           Hkv=wl.Hkv, Dv=wl.Dv, nthreads=nthreads, want_lse=want_lse)
    if want_lse:
        return (scores, idx) + tuple(res)
    return scores, idx, res


def assert_attn_close(got: np.ndarray, ref: np.ndarray, what: str = ""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    max_abs = float(err.max()) if err.size else 0.0
    rel = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30))
    assert max_abs <= ATOL and rel <= RTOL, f"{what}: max_abs={max_abs:.3e} rel={rel:.3e}"
    return max_abs, rel
