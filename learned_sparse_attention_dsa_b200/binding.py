"""ctypes binding of libdsa.so: argument marshalling only.

Each function takes CUDA tensors, reads their shapes, strides and data
pointers, and calls the C entry point of the same name on the current torch
stream. No arithmetic of the method happens here. The library is loaded on
first use; a missing library raises immediately (there is no CPU fallback).
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libdsa.so")

DSA_F32 = 0
DSA_BF16 = 1
DSA_E4M3 = 2
DSA_FLAG_INCLUDE_SELF = 1
DSA_INDEXER_CAUSAL_ONLY = 1

STATUS_NAMES = {0: "DSA_OK", 1: "DSA_ERR_INVALID_ARG", 2: "DSA_ERR_UNSUPPORTED",
                3: "DSA_ERR_WORKSPACE", 4: "DSA_ERR_CUDA", 5: "DSA_ERR_TIMEOUT", 6: "DSA_ERR_BAD_INDEX"}

# Symbols declared in include/dsa.h.
EXPORTED = ("dsa_version", "dsa_kernel_launch_count", "dsa_status_string", "dsa_indexer_scores",
            "dsa_indexer_scores_ex", "dsa_topk",
            "dsa_topk_workspace_bytes", "dsa_sparse_attn", "dsa_sparse_attn_workspace_bytes",
            "dsa_sparse_attn_row_group",
            "dsa_forward", "dsa_forward_workspace_bytes", "dsa_device_error", "dsa_set_wait_limit_ns", "dsa_topk_ex",
            "dsa_diag_gather",
            "dsa_indexer_kl", "dsa_indexer_backward", "dsa_indexer_backward_workspace_bytes",
            "dsa_cp_select_candidates", "dsa_cp_merge", "dsa_cp_localize", "dsa_cp_combine")


class DSAError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)}")


class AttnShape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Tq", ctypes.c_int), ("L", ctypes.c_int), ("k", ctypes.c_int),
                ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int), ("Dqk", ctypes.c_int), ("Dv", ctypes.c_int),
                ("scale", ctypes.c_float),
                ("k_stride_b", ctypes.c_int64), ("k_stride_s", ctypes.c_int64), ("k_stride_h", ctypes.c_int64),
                ("v_stride_b", ctypes.c_int64), ("v_stride_s", ctypes.c_int64), ("v_stride_h", ctypes.c_int64)]


class ForwardArgs(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Tq", ctypes.c_int), ("L", ctypes.c_int), ("q_pos0", ctypes.c_int),
                ("k", ctypes.c_int),
                ("q_idx", ctypes.c_void_p), ("k_idx", ctypes.c_void_p), ("w", ctypes.c_void_p),
                ("H_I", ctypes.c_int), ("d_I", ctypes.c_int), ("idx_dtype", ctypes.c_int),
                ("q", ctypes.c_void_p), ("k_cache", ctypes.c_void_p), ("v_cache", ctypes.c_void_p),
                ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int), ("Dqk", ctypes.c_int), ("Dv", ctypes.c_int),
                ("scale", ctypes.c_float),
                ("k_stride_b", ctypes.c_int64), ("k_stride_s", ctypes.c_int64), ("k_stride_h", ctypes.c_int64),
                ("v_stride_b", ctypes.c_int64), ("v_stride_s", ctypes.c_int64), ("v_stride_h", ctypes.c_int64),
                ("attn_dtype", ctypes.c_int),
                ("out", ctypes.c_void_p), ("lse", ctypes.c_void_p), ("idx_out", ctypes.c_void_p),
                ("scores_out", ctypes.c_void_p), ("flags", ctypes.c_uint)]


_lib = None


def load_library(path: str = LIB_PATH):
    """Load libdsa.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"libdsa.so not found at {path}; build it with "
                          "`python -m learned_sparse_attention_dsa_b200.build`")
    lib = ctypes.CDLL(path)
    vp, ci, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.dsa_version.argtypes, lib.dsa_version.restype = [], ci
    lib.dsa_kernel_launch_count.argtypes, lib.dsa_kernel_launch_count.restype = [], ctypes.c_uint64
    lib.dsa_status_string.argtypes, lib.dsa_status_string.restype = [ci], ctypes.c_char_p
    lib.dsa_indexer_scores.argtypes = [vp, vp, vp, ci, ci, ci, ci, ci, ci, ci, vp, vp]
    lib.dsa_indexer_scores.restype = ci
    lib.dsa_indexer_scores_ex.argtypes = [vp, vp, vp, ci, ci, ci, ci, ci, ci, ci, ctypes.c_uint, vp, vp]
    lib.dsa_indexer_scores_ex.restype = ci
    lib.dsa_topk.argtypes = [vp, ci, ci, ci, ci, ci, vp, vp, sz, vp]
    lib.dsa_topk.restype = ci
    lib.dsa_topk_ex.argtypes = [vp, ci, ci, ci, ci, ci, ctypes.c_uint, vp, vp, sz, vp]
    lib.dsa_topk_ex.restype = ci
    lib.dsa_topk_workspace_bytes.argtypes = [ci, ci, ci, ci, ci]
    lib.dsa_topk_workspace_bytes.restype = sz
    lib.dsa_sparse_attn.argtypes = [vp, vp, vp, vp, ctypes.POINTER(AttnShape), ci, vp, vp, vp, sz, vp]
    lib.dsa_sparse_attn.restype = ci
    lib.dsa_sparse_attn_workspace_bytes.argtypes = [ctypes.POINTER(AttnShape), ci]
    lib.dsa_sparse_attn_workspace_bytes.restype = sz
    lib.dsa_sparse_attn_row_group.argtypes = [ctypes.POINTER(AttnShape), ci]
    lib.dsa_sparse_attn_row_group.restype = ci
    lib.dsa_forward.argtypes = [ctypes.POINTER(ForwardArgs), vp, sz, vp]
    lib.dsa_forward.restype = ci
    lib.dsa_forward_workspace_bytes.argtypes = [ctypes.POINTER(ForwardArgs)]
    lib.dsa_forward_workspace_bytes.restype = sz
    lib.dsa_device_error.argtypes, lib.dsa_device_error.restype = [vp], ci
    lib.dsa_diag_gather.argtypes = [vp, ctypes.c_int64, ci, ci, vp, ctypes.c_int64, ci, vp, vp]
    lib.dsa_diag_gather.restype = ci
    lib.dsa_set_wait_limit_ns.argtypes, lib.dsa_set_wait_limit_ns.restype = [ctypes.c_uint64], ci
    lib.dsa_indexer_kl.argtypes = [vp, vp, vp, ci, ci, ci, ci, ci, vp, vp, vp, vp]
    lib.dsa_indexer_kl.restype = ci
    lib.dsa_indexer_backward.argtypes = [vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, ci, vp, vp, vp, vp, sz, vp]
    lib.dsa_indexer_backward.restype = ci
    lib.dsa_indexer_backward_workspace_bytes.argtypes = [ci, ci, ci, ci, ci, ci, ci]
    lib.dsa_indexer_backward_workspace_bytes.restype = sz
    lib.dsa_cp_select_candidates.argtypes = [vp, vp, ci, ci, ci, ci, vp, vp, vp]
    lib.dsa_cp_select_candidates.restype = ci
    lib.dsa_cp_merge.argtypes = [vp, vp, ci, ci, ci, ci, vp, vp]
    lib.dsa_cp_merge.restype = ci
    lib.dsa_cp_localize.argtypes = [vp, ci, ci, ci, ci, vp, vp]
    lib.dsa_cp_localize.restype = ci
    lib.dsa_cp_combine.argtypes = [vp, vp, ci, ci, ci, ci, ci, vp, vp, vp]
    lib.dsa_cp_combine.restype = ci
    _lib = lib
    return lib


def kernel_launch_count() -> int:
    """Kernels libdsa has enqueued in this process so far."""
    return int(load_library().dsa_kernel_launch_count())


def device_error(stream=None) -> None:
    """Synchronise `stream` and raise DSAError if a kernel recorded an error: a
    bounded wait that gave up (DSA_ERR_TIMEOUT) or a selected position outside
    [0, L) other than -1 that an attention call skipped (DSA_ERR_BAD_INDEX)."""
    _check(load_library().dsa_device_error(_stream(stream)), "dsa_device_error")


DEFAULT_WAIT_LIMIT_NS = 2_000_000_000


def diag_gather(src: torch.Tensor, row_bytes: int, n_src_rows: int, idx: torch.Tensor, sink: torch.Tensor,
                pitch_bytes=None, tile_rows: int = 32, stream=None) -> None:
    """dsa_diag_gather: the gather of rows idx of src (row_bytes each, pitch_bytes
    apart, default row_bytes) into shared memory alone, a measurement aid."""
    _need_cuda(src, idx, sink)
    pitch = row_bytes if pitch_bytes is None else pitch_bytes
    _check(load_library().dsa_diag_gather(_p(src), pitch, row_bytes, n_src_rows, _p(idx), idx.numel(), tile_rows,
                                          _p(sink), _stream(stream)), "dsa_diag_gather")


def set_wait_limit_ns(ns: int) -> None:
    """dsa_set_wait_limit_ns: the limit of the kernels' bounded device-side
    waits on the current device (0: every such wait gives up at once)."""
    _check(load_library().dsa_set_wait_limit_ns(int(ns)), "dsa_set_wait_limit_ns")


def _check(status: int, what: str):
    if status != 0:
        raise DSAError(status, what)


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return DSA_F32
    if t.dtype == torch.bfloat16:
        return DSA_BF16
    if t.dtype == torch.float8_e4m3fn:
        return DSA_E4M3
    raise TypeError(f"unsupported dtype {t.dtype}")


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("all tensors must live on a CUDA device")


def _cache_strides(t: torch.Tensor):
    if t.dim() != 4 or t.stride(3) != 1:
        raise ValueError("caches are [B, L, H_kv, D] with unit innermost stride")
    return t.stride(0), t.stride(1), t.stride(2)


def _workspace(nbytes: int, device, ws):
    if nbytes == 0:
        return None
    if ws is not None:
        if ws.numel() * ws.element_size() < nbytes:
            raise ValueError(f"workspace too small: need {nbytes} bytes")
        return ws
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def indexer_scores(q_idx, k_idx, w, q_pos0: int = 0, scores=None, stream=None, causal_only: bool = False):
    """dsa_indexer_scores_ex: fp32 [B, Tq, L] scores, -inf above the diagonal
    (with causal_only, the entries above the diagonal are not written)."""
    lib = load_library()
    _need_cuda(q_idx, k_idx, w, scores)
    B, Tq, H, d = q_idx.shape
    L = k_idx.shape[1]
    if scores is None:
        scores = torch.empty((B, Tq, L), dtype=torch.float32, device=q_idx.device)
    flags = DSA_INDEXER_CAUSAL_ONLY if causal_only else 0
    st = lib.dsa_indexer_scores_ex(_p(q_idx), _p(k_idx), _p(w), B, Tq, L, q_pos0, H, d, _dt(q_idx),
                                   flags, _p(scores), _stream(stream))
    _check(st, "dsa_indexer_scores_ex")
    return scores


def topk(scores, k: int, q_pos0: int = 0, idx=None, ws=None, stream=None, include_self: bool = False):
    """dsa_topk_ex: int32 [B, Tq, k], ascending positions then -1 (with
    include_self, S_t always holds t)."""
    lib = load_library()
    _need_cuda(scores, idx)
    B, Tq, L = scores.shape
    if idx is None:
        idx = torch.empty((B, Tq, k), dtype=torch.int32, device=scores.device)
    nbytes = lib.dsa_topk_workspace_bytes(B, Tq, L, q_pos0, k)
    ws = _workspace(nbytes, scores.device, ws)
    flags = DSA_FLAG_INCLUDE_SELF if include_self else 0
    st = lib.dsa_topk_ex(_p(scores), B, Tq, L, q_pos0, k, flags, _p(idx), _p(ws), nbytes, _stream(stream))
    _check(st, "dsa_topk_ex")
    return idx


def indexer_kl(scores, target, q_pos0: int = 0, idx=None, loss_rows=None, loss_sum=None, grad=None,
               want_grad: bool = True, want_sum: bool = True, stream=None):
    """dsa_indexer_kl: per-row KL(p_t || softmax(I_t)) over s <= t (idx None)
    or over the selected set (idx [B, Tq, k], target aligned with it).
    Returns (loss_rows [B*Tq], loss_sum [1] or None, grad [B, Tq, L] or None)."""
    lib = load_library()
    _need_cuda(scores, target, idx, loss_rows, loss_sum, grad)
    B, Tq, L = scores.shape
    k = 0 if idx is None else idx.shape[-1]
    dev = scores.device
    if loss_rows is None:
        loss_rows = torch.empty(B * Tq, dtype=torch.float32, device=dev)
    if loss_sum is None and want_sum:
        loss_sum = torch.empty(1, dtype=torch.float32, device=dev)
    if grad is None and want_grad:
        grad = torch.empty((B, Tq, L), dtype=torch.float32, device=dev)
    st = lib.dsa_indexer_kl(_p(scores), _p(target), _p(idx), B, Tq, L, q_pos0, k, _p(loss_rows), _p(loss_sum),
                            _p(grad), _stream(stream))
    _check(st, "dsa_indexer_kl")
    return loss_rows, loss_sum, grad


def indexer_backward_workspace_bytes(q_idx, k_idx, q_pos0: int = 0) -> int:
    B, Tq, H, d = q_idx.shape
    return int(load_library().dsa_indexer_backward_workspace_bytes(B, Tq, k_idx.shape[1], q_pos0, H, d,
                                                                   _dt(q_idx)))


def indexer_backward(q_idx, k_idx, w, grad, q_pos0: int = 0, dq=None, dk=None, dw=None,
                     want=("dq", "dk", "dw"), ws=None, stream=None):
    """dsa_indexer_backward: fp32 dq [B, Tq, H, d], dk [B, L, d], dw [B, Tq, H]
    for the incoming gradient grad = d loss / d I (outputs not in `want` and
    not given are skipped and returned as None)."""
    lib = load_library()
    _need_cuda(q_idx, k_idx, w, grad, dq, dk, dw)
    B, Tq, H, d = q_idx.shape
    L = k_idx.shape[1]
    dev = q_idx.device
    if dq is None and "dq" in want:
        dq = torch.empty((B, Tq, H, d), dtype=torch.float32, device=dev)
    if dk is None and "dk" in want:
        dk = torch.empty((B, L, d), dtype=torch.float32, device=dev)
    if dw is None and "dw" in want:
        dw = torch.empty((B, Tq, H), dtype=torch.float32, device=dev)
    nbytes = indexer_backward_workspace_bytes(q_idx, k_idx, q_pos0) if dk is not None else 0
    ws = _workspace(nbytes, dev, ws)
    st = lib.dsa_indexer_backward(_p(q_idx), _p(k_idx), _p(w), _p(grad), B, Tq, L, q_pos0, H, d, _dt(q_idx),
                                  _p(dq), _p(dk), _p(dw), _p(ws), nbytes, _stream(stream))
    _check(st, "dsa_indexer_backward")
    return dq, dk, dw


def cp_select_candidates(scores, idx, key_pos0: int, cand_scores=None, cand_idx=None, stream=None):
    """dsa_cp_select_candidates: ([..., k] fp32 scores, [..., k] int32 global
    positions) of a shard's selection (scores [..., L], idx [..., k])."""
    lib = load_library()
    _need_cuda(scores, idx, cand_scores, cand_idx)
    L, k = scores.shape[-1], idx.shape[-1]
    rows = idx.numel() // k
    if cand_scores is None:
        cand_scores = torch.empty(idx.shape, dtype=torch.float32, device=idx.device)
    if cand_idx is None:
        cand_idx = torch.empty(idx.shape, dtype=torch.int32, device=idx.device)
    st = lib.dsa_cp_select_candidates(_p(scores), _p(idx), rows, L, k, key_pos0, _p(cand_scores), _p(cand_idx),
                                      _stream(stream))
    _check(st, "dsa_cp_select_candidates")
    return cand_scores, cand_idx


def cp_merge(cand_scores, cand_idx, k: int, idx=None, stream=None):
    """dsa_cp_merge: candidates [P, rows..., kc] -> global selection
    [rows..., k] (ascending positions, -1 padded)."""
    lib = load_library()
    _need_cuda(cand_scores, cand_idx, idx)
    P, kc = cand_scores.shape[0], cand_scores.shape[-1]
    rows = cand_scores.numel() // (P * kc)
    if idx is None:
        idx = torch.empty(tuple(cand_scores.shape[1:-1]) + (k,), dtype=torch.int32, device=cand_scores.device)
    st = lib.dsa_cp_merge(_p(cand_scores), _p(cand_idx), P, rows, kc, k, _p(idx), _stream(stream))
    _check(st, "dsa_cp_merge")
    return idx


def cp_localize(idx, key_pos0: int, L_local: int, out=None, stream=None):
    """dsa_cp_localize: global positions -> this shard's positions (or -1)."""
    lib = load_library()
    _need_cuda(idx, out)
    k = idx.shape[-1]
    if out is None:
        out = torch.empty_like(idx)
    st = lib.dsa_cp_localize(_p(idx), idx.numel() // k, k, key_pos0, L_local, _p(out), _stream(stream))
    _check(st, "dsa_cp_localize")
    return out


def cp_combine(parts, parts_lse, out=None, lse=None, want_lse=False, stream=None):
    """dsa_cp_combine: parts [P, rows..., Hq, Dv], parts_lse [P, rows..., Hq]
    -> out [rows..., Hq, Dv] (and the merged lse)."""
    lib = load_library()
    _need_cuda(parts, parts_lse, out, lse)
    P, Hq, Dv = parts.shape[0], parts.shape[-2], parts.shape[-1]
    rows = parts.numel() // (P * Hq * Dv)
    if out is None:
        out = torch.empty(parts.shape[1:], dtype=parts.dtype, device=parts.device)
    if lse is None and want_lse:
        lse = torch.empty(parts_lse.shape[1:], dtype=torch.float32, device=parts.device)
    st = lib.dsa_cp_combine(_p(parts), _p(parts_lse), P, rows, Hq, Dv, _dt(parts), _p(out), _p(lse),
                            _stream(stream))
    _check(st, "dsa_cp_combine")
    return (out, lse) if want_lse else out


def attn_shape(q, k_cache, v_cache, k: int, scale=None) -> AttnShape:
    B, Tq, Hq, Dqk = q.shape
    ksb, kss, ksh = _cache_strides(k_cache)
    vsb, vss, vsh = _cache_strides(v_cache)
    return AttnShape(B, Tq, k_cache.shape[1], k, Hq, k_cache.shape[2], Dqk, v_cache.shape[3],
                     float(scale if scale is not None else Dqk ** -0.5),
                     ksb, kss, ksh, vsb, vss, vsh)


def sparse_attn_row_group(q, k_cache, v_cache, k: int) -> int:
    """dsa_sparse_attn_row_group: consecutive query rows whose attention
    shares the gathers of their selections (1: none share)."""
    lib = load_library()
    sh = attn_shape(q, k_cache, v_cache, k)
    return int(lib.dsa_sparse_attn_row_group(ctypes.byref(sh), _dt(q)))


def sparse_attn(q, k_cache, v_cache, idx, scale=None, out=None, lse=None, want_lse=False, ws=None,
                stream=None):
    """dsa_sparse_attn: [B, Tq, Hq, Dv] in q's dtype (and fp32 lse if asked)."""
    lib = load_library()
    _need_cuda(q, k_cache, v_cache, idx, out, lse)
    sh = attn_shape(q, k_cache, v_cache, idx.shape[-1], scale)
    if out is None:
        out = torch.empty((sh.B, sh.Tq, sh.Hq, sh.Dv), dtype=q.dtype, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((sh.B, sh.Tq, sh.Hq), dtype=torch.float32, device=q.device)
    nbytes = lib.dsa_sparse_attn_workspace_bytes(ctypes.byref(sh), _dt(q))
    ws = _workspace(nbytes, q.device, ws)
    st = lib.dsa_sparse_attn(_p(q), _p(k_cache), _p(v_cache), _p(idx), ctypes.byref(sh), _dt(q), _p(out),
                             _p(lse), _p(ws), nbytes, _stream(stream))
    _check(st, "dsa_sparse_attn")
    return (out, lse) if (want_lse or lse is not None) else out


def forward_args(q_idx, k_idx, w, q, k_cache, v_cache, k: int, q_pos0: int = 0, scale=None,
                 out=None, lse=None, idx_out=None, scores_out=None, include_self: bool = False) -> ForwardArgs:
    B, Tq, H, d = q_idx.shape
    sh = attn_shape(q, k_cache, v_cache, k, scale)
    return ForwardArgs(B, Tq, k_idx.shape[1], q_pos0, k,
                       q_idx.data_ptr(), k_idx.data_ptr(), w.data_ptr(), H, d, _dt(q_idx),
                       q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                       sh.Hq, sh.Hkv, sh.Dqk, sh.Dv, sh.scale,
                       sh.k_stride_b, sh.k_stride_s, sh.k_stride_h,
                       sh.v_stride_b, sh.v_stride_s, sh.v_stride_h, _dt(q),
                       out.data_ptr() if out is not None else None,
                       lse.data_ptr() if lse is not None else None,
                       idx_out.data_ptr() if idx_out is not None else None,
                       scores_out.data_ptr() if scores_out is not None else None,
                       DSA_FLAG_INCLUDE_SELF if include_self else 0)


def forward_workspace_bytes(args: ForwardArgs) -> int:
    return int(load_library().dsa_forward_workspace_bytes(ctypes.byref(args)))


def forward(q_idx, k_idx, w, q, k_cache, v_cache, k: int, q_pos0: int = 0, scale=None,
            out=None, lse=None, idx_out=None, scores_out=None, ws=None, stream=None,
            include_self: bool = False):
    """dsa_forward: all three stages; returns out (and fills lse/idx_out/scores_out if given)."""
    lib = load_library()
    _need_cuda(q_idx, k_idx, w, q, k_cache, v_cache, out, lse, idx_out, scores_out)
    if out is None:
        out = torch.empty((q.shape[0], q.shape[1], q.shape[2], v_cache.shape[3]), dtype=q.dtype,
                          device=q.device)
    args = forward_args(q_idx, k_idx, w, q, k_cache, v_cache, k, q_pos0, scale, out, lse, idx_out,
                        scores_out, include_self)
    nbytes = lib.dsa_forward_workspace_bytes(ctypes.byref(args))
    ws = _workspace(nbytes, q.device, ws)
    st = lib.dsa_forward(ctypes.byref(args), _p(ws), nbytes, _stream(stream))
    _check(st, "dsa_forward")
    return out
