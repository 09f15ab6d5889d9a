"""dsa_sparse_attn_noalloc: the attention stage for callers that cannot
allocate device memory at call time (an engine plugin handed a stream but no
allocator, a serving loop that must not call cudaMalloc). It keeps its split-k
scratch in a fixed array inside libdsa.so instead of a caller workspace.

Checked through the C ABI against dsa_sparse_attn (with a workspace) on two
calls in a row, plus the size limit. This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

from learned_sparse_attention_dsa_b200 import binding
from learned_sparse_attention_dsa_b200.inputs import Workload, make_inputs, to_device
from parity_helpers import ATOL, RTOL

pytestmark = pytest.mark.gpu

DSA_ERR_INVALID_ARG = 1
DSA_ERR_WORKSPACE = 3


def _declare(lib):
    lib.dsa_sparse_attn_noalloc.argtypes = [ctypes.c_void_p] * 4 + [ctypes.POINTER(binding.AttnShape),
                                                                     ctypes.c_int, ctypes.c_void_p,
                                                                     ctypes.c_void_p, ctypes.c_void_p]
    lib.dsa_sparse_attn_noalloc.restype = ctypes.c_int
    lib.dsa_sparse_attn_noalloc_max_scratch_bytes.argtypes = []
    lib.dsa_sparse_attn_noalloc_max_scratch_bytes.restype = ctypes.c_size_t


def _noalloc(lib, q, kc, vc, idx, sh, out, lse):
    return lib.dsa_sparse_attn_noalloc(q.data_ptr(), kc.data_ptr(), vc.data_ptr(), idx.data_ptr(),
                                       ctypes.byref(sh), binding._dt(q), out.data_ptr(),
                                       lse.data_ptr(), torch.cuda.current_stream().cuda_stream)


def _close(a, b):
    a = a.float().cpu().numpy()
    b = b.float().cpu().numpy()
    err = np.abs(a - b)
    assert err.max() <= ATOL
    assert np.linalg.norm(a - b) <= RTOL * max(np.linalg.norm(b), 1e-30)


def test_noalloc_matches_workspace_entry_point_twice(cuda, dsa_lib):
    _declare(dsa_lib)
    # decode-like: few rows, so the selected list is split across CTAs and the
    # partial results go through the scratch array
    wl = Workload("noalloc", B=3, Tq=1, L=5000, q_pos0=4999, H_I=64, d_I=128, k=2048, Hq=16, Hkv=1,
                  Dqk=128, Dv=128, seed=31)
    dev = to_device(make_inputs(wl), "cuda")
    gen = torch.Generator().manual_seed(5)
    idx = torch.stack([torch.randperm(wl.L, generator=gen)[: wl.k] for _ in range(wl.B)])
    idx = idx.to(torch.int32).reshape(wl.B, 1, wl.k).cuda()
    sh = binding.attn_shape(dev["q"], dev["k_cache"], dev["v_cache"], wl.k, wl.scale)
    need = dsa_lib.dsa_sparse_attn_workspace_bytes(ctypes.byref(sh), binding._dt(dev["q"]))
    assert 0 < need <= dsa_lib.dsa_sparse_attn_noalloc_max_scratch_bytes()

    ref, ref_lse = binding.sparse_attn(dev["q"], dev["k_cache"], dev["v_cache"], idx, wl.scale, want_lse=True)
    for call in range(2):
        out = torch.full_like(ref, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        st = _noalloc(dsa_lib, dev["q"], dev["k_cache"], dev["v_cache"], idx, sh, out, lse)
        torch.cuda.synchronize()
        assert st == 0, f"call {call}: status {st}"
        _close(out, ref)
        assert torch.allclose(lse, ref_lse, rtol=0, atol=1e-4)


def test_noalloc_rejects_problems_beyond_its_scratch(cuda, dsa_lib):
    _declare(dsa_lib)
    # Two sequences decoding with 128 heads over a latent row, 2048 positions
    # selected: the selection is split 32 ways, 2*128*32*(512*2+8) bytes of
    # partials (8.5 MB) > 4 MiB. dsa_sparse_attn runs this shape with a
    # workspace; the no-workspace entry point must refuse it.
    B, L, k, Hq, D, Dv = 2, 3000, 2048, 128, 576, 512
    q = torch.zeros((B, 1, Hq, D), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((B, L, 1, D), dtype=torch.bfloat16, device="cuda")
    vc = kc[..., :Dv]
    gen = torch.Generator().manual_seed(3)
    idx = torch.stack([torch.randperm(L, generator=gen)[:k] for _ in range(B)]).to(torch.int32)
    idx = idx.reshape(B, 1, k).cuda()
    out = torch.empty((B, 1, Hq, Dv), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, 1, Hq), dtype=torch.float32, device="cuda")
    sh = binding.attn_shape(q, kc, vc, k, D ** -0.5)
    need = dsa_lib.dsa_sparse_attn_workspace_bytes(ctypes.byref(sh), binding._dt(q))
    assert need > dsa_lib.dsa_sparse_attn_noalloc_max_scratch_bytes()
    binding.sparse_attn(q, kc, vc, idx, D ** -0.5, out=out)  # accepted with a workspace
    torch.cuda.synchronize()
    assert _noalloc(dsa_lib, q, kc, vc, idx, sh, out, lse) == DSA_ERR_WORKSPACE


def test_noalloc_checks_arguments_before_the_scratch_size(cuda, dsa_lib):
    """A malformed shape gets the argument status, not DSA_ERR_WORKSPACE (and
    no division by a zero head count on the host)."""
    _declare(dsa_lib)
    q = torch.zeros((1, 1, 16, 128), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((1, 64, 1, 128), dtype=torch.bfloat16, device="cuda")
    idx = torch.zeros((1, 1, 8), dtype=torch.int32, device="cuda")
    out = torch.empty((1, 1, 16, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((1, 1, 16), dtype=torch.float32, device="cuda")
    for field, value in (("Hkv", 0), ("B", -3), ("Tq", -1), ("k", 0)):
        sh = binding.attn_shape(q, kc, kc, 8, 128 ** -0.5)
        setattr(sh, field, value)
        assert dsa_lib.dsa_sparse_attn_workspace_bytes(ctypes.byref(sh), binding._dt(q)) == 0
        assert _noalloc(dsa_lib, q, kc, kc, idx, sh, out, lse) == DSA_ERR_INVALID_ARG, field
