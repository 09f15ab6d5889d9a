"""Host-side checks of the C ABI: the library loads, exports every entry point
that include/dsa.h declares, and rejects bad arguments before touching a GPU.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"\b(dsa_[a-z0-9_]+)\s*\(", text)
    return sorted(set(names))


def test_header_declares_the_entry_points():
    names = _declared_functions()
    for n in ("dsa_indexer_scores", "dsa_topk", "dsa_sparse_attn", "dsa_forward"):
        assert n in names


def test_library_exports_every_declared_symbol(dsa_lib):
    from learned_sparse_attention_dsa_b200 import binding
    for name in _declared_functions():
        assert hasattr(dsa_lib, name), name
    assert set(binding.EXPORTED) <= set(_declared_functions())


def test_version_and_status_strings(dsa_lib):
    assert dsa_lib.dsa_version() >= 100
    for code in range(7):
        assert dsa_lib.dsa_status_string(code)
    assert b"DSA_ERR_BAD_INDEX" in dsa_lib.dsa_status_string(6)
    assert b"unknown" in dsa_lib.dsa_status_string(99)


def test_null_pointers_rejected_before_any_launch(dsa_lib):
    assert dsa_lib.dsa_indexer_scores(None, None, None, 1, 1, 1, 0, 1, 1, 1, None, None) == 1
    assert dsa_lib.dsa_topk(None, 1, 1, 1, 0, 1, None, None, 0, None) == 1
    assert dsa_lib.dsa_sparse_attn(None, None, None, None, None, 1, None, None, None, 0, None) == 1
    assert dsa_lib.dsa_forward(None, None, 0, None) == 1
    assert dsa_lib.dsa_forward_workspace_bytes(None) == 0


def test_bad_sizes_rejected(dsa_lib):
    fake = ctypes.c_void_p(0x1000)  # never dereferenced: the checks fail first
    # q_pos0 + Tq > L
    assert dsa_lib.dsa_topk(fake, 1, 4, 3, 0, 2, fake, None, 0, None) == 1
    # k < 1
    assert dsa_lib.dsa_topk(fake, 1, 1, 3, 0, 0, fake, None, 0, None) == 1
    # negative q_pos0
    assert dsa_lib.dsa_indexer_scores(fake, fake, fake, 1, 1, 4, -1, 2, 2, 0, fake, None) == 1
    # unsupported dtype
    assert dsa_lib.dsa_indexer_scores(fake, fake, fake, 1, 1, 4, 0, 2, 2, 7, fake, None) == 2
    # misaligned bf16 pointer
    odd = ctypes.c_void_p(0x1001)
    assert dsa_lib.dsa_indexer_scores(odd, fake, fake, 1, 1, 4, 0, 2, 2, 1, fake, None) == 1
    # an indexer flag other than DSA_INDEXER_CAUSAL_ONLY
    assert dsa_lib.dsa_indexer_scores_ex(fake, fake, fake, 1, 1, 4, 0, 2, 2, 0, 2, fake, None) == 1
    assert dsa_lib.dsa_indexer_scores_ex(None, fake, fake, 1, 1, 4, 0, 2, 2, 0, 1, fake, None) == 1


def test_attention_shape_checks(dsa_lib):
    from learned_sparse_attention_dsa_b200.binding import AttnShape
    fake = ctypes.c_void_p(0x1000)
    sh = AttnShape(1, 1, 8, 4, 6, 4, 64, 64, 0.125, 512, 64, 64, 512, 64, 64)  # Hq % Hkv != 0
    assert dsa_lib.dsa_sparse_attn(fake, fake, fake, fake, ctypes.byref(sh), 1, fake, None, None, 0, None) == 1
    sh = AttnShape(1, 1, 8, 4, 8, 4, 64, 64, float("nan"), 512, 64, 64, 512, 64, 64)
    assert dsa_lib.dsa_sparse_attn(fake, fake, fake, fake, ctypes.byref(sh), 1, fake, None, None, 0, None) == 1
    sh = AttnShape(1, 1, 8, 4, 8, 4, 64, 64, 0.1, 512, 0, 64, 512, 64, 64)  # zero row stride
    assert dsa_lib.dsa_sparse_attn(fake, fake, fake, fake, ctypes.byref(sh), 1, fake, None, None, 0, None) == 1
    assert dsa_lib.dsa_sparse_attn_row_group(ctypes.byref(sh), 1) == 0  # invalid shape


def test_diag_gather_argument_checks(dsa_lib):
    fake = ctypes.c_void_p(0x1000)  # never dereferenced: the checks fail first
    g = dsa_lib.dsa_diag_gather
    g.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_int64,
                  ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]
    assert g(None, 256, 256, 10, fake, 4, 32, fake, None) == 1      # null source
    assert g(fake, 256, 24, 10, fake, 4, 32, fake, None) == 1       # row not a multiple of 16 bytes
    assert g(fake, 2048, 2048, 10, fake, 4, 32, fake, None) == 1    # row longer than 1024 bytes
    assert g(fake, 128, 256, 10, fake, 4, 32, fake, None) == 1      # pitch shorter than the row
    assert g(fake, 256, 256, 10, fake, 0, 32, fake, None) == 1      # no rows
    assert g(fake, 256, 256, 10, fake, 4, 12, fake, None) == 1      # tile rows not 8, 16 or 32
    assert g(ctypes.c_void_p(0x1008), 256, 256, 10, fake, 4, 32, fake, None) == 1  # source not 16-byte aligned


def test_workspace_size_of_an_invalid_attention_shape_is_zero(dsa_lib):
    """Invalid shapes are rejected before any size arithmetic (a zero KV head
    count would otherwise divide by zero on the host); the no-workspace entry
    point returns the argument status, not DSA_ERR_WORKSPACE."""
    from learned_sparse_attention_dsa_b200.binding import AttnShape
    dsa_lib.dsa_sparse_attn_workspace_bytes.restype = ctypes.c_size_t
    fake = ctypes.c_void_p(0x1000)  # never dereferenced: the checks fail first
    for fields in ((16, 1, 128, 0), (-2, 1, 128, 1), (1, -1, 128, 1), (1, 1, 0, 1)):
        B, Tq, Hq, Hkv = fields
        sh = AttnShape(B, Tq, 64, 8, Hq, Hkv, 128, 128, 0.1, 8192, 128, 128, 8192, 128, 128)
        assert dsa_lib.dsa_sparse_attn_workspace_bytes(ctypes.byref(sh), 1) == 0, fields
        assert dsa_lib.dsa_sparse_attn_noalloc(fake, fake, fake, fake, ctypes.byref(sh), 1, fake, None,
                                               None) == 1, fields


def test_binding_fails_loudly_without_library(tmp_path):
    from learned_sparse_attention_dsa_b200 import binding
    saved = binding._lib
    binding._lib = None
    try:
        with pytest.raises(ImportError):
            binding.load_library(str(tmp_path / "missing.so"))
    finally:
        binding._lib = saved


def test_unknown_flags_rejected(dsa_lib):
    fake = ctypes.c_void_p(0x1000)  # never dereferenced: the checks fail first
    dsa_lib.dsa_topk_ex.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                    ctypes.c_int, ctypes.c_uint, ctypes.c_void_p, ctypes.c_void_p,
                                    ctypes.c_size_t, ctypes.c_void_p]
    assert dsa_lib.dsa_topk_ex(fake, 1, 1, 3, 0, 2, 2, fake, None, 0, None) == 1
    assert dsa_lib.dsa_topk_ex(fake, 1, 1, 3, 0, 2, 0x80000000, fake, None, 0, None) == 1
