"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Index sets and (for integer-valued indexer inputs) scores must match bit for
bit; attention outputs must be within max-abs 2e-2 and norm-wise relative
1e-2 of the fp64 oracle.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from learned_sparse_attention_dsa_b200 import binding
from learned_sparse_attention_dsa_b200.inputs import (WORKLOADS, Workload, make_inputs,
                                                      random_score_rows, to_device)
from parity_helpers import LSE_ATOL, assert_attn_close, bits, oracle_forward, rows_of

pytestmark = pytest.mark.gpu

MEDIUM = {
    "prefill_mqa_700": Workload("prefill_mqa_700", B=2, Tq=700, L=700, q_pos0=0, H_I=64, d_I=128,
                                k=96, Hq=16, Hkv=1, Dqk=192, Dv=128, seed=11),
    "prefill_perhead_520": Workload("prefill_perhead_520", B=1, Tq=520, L=520, q_pos0=0, H_I=64,
                                    d_I=128, k=64, Hq=8, Hkv=8, Dqk=64, Dv=64, seed=12),
    "chunked_prefill": Workload("chunked_prefill", B=1, Tq=200, L=900, q_pos0=700, H_I=64, d_I=128,
                                k=128, Hq=16, Hkv=1, Dqk=128, Dv=128, seed=13),
    "decode_5000": Workload("decode_5000", B=3, Tq=1, L=5000, q_pos0=4999, H_I=64, d_I=128,
                            k=2048, Hq=16, Hkv=1, Dqk=128, Dv=128, seed=14),
    "decode_latent_3000": Workload("decode_latent_3000", B=2, Tq=1, L=3000, q_pos0=2999, H_I=64,
                                   d_I=128, k=256, Hq=128, Hkv=1, Dqk=576, Dv=512, kv_alias=True,
                                   seed=15),
    # latent rows with t+1 < k: -1 padding, partly and fully masked tiles
    "latent_short": Workload("latent_short", B=2, Tq=1, L=150, q_pos0=149, H_I=64, d_I=128, k=256,
                             Hq=128, Hkv=1, Dqk=576, Dv=512, kv_alias=True, seed=20),
    # latent rows, many query rows (no split of S_t), k not a multiple of the tile
    "latent_chunk": Workload("latent_chunk", B=1, Tq=80, L=400, q_pos0=320, H_I=64, d_I=128, k=100,
                             Hq=128, Hkv=1, Dqk=576, Dv=512, kv_alias=True, seed=21),
    # one latent row decoding over 2048 selected positions: 32 splits merged by
    # the split-k combine kernel
    "latent_single": Workload("latent_single", B=1, Tq=1, L=3000, q_pos0=2999, H_I=64, d_I=128, k=2048,
                              Hq=128, Hkv=1, Dqk=576, Dv=512, kv_alias=True, seed=22),
    "short_context": Workload("short_context", B=2, Tq=40, L=40, q_pos0=0, H_I=64, d_I=128, k=64,
                              Hq=8, Hkv=8, Dqk=64, Dv=64, seed=16),
    "odd_heads": Workload("odd_heads", B=1, Tq=300, L=300, q_pos0=0, H_I=32, d_I=64, k=50, Hq=4,
                          Hkv=2, Dqk=64, Dv=32, seed=17),
    "tiny_f32": Workload("tiny_f32", B=2, Tq=45, L=45, q_pos0=0, H_I=3, d_I=5, k=7, Hq=6, Hkv=3,
                         Dqk=20, Dv=12, dtype="f32", idx_range=4, seed=18),
    "single_position": Workload("single_position", B=2, Tq=1, L=1, q_pos0=0, H_I=64, d_I=128, k=1,
                                Hq=16, Hkv=1, Dqk=128, Dv=128, seed=19),
    # indexer heads other than 64 on the tensor cores: 128 heads (two queries
    # per tile, half the epilogue groups idle) and 32 heads of width 128
    "heads128_prefill": Workload("heads128_prefill", B=2, Tq=260, L=260, q_pos0=0, H_I=128, d_I=128, k=40,
                                 Hq=16, Hkv=1, Dqk=128, Dv=128, seed=23),
    "heads32_prefill": Workload("heads32_prefill", B=1, Tq=333, L=333, q_pos0=0, H_I=32, d_I=128, k=40,
                                Hq=16, Hkv=1, Dqk=128, Dv=128, seed=24),
    "heads128_decode": Workload("heads128_decode", B=3, Tq=1, L=3000, q_pos0=2999, H_I=128, d_I=128, k=256,
                                Hq=16, Hkv=1, Dqk=128, Dv=128, seed=25),
    # 32 query heads over one latent row: the CUDA-core latent-row kernel
    "latent_h32": Workload("latent_h32", B=2, Tq=1, L=3000, q_pos0=2999, H_I=64, d_I=128, k=256,
                           Hq=32, Hkv=1, Dqk=576, Dv=512, kv_alias=True, seed=26),
    # one KV head per query head of width 128, a chunk of 45 rows (groups of
    # query rows sharing their gathers, the last one partial) after 255
    # positions, k not a multiple of the 16-position stage
    "perhead_d128_chunk": Workload("perhead_d128_chunk", B=2, Tq=45, L=300, q_pos0=255, H_I=64, d_I=128, k=100,
                                   Hq=4, Hkv=4, Dqk=128, Dv=128, seed=27),
    # 16 heads over one KV head of width 128 in enough groups of 8 query rows
    # for the tensor-core group kernel; k not a multiple of the 64-row tile,
    # a partial last group in each batch entry
    "mqa128_groups": Workload("mqa128_groups", B=3, Tq=397, L=600, q_pos0=203, H_I=64, d_I=128, k=300,
                              Hq=16, Hkv=1, Dqk=128, Dv=128, seed=28),
}

FULL_ROWS = {  # None: every query row
    "toy16": None,
    "decode32k": None,
    "prefill8k": [0, 1, 2046, 2047, 2048, 5000, 8191],
    "prefill32k": [0, 2047, 2048, 20000, 32767],
    "decode128k": None,
    "decode32k_fp8": None,
}

_cache = {}


def _inputs(wl):
    if wl.name not in _cache:
        _cache.clear()
        cpu = make_inputs(wl)
        _cache[wl.name] = (cpu, to_device(cpu, "cuda"))
    return _cache[wl.name]


def _gpu_forward(wl, dev):
    out = torch.empty((wl.B, wl.Tq, wl.Hq, wl.Dv), dtype=dev["q"].dtype, device="cuda")
    idx = torch.empty((wl.B, wl.Tq, wl.k), dtype=torch.int32, device="cuda")
    scores = torch.empty((wl.B, wl.Tq, wl.L), dtype=torch.float32, device="cuda")
    binding.forward(dev["q_idx"], dev["k_idx"], dev["w"], dev["q"], dev["k_cache"], dev["v_cache"],
                    wl.k, wl.q_pos0, wl.scale, out=out, idx_out=idx, scores_out=scores)
    binding.device_error()  # synchronises; raises if a kernel gave up on a bounded wait
    return scores, idx, out


def _check_forward(wl, flat_rows):
    cpu, dev = _inputs(wl)
    scores, idx, out = _gpu_forward(wl, dev)
    if flat_rows is None:
        flat_rows = list(range(wl.B * wl.Tq))
    o_scores, o_idx, o_out = oracle_forward(wl, cpu, flat_rows)
    row_b, row_i, _ = rows_of(wl, flat_rows)
    rb = torch.from_numpy(row_b.astype(np.int64))
    ri = torch.from_numpy(row_i.astype(np.int64))
    g_scores = scores.cpu()[rb, ri].numpy()
    g_idx = idx.cpu()[rb, ri].numpy()
    g_out = out.float().cpu()[rb, ri].numpy()
    # integer-valued indexer inputs with power-of-two weights: exact scores
    assert np.array_equal(g_scores, o_scores), f"{wl.name}: scores differ"
    assert np.array_equal(g_idx, o_idx), f"{wl.name}: selected positions differ"
    assert_attn_close(g_out, o_out, wl.name)


@pytest.mark.parametrize("name", sorted(MEDIUM))
def test_forward_medium(cuda, name):
    _check_forward(MEDIUM[name], None)


@pytest.mark.parametrize("name", list(FULL_ROWS))
def test_forward_full_size_sampled_rows(cuda, name):
    _check_forward(WORKLOADS[name], FULL_ROWS[name])


def test_hand_trace_on_gpu(cuda):
    """The t=10 example: 10 keys at positions 0..9, H=2, d=2, k=3 -> S = {3, 8, 9}."""
    q = torch.tensor([[[[1.0, 2.0], [2.0, -1.0]]]], device="cuda")              # [1,1,2,2]
    k = torch.tensor([[[1, 0], [0, 1], [-1, 1], [2, 1], [0, -1], [1, 1], [-1, 0], [1, -1],
                       [0, 2], [2, 0]]], dtype=torch.float32, device="cuda")     # [1,10,2]
    w = torch.tensor([[[0.5, 0.3]]], device="cuda")
    scores = binding.indexer_scores(q, k, w, q_pos0=9)
    expect = [1.1, 1.0, 0.5, 2.9, 0.3, 1.8, 0.0, 0.9, 2.0, 2.2]
    assert np.allclose(scores.cpu().numpy()[0, 0], expect, rtol=0, atol=1e-6)
    idx = binding.topk(scores, 3, q_pos0=9)
    assert idx.cpu().tolist() == [[[3, 8, 9]]]


@pytest.mark.parametrize("name", ["prefill_mqa_700", "chunked_prefill", "decode_5000", "odd_heads",
                                  "tiny_f32", "heads128_prefill", "heads32_prefill", "heads128_decode"])
def test_indexer_stage_all_rows(cuda, name):
    wl = MEDIUM[name]
    cpu, dev = _inputs(wl)
    scores = binding.indexer_scores(dev["q_idx"], dev["k_idx"], dev["w"], wl.q_pos0).cpu().numpy()
    flat = np.arange(wl.B * wl.Tq)
    row_b, row_i, row_t = rows_of(wl, flat)
    ref = oracle.indexer_rows(bits(cpu["q_idx"][row_b, row_i]), cpu["w"][row_b, row_i].numpy(),
                              bits(cpu["k_idx"]), row_b, row_t)
    assert np.array_equal(scores.reshape(-1, wl.L), ref)


@pytest.mark.parametrize("name", ["prefill_mqa_700", "chunked_prefill", "decode_5000", "odd_heads", "tiny_f32"])
@pytest.mark.parametrize("e4m3", [False, True])
def test_indexer_causal_only_leaves_the_upper_triangle(cuda, name, e4m3):
    """DSA_INDEXER_CAUSAL_ONLY: the causal entries equal the oracle bit for bit
    (tensor-core and CUDA-core kernels, bf16 and e4m3) and every entry above
    the diagonal keeps the sentinel that was in the buffer."""
    wl = MEDIUM[name]
    if e4m3:
        if wl.dtype == "f32":
            pytest.skip("the e4m3 indexer inputs replace bf16 ones")
        wl = wl.replace(idx_dtype="e4m3", name=wl.name + "_e4m3")  # its own input cache entry
    cpu, dev = _inputs(wl)
    sentinel = 7.25
    scores = torch.full((wl.B, wl.Tq, wl.L), sentinel, dtype=torch.float32, device="cuda")
    binding.indexer_scores(dev["q_idx"], dev["k_idx"], dev["w"], wl.q_pos0, scores=scores, causal_only=True)
    got = scores.cpu().numpy().reshape(-1, wl.L)
    flat = np.arange(wl.B * wl.Tq)
    row_b, row_i, row_t = rows_of(wl, flat)
    ref = oracle.indexer_rows(bits(cpu["q_idx"][row_b, row_i]), cpu["w"][row_b, row_i].numpy(),
                              bits(cpu["k_idx"]), row_b, row_t)
    causal = np.arange(wl.L)[None, :] <= row_t[:, None]
    assert np.array_equal(got[causal], ref[causal])
    assert np.all(got[~causal] == sentinel)


@pytest.mark.parametrize("kind", ["int", "equal", "normal", "neg", "mixed"])
@pytest.mark.parametrize("L,Tq,q_pos0,k", [(37, 37, 0, 5), (5000, 3, 4997, 2048), (3000, 2, 2998, 1),
                                           (12000, 3, 11997, 2048), (32768, 2, 32766, 2048),
                                           (32768, 3, 32765, 1000), (70000, 2, 69998, 2048),
                                           (140000, 1, 139999, 2048), (2100, 2100, 0, 2048),
                                           # many rows of 16K-49K scores: the shared-memory kernel
                                           (20003, 200, 19803, 2048), (49152, 150, 49002, 1000),
                                           # fewer rows than SMs: clusters of 8, 4 and 2 CTAs per row
                                           (20000, 20, 19980, 2048), (6000, 40, 5960, 2048),
                                           (9000, 80, 8920, 1000),
                                           # at least as many rows as SMs, rows longer than 49,152
                                           # scores: the cluster kernel with one CTA per row
                                           (60000, 160, 59840, 2048), (70000, 150, 69850, 1000)])
def test_topk_stage(cuda, kind, L, Tq, q_pos0, k):
    gen = torch.Generator().manual_seed(L + Tq + k)
    scores = random_score_rows(gen, Tq, L, kind)[None]            # [1, Tq, L]
    got = binding.topk(scores.cuda(), k, q_pos0=q_pos0).cpu().numpy()[0]
    row_t = q_pos0 + np.arange(Tq)
    ref = oracle.topk_rows(scores[0].numpy(), row_t, k)
    assert np.array_equal(got, ref)


def test_attention_row_groups(cuda):
    """Per-head prefill shares gathers across 16 query rows (8 heads of 64,
    L = 520) or fewer for wider rows, 16-head prefill across 8 rows when the
    groups cover the GPU; decode rows and the latent-row kernels gather per
    row."""
    def group(name, Tq=None):
        wl = MEDIUM[name] if Tq is None else MEDIUM[name].replace(Tq=Tq, q_pos0=MEDIUM[name].L - Tq,
                                                                   name=f"{name}_tq{Tq}")
        _, dev = _inputs(wl)
        return binding.sparse_attn_row_group(dev["q"], dev["k_cache"], dev["v_cache"], wl.k)
    assert group("prefill_perhead_520") == 16
    assert group("perhead_d128_chunk") >= 2
    assert group("prefill_perhead_520", Tq=1) == 1
    assert group("prefill_mqa_700") == 8
    assert group("mqa128_groups") == 8
    assert group("chunked_prefill") == 1  # too few groups of 8 rows to cover the GPU
    assert group("decode_latent_3000") == 1


@pytest.mark.parametrize("name", ["prefill_mqa_700", "decode_latent_3000", "latent_chunk",
                                  "latent_single", "latent_h32", "prefill_perhead_520", "perhead_d128_chunk",
                                  "mqa128_groups", "tiny_f32"])
def test_sparse_attn_stage_shuffled_and_padded(cuda, name):
    """Attention on its own, with the oracle's index sets shuffled and padded."""
    wl = MEDIUM[name]
    cpu, dev = _inputs(wl)
    flat = np.arange(wl.B * wl.Tq)
    _, o_idx, _ = oracle_forward(wl, cpu, flat)
    rng = np.random.default_rng(0)
    idx = o_idx.copy()
    for r in range(idx.shape[0]):
        rng.shuffle(idx[r])
    _, _, ref, ref_lse = oracle_forward(wl, cpu, flat, idx_override=idx, want_lse=True)
    idx_t = torch.from_numpy(idx).reshape(wl.B, wl.Tq, wl.k).cuda()
    out, lse = binding.sparse_attn(dev["q"], dev["k_cache"], dev["v_cache"], idx_t, wl.scale,
                                   want_lse=True)
    binding.device_error()
    assert_attn_close(out.float().cpu().numpy().reshape(-1, wl.Hq, wl.Dv), ref, name)
    got_lse = lse.cpu().numpy().reshape(-1, wl.Hq).astype(np.float64)
    assert np.all(np.isfinite(got_lse))
    assert np.max(np.abs(got_lse - ref_lse)) <= LSE_ATOL, f"{name}: lse differs"


def test_sparse_attn_all_padding_row(cuda):
    wl = MEDIUM["odd_heads"]
    _, dev = _inputs(wl)
    idx = torch.full((wl.B, wl.Tq, 4), -1, dtype=torch.int32, device="cuda")
    idx[:, 1:, 0] = 0
    out, lse = binding.sparse_attn(dev["q"], dev["k_cache"], dev["v_cache"], idx, wl.scale,
                                   want_lse=True)
    assert torch.count_nonzero(out[:, 0]) == 0
    assert torch.isneginf(lse[:, 0]).all()
    # |S| = 1: the output is the value row itself (rounded to bf16)
    v0 = dev["v_cache"][:, 0]                                                   # [B, Hkv, Dv]
    g = torch.arange(wl.Hq, device="cuda") // (wl.Hq // wl.Hkv)
    assert torch.equal(out[:, 1], v0[:, g])


@pytest.mark.parametrize("name", ["decode_5000", "decode_latent_3000", "latent_h32", "prefill_perhead_520",
                                  "odd_heads", "tiny_f32"])
def test_sparse_attn_reports_malformed_positions(cuda, name):
    """Positions that are neither -1 nor inside [0, L) are skipped like -1
    (no access outside the cache) and reported as DSA_ERR_BAD_INDEX by
    dsa_device_error, which then clears the report. Each case reaches one
    attention kernel: 16 heads per KV head, 128 and 32 heads over a latent
    row, one KV head per query head, and the CUDA-core kernel."""
    wl = MEDIUM[name]
    _, dev = _inputs(wl)
    gen = torch.Generator().manual_seed(7)
    rows = wl.B * wl.Tq
    k = min(wl.k, wl.L)
    clean = torch.stack([torch.randperm(wl.L, generator=gen)[:k] for _ in range(rows)]).to(torch.int32)
    bad = clean.clone()
    bad[:, 1] = wl.L             # one past the cache
    bad[:, k // 2] = -7          # negative, not the padding value
    bad[:, k - 1] = wl.L + 4096  # far past the cache
    clean[:, [1, k // 2, k - 1]] = -1
    clean = clean.reshape(wl.B, wl.Tq, k).cuda()
    bad = bad.reshape(wl.B, wl.Tq, k).cuda()
    binding.device_error()  # nothing pending from earlier tests
    out_clean, lse_clean = binding.sparse_attn(dev["q"], dev["k_cache"], dev["v_cache"], clean, wl.scale,
                                               want_lse=True)
    binding.device_error()
    out_bad, lse_bad = binding.sparse_attn(dev["q"], dev["k_cache"], dev["v_cache"], bad, wl.scale,
                                           want_lse=True)
    with pytest.raises(binding.DSAError) as exc:
        binding.device_error()
    assert exc.value.status == 6  # DSA_ERR_BAD_INDEX
    binding.device_error()        # cleared by the previous call
    assert torch.equal(out_bad, out_clean)
    assert torch.equal(lse_bad, lse_clean)


def test_bounded_waits_give_up_and_report_timeout(cuda):
    """With a wait limit of 0 every bounded wait of the tensor-core kernels
    gives up at its first call, before its role has issued a copy or an MMA:
    the indexer, the latent-row attention and the indexer backward return
    without their outputs and dsa_device_error reports DSA_ERR_TIMEOUT. With
    the default limit restored, the same calls pass parity again."""
    wl = MEDIUM["decode_5000"]             # tensor-core indexer (one query per tile)
    lat = MEDIUM["decode_latent_3000"]     # latent-row tensor-core attention
    bwd = MEDIUM["heads128_prefill"]       # tensor-core indexer backward
    _, dev = _inputs(wl)
    binding.device_error()
    try:
        binding.set_wait_limit_ns(0)
        binding.indexer_scores(dev["q_idx"], dev["k_idx"], dev["w"], wl.q_pos0)
        with pytest.raises(binding.DSAError) as exc:
            binding.device_error()
        assert exc.value.status == 5  # DSA_ERR_TIMEOUT
        _, ldev = _inputs(lat)
        idx = torch.arange(lat.k, dtype=torch.int32, device="cuda").expand(lat.B, lat.Tq, lat.k).contiguous()
        binding.sparse_attn(ldev["q"], ldev["k_cache"], ldev["v_cache"], idx, lat.scale)
        with pytest.raises(binding.DSAError) as exc:
            binding.device_error()
        assert exc.value.status == 5
        _, bdev = _inputs(bwd)
        grad = torch.ones((bwd.B, bwd.Tq, bwd.L), dtype=torch.float32, device="cuda")
        binding.indexer_backward(bdev["q_idx"], bdev["k_idx"], bdev["w"], grad, bwd.q_pos0,
                                 dq=torch.empty((bwd.B, bwd.Tq, bwd.H_I, bwd.d_I), device="cuda"))
        with pytest.raises(binding.DSAError) as exc:
            binding.device_error()
        assert exc.value.status == 5
    finally:
        binding.set_wait_limit_ns(binding.DEFAULT_WAIT_LIMIT_NS)
    binding.device_error()  # cleared; nothing pending
    _check_forward(wl, None)
    _check_forward(lat, None)


def test_diag_gather_runs_on_selected_rows(cuda):
    """The measurement aid gathers selected rows (skipping invalid entries)
    without error and without touching memory outside the source."""
    wl = MEDIUM["prefill_mqa_700"]
    _, dev = _inputs(wl)
    kc = dev["k_cache"]
    idx = torch.randint(-3, wl.L + 3, (5000,), dtype=torch.int32, device="cuda")  # some out of range
    sink = torch.zeros(1, dtype=torch.int32, device="cuda")
    n0 = binding.kernel_launch_count()
    binding.diag_gather(kc, wl.Dqk * 2, wl.L, idx, sink, pitch_bytes=kc.stride(1) * 2)
    binding.diag_gather(dev["v_cache"], wl.Dv * 2, wl.L, idx[:37], sink, tile_rows=8)
    torch.cuda.synchronize()
    assert binding.kernel_launch_count() - n0 == 2


def test_forward_equals_stage_calls(cuda):
    wl = MEDIUM["prefill_mqa_700"]
    _, dev = _inputs(wl)
    scores_f, idx_f, out_f = _gpu_forward(wl, dev)
    scores = binding.indexer_scores(dev["q_idx"], dev["k_idx"], dev["w"], wl.q_pos0)
    idx = binding.topk(scores, wl.k, wl.q_pos0)
    out = binding.sparse_attn(dev["q"], dev["k_cache"], dev["v_cache"], idx, wl.scale)
    assert torch.equal(scores, scores_f)
    assert torch.equal(idx, idx_f)
    assert torch.equal(out, out_f)


def test_invalid_arguments_enqueue_nothing(cuda):
    wl = MEDIUM["odd_heads"]
    _, dev = _inputs(wl)
    with pytest.raises(binding.DSAError):
        binding.indexer_scores(dev["q_idx"], dev["k_idx"], dev["w"], q_pos0=wl.L)   # q_pos0+Tq > L
    with pytest.raises(binding.DSAError):
        binding.topk(torch.zeros((1, 2, 8), device="cuda"), 0)
    torch.cuda.synchronize()


# ---------------------------------------------------------------- current token always kept

@pytest.mark.parametrize("kind", ["int", "normal", "mixed"])
@pytest.mark.parametrize("L,Tq,q_pos0,k", [(37, 37, 0, 5), (5000, 3, 4997, 2048), (3000, 2, 2998, 1),
                                           (140000, 1, 139999, 2048), (2100, 2100, 0, 2048),
                                           (20003, 200, 19803, 2048), (6000, 40, 5960, 2048),
                                           (60000, 160, 59840, 2048)])
def test_topk_stage_include_self(cuda, kind, L, Tq, q_pos0, k):
    gen = torch.Generator().manual_seed(L + Tq + k + 1)
    scores = random_score_rows(gen, Tq, L, kind)[None]
    got = binding.topk(scores.cuda(), k, q_pos0=q_pos0, include_self=True).cpu().numpy()[0]
    row_t = q_pos0 + np.arange(Tq)
    ref = oracle.topk_rows(scores[0].numpy(), row_t, k, include_self=True)
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("name", ["prefill_mqa_700", "chunked_prefill", "decode_5000"])
def test_forward_include_self(cuda, name):
    wl = MEDIUM[name]
    cpu, dev = _inputs(wl)
    out = torch.empty((wl.B, wl.Tq, wl.Hq, wl.Dv), dtype=dev["q"].dtype, device="cuda")
    idx = torch.empty((wl.B, wl.Tq, wl.k), dtype=torch.int32, device="cuda")
    binding.forward(dev["q_idx"], dev["k_idx"], dev["w"], dev["q"], dev["k_cache"], dev["v_cache"],
                    wl.k, wl.q_pos0, wl.scale, out=out, idx_out=idx, include_self=True)
    binding.device_error()
    flat = np.arange(wl.B * wl.Tq)
    _, o_idx, o_out = oracle_forward(wl, cpu, flat, include_self=True)
    assert np.array_equal(idx.cpu().numpy().reshape(-1, wl.k), o_idx)
    assert_attn_close(out.float().cpu().numpy().reshape(-1, wl.Hq, wl.Dv), o_out, name)


# ---------------------------------------------------------------- short context: no top-k

@pytest.mark.parametrize("name", ["short_context", "latent_short"])
def test_short_context_forward_without_scores(cuda, name):
    """q_pos0 + Tq <= k: the selection is every causal position; without
    scores_out the forward skips the indexer and the top-k. Same outputs as
    the path that computes the scores, and as the oracle."""
    wl = MEDIUM[name]
    assert wl.q_pos0 + wl.Tq <= wl.k
    cpu, dev = _inputs(wl)
    out = torch.empty((wl.B, wl.Tq, wl.Hq, wl.Dv), dtype=dev["q"].dtype, device="cuda")
    idx = torch.empty((wl.B, wl.Tq, wl.k), dtype=torch.int32, device="cuda")
    n0 = binding.kernel_launch_count()
    binding.forward(dev["q_idx"], dev["k_idx"], dev["w"], dev["q"], dev["k_cache"], dev["v_cache"],
                    wl.k, wl.q_pos0, wl.scale, out=out, idx_out=idx)
    launches_short = binding.kernel_launch_count() - n0
    binding.device_error()
    _, idx_full, out_full = _gpu_forward(wl, dev)          # with scores_out: the indexer runs
    assert torch.equal(idx, idx_full)
    assert torch.equal(out, out_full)
    n0 = binding.kernel_launch_count()
    _gpu_forward(wl, dev)
    assert launches_short < binding.kernel_launch_count() - n0
    flat = np.arange(wl.B * wl.Tq)
    _, o_idx, o_out = oracle_forward(wl, cpu, flat)
    assert np.array_equal(idx.cpu().numpy().reshape(-1, wl.k), o_idx)
    assert_attn_close(out.float().cpu().numpy().reshape(-1, wl.Hq, wl.Dv), o_out, name)


# ---------------------------------------------------------------- e4m3 indexer inputs

@pytest.mark.parametrize("name", ["prefill_mqa_700", "decode_5000", "odd_heads", "tiny_f32"])
def test_indexer_stage_e4m3(cuda, name):
    """The same integers in e4m3: scores bit-exact against the oracle reading
    the 8-bit codes (tensor-core kernel for d = 128, CUDA cores otherwise)."""
    wl = MEDIUM[name].replace(idx_dtype="e4m3")
    cpu = make_inputs(wl)
    q8, k8 = cpu["q_idx"].cuda(), cpu["k_idx"].cuda()
    assert q8.dtype == torch.float8_e4m3fn
    scores = binding.indexer_scores(q8, k8, cpu["w"].cuda(), wl.q_pos0).cpu().numpy()
    flat = np.arange(wl.B * wl.Tq)
    row_b, row_i, row_t = rows_of(wl, flat)
    ref = oracle.indexer_rows(bits(cpu["q_idx"][row_b, row_i]), cpu["w"][row_b, row_i].numpy(),
                              bits(cpu["k_idx"]), row_b, row_t)
    assert np.array_equal(scores.reshape(-1, wl.L), ref)


@pytest.mark.parametrize("name", ["decode_5000", "chunked_prefill"])
def test_forward_e4m3_equals_bf16(cuda, name):
    """Integer indexer inputs are exact in both formats, so the e4m3 forward
    gives the bf16 forward's scores, selections and outputs bit for bit."""
    wl = MEDIUM[name]
    cpu, dev = _inputs(wl)
    s16, i16, o16 = _gpu_forward(wl, dev)
    dev8 = dict(dev, q_idx=dev["q_idx"].to(torch.float8_e4m3fn), k_idx=dev["k_idx"].to(torch.float8_e4m3fn))
    s8, i8, o8 = _gpu_forward(wl, dev8)
    assert torch.equal(s8, s16)
    assert torch.equal(i8, i16)
    assert torch.equal(o8, o16)
