"""Pins for the CPU oracle, independent of the oracle's own code.

Each check ties the oracle to something the pages or the mathematics fix:
the hand-traced t=10 example ("DeepSeek Sparse Attention: Learned Token
Selection from Scratch" §2.3-3.2, fixture tests/golden/hand_trace_t10.txt),
the closed-form entry counts (§7.2-7.3, fixture tests/golden/entry_counts.txt),
brute-force sorting with Python's own sort on tiny rows, numpy matrix
products, and torch's dense causal scaled_dot_product_attention for the
full-budget case ("with k >= n, DSA collapses to full attention", §7.6 note
and §9.3).
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_trace():
    rec = {"q": {}, "w": {}, "k": {}, "dot": {}, "contrib": {}, "I": {}, "rank": {}, "S": None}
    with open(os.path.join(GOLDEN, "hand_trace_t10.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            tag, *vals = line.split()
            if tag == "S":
                rec["S"] = [int(v) for v in vals]
            elif tag == "rank":
                rec["rank"][int(vals[0])] = int(vals[1])
            else:
                rec[tag][int(vals[0])] = [float(v) for v in vals[1:]]
    return rec


TRACE = _read_trace()


def _trace_inputs(w=None, extra_key=None):
    q = np.array([TRACE["q"][1], TRACE["q"][2]], dtype=np.float32)[None]      # [1, H=2, d=2]
    keys = [TRACE["k"][s] for s in range(10)]
    if extra_key is not None:
        keys.append(extra_key)
    k = np.array(keys, dtype=np.float32)[None]                                  # [1, L, 2]
    if w is None:
        w = [TRACE["w"][1][0], TRACE["w"][2][0]]
    w = np.array([w], dtype=np.float32)                                          # [1, 2]
    return q, w, k


def _scores(w=None, extra_key=None, t=None):
    q, w, k = _trace_inputs(w, extra_key)
    L = k.shape[1]
    t = L - 1 if t is None else t
    return oracle.indexer_rows(q, w, k, [0], [t])[0], t


# ---------------------------------------------------------------- indexer

def test_trace_relu_per_head():
    """w one-hot on head j gives ReLU(q_j . k_s): the §2.4 ReLU columns."""
    for head in (1, 2):
        w = [1.0, 0.0] if head == 1 else [0.0, 1.0]
        s_row, _ = _scores(w=w, t=9)
        for s in range(10):
            dot = TRACE["dot"][s][head - 1]
            assert s_row[s] == max(dot, 0.0), (head, s)


def test_trace_negative_weight_flips_sign():
    """w = -1 on one head gives -ReLU(dot), never -dot (ReLU before weighting)."""
    s_row, _ = _scores(w=[-1.0, 0.0], t=9)
    for s in range(10):
        assert s_row[s] == -max(TRACE["dot"][s][0], 0.0)


def test_trace_weighted_contributions():
    """Each head's w*ReLU column of §2.4 (0.3 is inexact in binary: 1e-6)."""
    w1, w2 = TRACE["w"][1][0], TRACE["w"][2][0]
    row1, _ = _scores(w=[w1, 0.0], t=9)
    row2, _ = _scores(w=[0.0, w2], t=9)
    for s in range(10):
        c1, c2 = TRACE["contrib"][s]
        assert abs(row1[s] - c1) <= 1e-6
        assert abs(row2[s] - c2) <= 1e-6


def test_trace_combined_scores():
    """I_{10,s} of §2.5, all ten preceding positions."""
    row, _ = _scores(t=9)
    for s in range(10):
        assert abs(row[s] - TRACE["I"][s][0]) <= 1e-6, s


def test_trace_future_positions_masked():
    """Positions s > t are not candidates: -inf in the score row."""
    q, w, k = _trace_inputs()
    row = oracle.indexer_rows(q, w, k, [0], [4])[0]
    assert np.all(np.isneginf(row[5:]))
    assert np.all(np.isfinite(row[:5]))


def test_single_head_unit_weight_is_relu_matmul():
    """H=1, w=1: I = ReLU(Q K^T) below the diagonal (numpy matmul)."""
    rng = np.random.default_rng(0)
    n, d = 37, 16
    q = rng.integers(-5, 6, size=(n, 1, d)).astype(np.float32)
    k = rng.integers(-5, 6, size=(1, n, d)).astype(np.float32)
    w = np.ones((n, 1), dtype=np.float32)
    got = oracle.indexer_rows(q, w, k, np.zeros(n), np.arange(n))
    ref = np.maximum(q[:, 0, :].astype(np.float64) @ k[0].T.astype(np.float64), 0.0)
    for t in range(n):
        assert np.array_equal(got[t, : t + 1], ref[t, : t + 1].astype(np.float32))
        assert np.all(np.isneginf(got[t, t + 1:]))


def test_indexer_linear_in_weights_and_head_order():
    """I is linear in w and invariant to relabelling heads (exact integers)."""
    rng = np.random.default_rng(1)
    n, H, d = 19, 8, 12
    q = rng.integers(-8, 9, size=(n, H, d)).astype(np.float32)
    k = rng.integers(-8, 9, size=(1, n, d)).astype(np.float32)
    wa = rng.choice([-1.0, -0.5, 0.25, 2.0], size=(n, H)).astype(np.float32)
    wb = rng.choice([-2.0, 0.5, 1.0], size=(n, H)).astype(np.float32)
    rows_b, rows_t = np.zeros(n), np.arange(n)
    Ia = oracle.indexer_rows(q, wa, k, rows_b, rows_t)
    Ib = oracle.indexer_rows(q, wb, k, rows_b, rows_t)
    Iab = oracle.indexer_rows(q, wa + wb, k, rows_b, rows_t)
    mask = np.tril(np.ones((n, n), dtype=bool))
    assert np.array_equal(Iab[mask], (Ia + Ib)[mask])
    perm = rng.permutation(H)
    Ip = oracle.indexer_rows(q[:, perm], wa[:, perm], k, rows_b, rows_t)
    assert np.array_equal(Ip[mask], Ia[mask])


def test_indexer_bf16_bits_equal_fp32_values():
    """bf16 inputs (raw bits) give the same scores as the same values in fp32."""
    rng = np.random.default_rng(2)
    n, H, d = 11, 4, 8
    q32 = rng.integers(-8, 9, size=(n, H, d)).astype(np.float32)
    k32 = rng.integers(-8, 9, size=(1, n, d)).astype(np.float32)
    w = rng.choice([0.125, -0.5, 1.0], size=(n, H)).astype(np.float32)
    q16 = torch.from_numpy(q32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    k16 = torch.from_numpy(k32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    a = oracle.indexer_rows(q32, w, k32, np.zeros(n), np.arange(n))
    b = oracle.indexer_rows(q16, w, k16, np.zeros(n), np.arange(n))
    assert np.array_equal(a, b)


# ---------------------------------------------------------------- top-k

def test_trace_selection_and_rank():
    """S_10 = {3, 8, 9} (§3.2); the ranks 3 > 9 > 8 follow the scores."""
    row, t = _scores(t=9)
    idx = oracle.topk_rows(row[None], [t], 3)[0]
    assert sorted(idx.tolist()) == TRACE["S"]
    by_rank = sorted(range(10), key=lambda s: -row[s])[:3]
    assert by_rank == [TRACE["rank"][r] for r in (1, 2, 3)]


def test_trace_with_own_key_candidate():
    """Query t=10 as its own candidate (k_10 = [-1,-1]): I_10 = 0, S stays {3,8,9}."""
    row, t = _scores(extra_key=[-1.0, -1.0])
    assert t == 10 and row[10] == 0.0
    idx = oracle.topk_rows(row[None], [t], 3)[0]
    assert sorted(idx.tolist()) == TRACE["S"]


@pytest.mark.parametrize("k,expected", [(2, [3, 8]), (3, [3, 8, 9]), (4, [3, 5, 8, 9]),
                                        (5, [0, 3, 5, 8, 9])])
def test_trace_ties_go_to_lower_position(k, expected):
    """w_2 = 0.25 makes exact ties I_8 = I_9 = 2.0 and I_0 = I_1 = 1.0."""
    row, t = _scores(w=[0.5, 0.25], t=9)
    assert row[8] == row[9] == 2.0 and row[0] == row[1] == 1.0
    idx = oracle.topk_rows(row[None], [t], k)[0]
    assert idx.tolist() == expected


def _brute_topk(row, t, k):
    order = sorted(range(t + 1), key=lambda s: (-float(row[s]), s))
    sel = sorted(order[:k])
    return sel + [-1] * (k - len(sel))


@pytest.mark.parametrize("kind", ["int", "equal", "normal", "neg", "mixed"])
def test_topk_brute_force_sort(kind):
    from learned_sparse_attention_dsa_b200.inputs import random_score_rows
    gen = torch.Generator().manual_seed(7)
    L = 41
    rows = random_score_rows(gen, 60, L, kind).numpy()
    rng = np.random.default_rng(3)
    row_t = rng.integers(0, L, size=60).astype(np.int32)
    row_t[:3] = [0, 1, L - 1]
    for k in (1, 2, 5, 17, 40, 64):
        got = oracle.topk_rows(rows, row_t, k)
        for r in range(60):
            assert got[r].tolist() == _brute_topk(rows[r], int(row_t[r]), k), (kind, k, r)


def test_topk_keeps_every_candidate_when_short():
    """t+1 <= k: S_t = {0..t} (§7.6 note: DSA collapses to full attention)."""
    rng = np.random.default_rng(4)
    L, k = 30, 12
    rows = rng.normal(size=(L, L)).astype(np.float32)
    got = oracle.topk_rows(rows, np.arange(L), k)
    for t in range(k):
        assert got[t].tolist() == list(range(t + 1)) + [-1] * (k - t - 1)
    for t in range(k, L):
        assert np.all(got[t] >= 0)


def _read_counts():
    out = []
    with open(os.path.join(GOLDEN, "entry_counts.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                kind, n, k, c = line.split()
                out.append((kind, int(n), None if k == "-" else int(k), int(c)))
    return out


def test_entry_counts_closed_form():
    """Selected entries over all t: 45 at n=16, k=3; 136 with a full budget (§7.3)."""
    rng = np.random.default_rng(5)
    for kind, n, k, count in _read_counts():
        kk = n if k is None else k
        rows = rng.integers(-3, 4, size=(n, n)).astype(np.float32)
        idx = oracle.topk_rows(rows, np.arange(n), kk)
        assert int((idx >= 0).sum()) == count, (kind, n, k)
    for n, k in [(100, 7), (64, 64), (50, 80), (257, 31)]:
        rows = rng.normal(size=(n, n)).astype(np.float32)
        idx = oracle.topk_rows(rows, np.arange(n), k)
        expect = n * (n + 1) // 2 if n <= k else k * (k + 1) // 2 + (n - k) * k
        assert int((idx >= 0).sum()) == expect


# ---------------------------------------------------------------- attention

def _attn_inputs(rng, n, Hq, Hkv, Dqk, Dv):
    q = rng.normal(size=(n, Hq, Dqk)).astype(np.float32)
    k = rng.normal(size=(1, n, Hkv, Dqk)).astype(np.float32)
    v = rng.normal(size=(1, n, Hkv, Dv)).astype(np.float32)
    return q, k, v


@pytest.mark.parametrize("Hq,Hkv,Dqk,Dv", [(8, 8, 64, 64), (16, 1, 24, 16), (4, 2, 8, 12)])
def test_full_budget_equals_dense_causal_attention(Hq, Hkv, Dqk, Dv):
    """k >= t+1 for every row: sparse attention equals dense causal attention."""
    rng = np.random.default_rng(6)
    n = 23
    q, k, v = _attn_inputs(rng, n, Hq, Hkv, Dqk, Dv)
    scale = 1.0 / math.sqrt(Dqk)
    idx = oracle.topk_rows(rng.normal(size=(n, n)).astype(np.float32), np.arange(n), n)
    got = oracle.attn_rows(q, k, v, idx, np.zeros(n), scale)
    qt = torch.from_numpy(q).double().permute(1, 0, 2)[None]                     # [1, Hq, n, D]
    kt = torch.from_numpy(k[0]).double().permute(1, 0, 2).repeat_interleave(Hq // Hkv, 0)[None]
    vt = torch.from_numpy(v[0]).double().permute(1, 0, 2).repeat_interleave(Hq // Hkv, 0)[None]
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True, scale=scale)
    ref = ref[0].permute(1, 0, 2).numpy()
    assert np.max(np.abs(got - ref)) < 1e-12


def test_single_selected_row_returns_its_value():
    rng = np.random.default_rng(8)
    n, Hq, D = 9, 4, 16
    q, k, v = _attn_inputs(rng, n, Hq, Hq, D, D)
    idx = np.full((n, 5), -1, dtype=np.int32)
    sel = rng.integers(0, n, size=n)
    idx[np.arange(n), rng.integers(0, 5, size=n)] = sel
    got = oracle.attn_rows(q, k, v, idx, np.zeros(n), 0.3)
    for r in range(n):
        assert np.array_equal(got[r], v[0, sel[r]].astype(np.float64))


def test_equal_logits_give_mean_of_selected_values():
    rng = np.random.default_rng(9)
    n, Hq, Hkv, D = 12, 6, 3, 8
    q, k, v = _attn_inputs(rng, n, Hq, Hkv, D, D)
    q[:] = 0.0
    idx = np.stack([rng.choice(n, size=5, replace=False) for _ in range(n)]).astype(np.int32)
    got = oracle.attn_rows(q, k, v, idx, np.zeros(n), 1.0)
    for r in range(n):
        for h in range(Hq):
            mean = v[0, idx[r], h // (Hq // Hkv)].astype(np.float64).mean(axis=0)
            assert np.allclose(got[r, h], mean, rtol=0, atol=1e-12)


def test_attention_invariant_to_index_order_and_padding():
    rng = np.random.default_rng(10)
    n, Hq, D = 15, 4, 16
    q, k, v = _attn_inputs(rng, n, Hq, 2, D, D)
    idx = np.stack([rng.choice(n, size=6, replace=False) for _ in range(n)]).astype(np.int32)
    a = oracle.attn_rows(q, k, v, idx, np.zeros(n), 0.25)
    shuffled = np.concatenate([idx, np.full((n, 3), -1, np.int32)], axis=1)
    for r in range(n):
        rng.shuffle(shuffled[r])
    b = oracle.attn_rows(q, k, v, shuffled, np.zeros(n), 0.25)
    assert np.allclose(a, b, rtol=0, atol=1e-12)


def test_lse_matches_logsumexp_of_selected_logits():
    rng = np.random.default_rng(11)
    n, Hq, D = 10, 3, 8
    q, k, v = _attn_inputs(rng, n, Hq, Hq, D, D)
    idx = np.stack([rng.choice(n, size=4, replace=False) for _ in range(n)]).astype(np.int32)
    scale = 0.7
    _, lse = oracle.attn_rows(q, k, v, idx, np.zeros(n), scale, want_lse=True)
    for r in range(n):
        for h in range(Hq):
            z = torch.tensor([scale * float(np.dot(q[r, h].astype(np.float64),
                                                   k[0, s, h].astype(np.float64))) for s in idx[r]],
                             dtype=torch.float64)
            assert abs(lse[r, h] - torch.logsumexp(z, 0).item()) < 1e-12


def test_value_view_of_key_rows():
    """V as the first Dv columns of each K row (latent-cache layout) via strides."""
    rng = np.random.default_rng(12)
    B, n, Hq, Dqk, Dv = 2, 14, 8, 24, 16
    q = rng.normal(size=(B * n, Hq, Dqk)).astype(np.float32)
    kv = rng.normal(size=(B, n, 1, Dqk)).astype(np.float32)
    idx = np.stack([rng.choice(n, size=5, replace=False) for _ in range(B * n)]).astype(np.int32)
    row_b = np.repeat(np.arange(B), n)
    a = oracle.attn_rows(q, kv, np.ascontiguousarray(kv[..., :Dv]), idx, row_b, 0.2)
    strides = (n * Dqk, Dqk, Dqk)
    b = oracle.attn_rows(q, kv, kv, idx, row_b, 0.2, k_strides=strides, v_strides=strides,
                         Hkv=1, Dv=Dv)
    assert np.array_equal(a, b)


def test_forward_rows_subset_equals_full():
    """Evaluating a sample of rows gives those rows of the full evaluation."""
    from learned_sparse_attention_dsa_b200.inputs import WORKLOADS, make_inputs
    wl = WORKLOADS["toy16"]
    inp = make_inputs(wl)
    n = wl.Tq
    q_idx = inp["q_idx"][0].numpy()
    w = inp["w"][0].numpy()
    k_idx = inp["k_idx"].numpy()
    q = inp["q"][0].numpy()
    kc, vc = inp["k_cache"].numpy(), inp["v_cache"].numpy()
    full = oracle.forward_rows(q_idx, w, k_idx, q, kc, vc, np.zeros(n), np.arange(n), wl.k, wl.scale)
    rows = np.array([15, 3, 0, 10])
    part = oracle.forward_rows(q_idx[rows], w[rows], k_idx, q[rows], kc, vc,
                               np.zeros(len(rows)), rows, wl.k, wl.scale)
    for a, b in zip(full, part):
        assert np.array_equal(a[rows], b)
    # count invariant on the worked-example workload itself (§7.3: 45)
    assert int((full[1] >= 0).sum()) == 45


# ---------------------------------------------------------------- top-k, current token always kept

def test_trace_include_self_keeps_token_10():
    """§3.4: token 10 misses the top 3 of its own row (I_10 = 0 with
    k^I_10 = [-1, -1]); keeping the current token gives {3, 9, 10}: 10 plus
    the two best of positions 0..9 (2.9 at 3, 2.2 at 9 in §2.5)."""
    row, t = _scores(extra_key=[-1.0, -1.0])
    assert t == 10
    plain = oracle.topk_rows(row[None], [t], 3)[0].tolist()
    kept = oracle.topk_rows(row[None], [t], 3, include_self=True)[0].tolist()
    assert plain == [3, 8, 9]
    assert kept == [3, 9, 10]


def _brute_topk_self(row, t, k):
    if t + 1 <= k:
        return list(range(t + 1)) + [-1] * (k - t - 1)
    order = sorted(range(t), key=lambda s: (-float(row[s]), s))
    sel = sorted(order[: k - 1] + [t])
    return sel + [-1] * (k - len(sel))


@pytest.mark.parametrize("kind", ["int", "equal", "normal", "neg", "mixed"])
def test_topk_include_self_brute_force(kind):
    from learned_sparse_attention_dsa_b200.inputs import random_score_rows
    gen = torch.Generator().manual_seed(11)
    L = 41
    rows = random_score_rows(gen, 60, L, kind).numpy()
    rng = np.random.default_rng(5)
    row_t = rng.integers(0, L, size=60).astype(np.int32)
    row_t[:3] = [0, 1, L - 1]
    for k in (1, 2, 5, 17, 40, 64):
        got = oracle.topk_rows(rows, row_t, k, include_self=True)
        plain = oracle.topk_rows(rows, row_t, k)
        for r in range(60):
            t = int(row_t[r])
            assert got[r].tolist() == _brute_topk_self(rows[r], t, k), (kind, k, r)
            assert t in got[r].tolist()
            if t in plain[r].tolist():  # already selected: the rule changes nothing
                assert got[r].tolist() == plain[r].tolist()


# ---------------------------------------------------------------- e4m3 indexer inputs

def test_e4m3_decode_matches_torch_for_every_code():
    """The oracle's e4m3 decoding (written from the format's definition)
    against torch's float8_e4m3fn conversion, all 256 codes."""
    codes = np.arange(256, dtype=np.uint8)
    got = oracle.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert nan.sum() == 2                                  # 0x7f and 0xff
    assert got[0x7e] == 448.0 and got[0x01] == 2.0 ** -9   # largest finite, smallest subnormal


def test_e4m3_indexer_equals_fp32_on_integers():
    """Integers in [-8, 8] are exact in e4m3, and their products sum exactly:
    the e4m3 indexer equals the fp32 one on the same values."""
    rng = np.random.default_rng(12)
    n, H, d = 23, 4, 32
    qf = rng.integers(-8, 9, size=(n, H, d)).astype(np.float32)
    kf = rng.integers(-8, 9, size=(1, n, d)).astype(np.float32)
    w = (2.0 ** rng.integers(-3, 1, size=(n, H)) * rng.choice([-1, 1], size=(n, H))).astype(np.float32)
    q8 = torch.from_numpy(qf).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    k8 = torch.from_numpy(kf).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3_decode(q8).reshape(qf.shape), qf)
    got = oracle.indexer_rows(q8, w, k8, np.zeros(n), np.arange(n))
    ref = oracle.indexer_rows(qf, w, kf, np.zeros(n), np.arange(n))
    assert np.array_equal(got, ref)
