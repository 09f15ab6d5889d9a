"""Pins for the oracle of the indexer's training loss and backward pass,
independent of the oracle's own code.

Each check ties oracle/kl.py to something the pages or the mathematics fix:
the §5.3 numerical check of "DeepSeek Sparse Attention: Learned Token
Selection from Scratch" (fixture tests/golden/kl_target_t10.txt), closed
forms of the KL divergence, torch's kl_div on random rows, central
differences (of the loss, and of the C oracle's indexer scores for the
backward pass), torch autograd in fp64, and brute-force loops on tiny inputs.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import kl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_target_example():
    rec = {}
    with open(os.path.join(GOLDEN, "kl_target_t10.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            tag, *vals = line.split()
            rec[tag] = [float(v) for v in vals]
    return rec


def test_target_matches_page_example():
    """§5.3: the 8 heads' weights at s=3 sum to 0.91 and p_{10,3} = 0.11375."""
    ex = _read_target_example()
    h = int(ex["heads"][0])
    col3 = np.array(ex["alpha"][1:])
    assert col3.size == h
    n = 11  # positions 0..10 for query t = 10
    rng = np.random.default_rng(0)
    alpha = np.zeros((h, n))
    alpha[:, 3] = col3
    # the rest of each head's weight spread over the other positions, so that
    # every head sums to 1 (softmax rows)
    rest = rng.random((h, n - 1))
    rest = rest / rest.sum(axis=1, keepdims=True) * (1.0 - col3)[:, None]
    alpha[:, [s for s in range(n) if s != 3]] = rest
    assert np.allclose(alpha.sum(axis=1), 1.0)
    assert math.isclose(alpha[:, 3].sum(), ex["a"][1], abs_tol=1e-12)
    p = kl.target_from_heads(alpha)
    assert math.isclose(p[3], ex["p"][1], abs_tol=1e-12)
    assert math.isclose(p.sum(), 1.0, abs_tol=1e-12)
    # the L1 normalisation divides by h when every head sums to 1
    assert np.allclose(p, alpha.mean(axis=0), atol=1e-15)


def test_kl_zero_when_scores_are_log_target():
    """KL(p || softmax(log p + c)) = 0 and the gradient vanishes."""
    rng = np.random.default_rng(1)
    p = rng.random(37) + 0.01
    p /= p.sum()
    loss, g = kl.kl_row(np.log(p) + 3.7, p)
    assert abs(loss) < 1e-12
    assert np.abs(g).max() < 1e-12


def test_kl_equal_scores_is_log_n_minus_entropy():
    """softmax of equal scores is uniform: KL(p || u) = log n - H(p)."""
    rng = np.random.default_rng(2)
    p = rng.random(50)
    p /= p.sum()
    loss, _ = kl.kl_row(np.full(50, -2.5), p)
    entropy = -sum(x * math.log(x) for x in p)
    assert math.isclose(loss, math.log(50) - entropy, rel_tol=1e-12)


def test_kl_one_hot_target_is_cross_entropy():
    """p = e_{s*}: KL = log sum_s exp(I_s) - I_{s*} (the cross-entropy)."""
    I = np.array([0.5, -1.0, 2.0, 0.0, 3.25])
    a = np.array([0.0, 0.0, 1.0, 0.0, 0.0])
    loss, g = kl.kl_row(I, a)
    lse = math.log(sum(math.exp(x) for x in I))
    assert math.isclose(loss, lse - 2.0, rel_tol=1e-13)
    soft = np.exp(I - lse)
    assert np.allclose(g, soft - a, atol=1e-15)


def test_kl_matches_torch_kl_div():
    """torch.nn.functional.kl_div(log_softmax(I), p, 'sum') on random rows."""
    rng = np.random.default_rng(3)
    for n in (1, 2, 7, 300):
        I = rng.normal(size=n) * 4
        a = rng.random(n)
        a[rng.random(n) < 0.3] = 0.0
        if a.sum() == 0:
            a[0] = 1.0
        loss, _ = kl.kl_row(I, a)
        p = torch.tensor(a / a.sum())
        ref = torch.nn.functional.kl_div(torch.log_softmax(torch.tensor(I), 0), p, reduction="sum")
        assert math.isclose(loss, float(ref), rel_tol=1e-10, abs_tol=1e-12)


def test_kl_gradient_central_differences():
    """d loss / d I_s against central differences of the loss itself."""
    rng = np.random.default_rng(4)
    I = rng.normal(size=12)
    a = rng.random(12) * 3  # unnormalised weights: the loss normalises them
    _, g = kl.kl_row(I, a)
    h = 1e-6
    for s in range(12):
        e = np.zeros(12)
        e[s] = h
        fd = (kl.kl_row(I + e, a)[0] - kl.kl_row(I - e, a)[0]) / (2 * h)
        assert abs(fd - g[s]) < 1e-8


def test_kl_invariances_and_degenerate_rows():
    rng = np.random.default_rng(5)
    I = rng.normal(size=20)
    a = rng.random(20)
    l0, g0 = kl.kl_row(I, a)
    l1, g1 = kl.kl_row(I + 100.0, 7.5 * a)  # shift of I, scale of the weights
    assert math.isclose(l0, l1, rel_tol=1e-9)
    assert np.allclose(g0, g1, atol=1e-12)
    assert l0 >= 0.0
    assert math.isclose(g0.sum(), 0.0, abs_tol=1e-12)
    lz, gz = kl.kl_row(I, np.zeros(20))  # no target weight: no loss, no gradient
    assert lz == 0.0 and not gz.any()
    l1e, g1e = kl.kl_row(np.array([4.0]), np.array([2.0]))  # one candidate
    assert l1e == 0.0 and g1e[0] == 0.0


def test_kl_rows_dense_and_restricted():
    """Dense rows use s <= t; restricted rows use the valid idx entries with
    the target renormalised over them; a full budget equals the dense loss."""
    rng = np.random.default_rng(6)
    L = 9
    scores = rng.normal(size=(3, L))
    target = rng.random((3, L))
    row_t = np.array([0, 4, 8])
    loss, grad = kl.kl_rows(scores, target, row_t)
    for r, t in enumerate(row_t):
        ref, g = kl.kl_row(scores[r, : t + 1], target[r, : t + 1])
        assert math.isclose(loss[r], ref, rel_tol=1e-14, abs_tol=1e-15)
        assert np.array_equal(grad[r, t + 1:], np.zeros(L - t - 1))
    # a budget covering every candidate: idx = 0..t padded with -1
    k = L
    idx = np.full((3, k), -1, dtype=np.int32)
    tsel = np.zeros((3, k))
    for r, t in enumerate(row_t):
        idx[r, : t + 1] = np.arange(t + 1)
        tsel[r, : t + 1] = target[r, : t + 1]
    loss_r, grad_r = kl.kl_rows(scores, tsel, row_t, idx=idx)
    assert np.allclose(loss_r, loss, rtol=1e-14, atol=1e-15)
    assert np.allclose(grad_r, grad, atol=1e-15)
    # a real restriction to S = {1, 3}: the target renormalised over S
    idx2 = np.array([[3, 1, -1]], dtype=np.int32)
    a2 = np.array([[0.2, 0.6, 5.0]])  # the padding entry's weight is ignored
    l2, g2 = kl.kl_rows(scores[2:3], a2, [8], idx=idx2)
    p = np.array([0.6, 0.2]) / 0.8        # positions 1, 3
    I = scores[2, [1, 3]]
    q = np.exp(I) / np.exp(I).sum()
    assert math.isclose(l2[0], float(np.sum(p * np.log(p / q))), rel_tol=1e-12)
    assert np.allclose(g2[0, [1, 3]], q - p, atol=1e-15)
    assert np.count_nonzero(g2[0]) == 2


# ---------------------------------------------------------------- backward

def _indexer_loss(q, k, w, g, q_pos0):
    """F = sum_{t,s<=t} g[t,s] I[t,s] with I from the C oracle (§2.1)."""
    B, Tq = q.shape[0], q.shape[1]
    total = 0.0
    for b in range(B):
        rows_t = np.arange(Tq) + q_pos0
        I = oracle.indexer_rows(q[b], w[b], k[b:b + 1], np.zeros(Tq, np.int32), rows_t).astype(np.float64)
        for i, t in enumerate(rows_t):
            total += float(np.dot(g[b, i, : t + 1], I[i, : t + 1]))
    return total


def test_backward_central_differences_of_c_indexer():
    """dq, dk, dw against central differences of the C oracle's scores on
    continuous inputs (the scores are piecewise bilinear, so a step that
    crosses no ReLU kink gives the exact derivative up to fp32 rounding)."""
    rng = np.random.default_rng(7)
    B, Tq, L, H, d, q_pos0 = 1, 3, 5, 2, 3, 2
    q = rng.normal(size=(B, Tq, H, d)).astype(np.float32)
    k = rng.normal(size=(B, L, d)).astype(np.float32)
    w = rng.normal(size=(B, Tq, H)).astype(np.float32)
    g = rng.normal(size=(B, Tq, L))
    ref = kl.indexer_backward(q, k, w, g, q_pos0)
    h = 1e-2

    def fd(arr, pos):
        a1, a2 = arr.copy(), arr.copy()
        a1[pos] += h
        a2[pos] -= h
        return a1, a2

    for pos in [(0, 0, 0, 0), (0, 1, 1, 2), (0, 2, 0, 1), (0, 2, 1, 0)]:
        x = float(np.dot(q[pos[:3]], k[0, 0]))
        q1, q2 = fd(q, pos)
        num = (_indexer_loss(q1, k, w, g, q_pos0) - _indexer_loss(q2, k, w, g, q_pos0)) / (2 * h)
        assert abs(num - ref["dq"][pos]) < 2e-3 * (1 + abs(num)), (pos, x)
    for pos in [(0, 0, 0), (0, 3, 2), (0, 4, 1)]:
        k1, k2 = fd(k, pos)
        num = (_indexer_loss(q, k1, w, g, q_pos0) - _indexer_loss(q, k2, w, g, q_pos0)) / (2 * h)
        assert abs(num - ref["dk"][pos]) < 2e-3 * (1 + abs(num)), pos
    for pos in [(0, 0, 1), (0, 2, 0)]:
        w1, w2 = fd(w, pos)
        num = (_indexer_loss(q, k, w1, g, q_pos0) - _indexer_loss(q, k, w2, g, q_pos0)) / (2 * h)
        assert abs(num - ref["dw"][pos]) < 2e-3 * (1 + abs(num)), pos


def test_backward_matches_torch_autograd_on_integers():
    """Integer inputs (many dot products exactly 0): torch autograd in fp64,
    whose ReLU passes no gradient at 0, gives the same dq, dk, dw."""
    rng = np.random.default_rng(8)
    B, Tq, L, H, d, q_pos0 = 2, 6, 9, 3, 4, 3
    q = rng.integers(-2, 3, size=(B, Tq, H, d)).astype(np.float32)
    k = rng.integers(-2, 3, size=(B, L, d)).astype(np.float32)
    w = (2.0 ** rng.integers(-3, 1, size=(B, Tq, H)) * rng.choice([-1, 1], size=(B, Tq, H))).astype(np.float32)
    g = rng.normal(size=(B, Tq, L))
    ref = kl.indexer_backward(q, k, w, g, q_pos0)
    qt = torch.tensor(q, dtype=torch.float64, requires_grad=True)
    kt = torch.tensor(k, dtype=torch.float64, requires_grad=True)
    wt = torch.tensor(w, dtype=torch.float64, requires_grad=True)
    x = torch.einsum("bihd,bsd->bihs", qt, kt)
    I = (wt[..., None] * torch.relu(x)).sum(dim=2)                  # [B, Tq, L]
    t = torch.arange(Tq)[:, None] + q_pos0
    causal = torch.arange(L)[None, :] <= t
    F = (torch.tensor(g) * I * causal).sum()
    F.backward()
    assert (x == 0).any()
    assert np.allclose(ref["dq"], qt.grad.numpy(), atol=1e-12)
    assert np.allclose(ref["dk"], kt.grad.numpy(), atol=1e-12)
    assert np.allclose(ref["dw"], wt.grad.numpy(), atol=1e-12)


def test_backward_single_head_brute_force():
    """H = 1, w = 1: I = ReLU(q . k); brute-force loops over every pair."""
    rng = np.random.default_rng(9)
    Tq, L, d = 4, 4, 3
    q = rng.integers(-3, 4, size=(1, Tq, 1, d)).astype(np.float32)
    k = rng.integers(-3, 4, size=(1, L, d)).astype(np.float32)
    w = np.ones((1, Tq, 1), np.float32)
    g = rng.normal(size=(1, Tq, L))
    ref = kl.indexer_backward(q, k, w, g, 0)
    dq = np.zeros((Tq, d))
    dk = np.zeros((L, d))
    dw = np.zeros(Tq)
    for t in range(Tq):
        for s in range(t + 1):
            x = sum(float(q[0, t, 0, e]) * float(k[0, s, e]) for e in range(d))
            if x > 0:
                dw[t] += g[0, t, s] * x
                for e in range(d):
                    dq[t, e] += g[0, t, s] * float(k[0, s, e])
                    dk[s, e] += g[0, t, s] * float(q[0, t, 0, e])
    assert np.allclose(ref["dq"][0, :, 0], dq, atol=1e-12)
    assert np.allclose(ref["dk"][0], dk, atol=1e-12)
    assert np.allclose(ref["dw"][0, :, 0], dw, atol=1e-12)


def test_backward_bf16_bits_decode():
    """bf16 bit patterns (uint16) decode to the same values as fp32 inputs."""
    rng = np.random.default_rng(10)
    qf = rng.integers(-8, 9, size=(1, 3, 2, 4)).astype(np.float32)
    kf = rng.integers(-8, 9, size=(1, 3, 4)).astype(np.float32)
    w = np.ones((1, 3, 2), np.float32)
    g = rng.normal(size=(1, 3, 3))
    qb = torch.tensor(qf).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    kb = torch.tensor(kf).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    a = kl.indexer_backward(qf, kf, w, g, 0)
    b = kl.indexer_backward(qb, kb, w, g, 0)
    for key in ("dq", "dk", "dw"):
        assert np.array_equal(a[key], b[key])
