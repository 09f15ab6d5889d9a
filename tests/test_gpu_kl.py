"""GPU parity of the indexer's training loss (dsa_indexer_kl) against the
fp64 oracle (oracle/kl.py), through the C ABI.

Tolerances follow from the kernel's fp32 arithmetic. The loss of a row is
formed from the sums sum(a), sum(a I), sum(a log a) and the log-sum-exp of I,
each accumulated over at most a few thousand terms per thread plus a tree of
256, so its error stays within a few hundred ulps (u = 2^-24) of the
magnitude M = sum p|log p| + sum p|I| + |LSE| + 1: the tests allow 2e-5 * M.
A gradient entry exp(I - LSE) - p inherits the error of LSE (at most
2e-5 * M absolute) relative to softmax(I), plus a few ulps: the tests allow
1e-6 + 2e-5 * M * (q + p).
"""
import numpy as np
import pytest
import torch

from oracle import kl
from learned_sparse_attention_dsa_b200 import binding
from learned_sparse_attention_dsa_b200.inputs import (WORKLOADS, make_inputs, random_score_rows,
                                                      target_weights, to_device)

pytestmark = pytest.mark.gpu


def _magnitude(scores, target, row_t, idx=None):
    """Per row: M = sum p|log p| + sum p|I| + |LSE| + 1 over the row's set."""
    R = scores.shape[0]
    M = np.ones(R)
    for r in range(R):
        t = int(row_t[r])
        if idx is None:
            pos = np.arange(t + 1)
            a = target[r, : t + 1].astype(np.float64)
        else:
            valid = idx[r] >= 0
            pos = idx[r][valid]
            a = target[r][valid].astype(np.float64)
        if a.sum() == 0:
            continue
        p = a / a.sum()
        I = scores[r, pos].astype(np.float64)
        lse = I.max() + np.log(np.exp(I - I.max()).sum())
        on = p > 0
        M[r] += np.sum(p[on] * np.abs(np.log(p[on]))) + np.sum(p * np.abs(I)) + abs(lse)
    return M


def _check(scores, target, row_t, idx, loss, lsum, grad):
    """Compare GPU outputs (numpy) with the oracle on the same inputs."""
    s64 = scores.astype(np.float64)
    ref_loss, ref_grad = kl.kl_rows(s64, target, row_t, idx)
    M = _magnitude(scores, target, row_t, idx)
    err = np.abs(loss.astype(np.float64) - ref_loss)
    assert np.all(err <= 2e-5 * M), f"loss: worst {np.max(err / M):.3g} of M"
    if lsum is not None:
        total = float(ref_loss.sum())
        assert abs(float(lsum) - total) <= 2e-5 * float(M.sum()) + 1e-6 * abs(total)
    if grad is not None:
        ref_q = ref_grad.copy()
        # q + p for the tolerance: |grad| bounds neither, so rebuild both
        qp = np.zeros_like(ref_grad)
        for r in range(len(row_t)):
            t = int(row_t[r])
            if idx is None:
                pos = np.arange(t + 1)
                a = target[r, : t + 1].astype(np.float64)
            else:
                valid = idx[r] >= 0
                pos = idx[r][valid]
                a = target[r][valid].astype(np.float64)
            if a.sum() == 0:
                continue
            I = s64[r, pos]
            q = np.exp(I - I.max())
            qp[r, pos] = q / q.sum() + a / a.sum()
        tol = 1e-6 + 2e-5 * M[:, None] * qp
        gerr = np.abs(grad.astype(np.float64) - ref_q)
        assert np.all(gerr <= tol), f"grad: worst excess {np.max(gerr - tol):.3g}"
        # entries off the set are exactly zero
        off = qp == 0
        assert np.all(grad[off] == 0.0)


def _rows_t(B, Tq, q_pos0):
    return np.tile(np.arange(Tq) + q_pos0, B)


@pytest.mark.parametrize("B,Tq,L,q_pos0", [(1, 37, 37, 0), (2, 300, 300, 0), (1, 5, 4099, 4094),
                                           (3, 1, 2050, 2049), (1, 64, 70, 6)])
@pytest.mark.parametrize("kind", ["normal", "int"])
def test_kl_dense(cuda, B, Tq, L, q_pos0, kind):
    gen = torch.Generator().manual_seed(100 + L + Tq)
    scores = random_score_rows(gen, B * Tq, L, kind).reshape(B, Tq, L) * 3.0
    target = target_weights(gen, (B, Tq, L))
    loss, lsum, grad = binding.indexer_kl(scores.cuda(), target.cuda(), q_pos0)
    torch.cuda.synchronize()
    _check(scores.reshape(B * Tq, L).numpy(), target.reshape(B * Tq, L).numpy(), _rows_t(B, Tq, q_pos0),
           None, loss.cpu().numpy(), lsum.item(), grad.cpu().reshape(B * Tq, L).numpy())


@pytest.mark.parametrize("B,Tq,L,q_pos0,k", [(1, 300, 300, 0, 64), (2, 3, 5000, 4997, 2048),
                                             (1, 40, 40, 0, 64), (1, 130, 1030, 900, 1000)])
def test_kl_restricted_to_topk(cuda, B, Tq, L, q_pos0, k):
    """The sparse-stage loss over S_t from dsa_topk (with -1 padding when
    t + 1 < k), target aligned with idx."""
    gen = torch.Generator().manual_seed(200 + L + k)
    scores = random_score_rows(gen, B * Tq, L, "normal").reshape(B, Tq, L) * 3.0
    sd = scores.cuda()
    idx = binding.topk(sd, k, q_pos0)
    target = target_weights(gen, (B, Tq, k))
    loss, lsum, grad = binding.indexer_kl(sd, target.cuda(), q_pos0, idx=idx)
    torch.cuda.synchronize()
    _check(scores.reshape(B * Tq, L).numpy(), target.reshape(B * Tq, k).numpy(), _rows_t(B, Tq, q_pos0),
           idx.cpu().reshape(B * Tq, k).numpy(), loss.cpu().numpy(), lsum.item(),
           grad.cpu().reshape(B * Tq, L).numpy())


def test_kl_degenerate_rows(cuda):
    """All-zero target rows (loss 0, zero gradient), a single candidate
    (loss 0), a one-hot target, shuffled idx with padding, grad not asked."""
    L = 16
    scores = torch.randn(4, 1, L, generator=torch.Generator().manual_seed(7)) * 2
    target = torch.rand(4, 1, L, generator=torch.Generator().manual_seed(8))
    target[0] = 0.0
    target[2] = 0.0
    target[2, 0, 5] = 3.0
    loss, lsum, grad = binding.indexer_kl(scores.cuda(), target.cuda(), L - 1)
    torch.cuda.synchronize()
    _check(scores.reshape(4, L).numpy(), target.reshape(4, L).numpy(), np.full(4, L - 1), None,
           loss.cpu().numpy(), lsum.item(), grad.cpu().reshape(4, L).numpy())
    assert loss[0].item() == 0.0 and not grad[0].any()
    # a single candidate: position 0 of a one-row prefill
    l1, _, g1 = binding.indexer_kl(scores[:1, :, :1].contiguous().cuda(), target[1:2, :, :1].contiguous().cuda(), 0)
    # exactly 0 up to the hardware exp/log approximations (relative 2^-21)
    assert abs(l1.item()) <= 1e-6 and abs(g1.item()) <= 1e-6
    # shuffled selection with padding in the middle; no gradient requested
    idx = torch.tensor([[[9, -1, 2, 15, 0, -1]]], dtype=torch.int32).repeat(4, 1, 1)
    tsel = torch.rand(4, 1, 6, generator=torch.Generator().manual_seed(9))
    l2, s2, g2 = binding.indexer_kl(scores.cuda(), tsel.cuda(), L - 1, idx=idx.cuda(), want_grad=False)
    torch.cuda.synchronize()
    assert g2 is None
    _check(scores.reshape(4, L).numpy(), tsel.reshape(4, 6).numpy(), np.full(4, L - 1),
           idx.reshape(4, 6).numpy(), l2.cpu().numpy(), s2.item(), None)


def test_kl_on_indexer_scores_prefill8k_sampled(cuda):
    """The dense warm-up loss on the indexer's own prefill8k scores (integer
    inputs: scores in the hundreds of thousands, near one-hot softmax rows),
    checked on sampled rows."""
    wl = WORKLOADS["prefill8k"]
    dev = to_device(make_inputs(wl), "cuda")
    scores = binding.indexer_scores(dev["q_idx"], dev["k_idx"], dev["w"], wl.q_pos0)
    target = target_weights(torch.Generator().manual_seed(31), (1, wl.Tq, wl.L)).cuda()
    loss, lsum, grad = binding.indexer_kl(scores, target, wl.q_pos0)
    torch.cuda.synchronize()
    rows = np.array([0, 1, 2047, 4096, 8191])
    s = scores[0, rows].cpu().numpy()
    a = target[0, rows].cpu().numpy()
    _check(s, a, rows, None, loss.cpu().numpy()[rows], None, grad[0, rows].cpu().numpy())
    assert np.isfinite(lsum.item())


def test_kl_invalid_arguments(cuda):
    s = torch.zeros(1, 4, 4, device="cuda")
    with pytest.raises(binding.DSAError):
        binding.indexer_kl(s, s, q_pos0=1)  # q_pos0 + Tq > L
    with pytest.raises(binding.DSAError):
        binding.indexer_kl(s, s, q_pos0=-1)


# ---------------------------------------------------------------- backward

def _bf16_exact_grad(gen, shape):
    """Incoming gradients m / 64 with m uniform in [-64, 64]: exact in bf16,
    so a path that rounds G = g w [x > 0] to bf16 loses nothing."""
    return torch.randint(-64, 65, shape, generator=gen).to(torch.float32) / 64.0


def _check_backward(wl, cpu, grad, dq, dk, dw, rows=None, keys=None, rel=1e-5):
    """GPU dq/dw on `rows` (flat b*Tq+i) and dk on `keys` (flat b*L+s)
    against the oracle: |err| <= rel * (sum of |terms|) + 1e-6."""
    from parity_helpers import bits
    q, k, w = bits(cpu["q_idx"]), bits(cpu["k_idx"]), cpu["w"].numpy()
    g = grad.cpu().numpy() if torch.is_tensor(grad) else grad
    if rows is None:
        rows = np.arange(wl.B * wl.Tq)
    if keys is None:
        keys = np.arange(wl.B * wl.L)
    rb, ri = rows // wl.Tq, rows % wl.Tq
    ref = kl.indexer_backward_rows(q, k, w, g, rb, ri + wl.q_pos0, ri)
    got_dq = dq.cpu().numpy()[rb, ri].astype(np.float64)
    got_dw = dw.cpu().numpy()[rb, ri].astype(np.float64)
    assert np.all(np.abs(got_dq - ref["dq"]) <= rel * ref["dq_abs"] + 1e-6), "dq"
    # the tensor-core path forms dw as q . sum_s M k with M = g [x > 0] in bf16:
    # rel of sum |g| ReLU(x), plus fp32 rounding of the 128-term dot product
    from oracle.kl import to_f64
    qa = np.abs(to_f64(q)[rb, ri])
    wa = np.abs(w[rb, ri]).astype(np.float64)
    dot_abs = (qa * ref["dq_abs"]).sum(axis=-1) / np.where(wa > 0, wa, 1.0)
    assert np.all(np.abs(got_dw - ref["dw"]) <= rel * ref["dw_abs"] + 1e-6 * dot_abs + 1e-6), "dw"
    kb, ks = keys // wl.L, keys % wl.L
    refk = kl.indexer_backward_keys(q, k, w, g, kb, ks, wl.q_pos0)
    got_dk = dk.cpu().numpy()[kb, ks].astype(np.float64)
    assert np.all(np.abs(got_dk - refk["dk"]) <= rel * refk["dk_abs"] + 1e-6), "dk"


BWD_SHAPES = {
    "toy16": WORKLOADS["toy16"],
    "bwd_small_f32": WORKLOADS["toy16"].replace(name="bwd_small_f32", B=2, Tq=45, L=45, H_I=3, d_I=5,
                                                seed=40),
    "bwd_chunked": WORKLOADS["prefill8k"].replace(name="bwd_chunked", B=2, Tq=70, L=340, q_pos0=230,
                                                  seed=41),
    "bwd_prefill_300": WORKLOADS["prefill8k"].replace(name="bwd_prefill_300", Tq=300, L=300, seed=42),
    "bwd_odd": WORKLOADS["prefill8k"].replace(name="bwd_odd", Tq=150, L=150, H_I=32, d_I=64, seed=43),
    # the tensor-core path with 32 and 128 heads (four and one queries per group)
    "bwd_heads32": WORKLOADS["prefill8k"].replace(name="bwd_heads32", Tq=260, L=260, H_I=32, seed=44),
    "bwd_heads128": WORKLOADS["prefill8k"].replace(name="bwd_heads128", B=2, Tq=131, L=200, q_pos0=69, H_I=128,
                                                   seed=45),
}


@pytest.mark.parametrize("name", sorted(BWD_SHAPES))
@pytest.mark.parametrize("grad_kind", ["exact", "kl"])
def test_indexer_backward(cuda, name, grad_kind):
    wl = BWD_SHAPES[name]
    cpu = make_inputs(wl)
    dev = to_device(cpu, "cuda")
    gen = torch.Generator().manual_seed(wl.seed + 1000)
    if grad_kind == "exact":
        grad = _bf16_exact_grad(gen, (wl.B, wl.Tq, wl.L)).cuda()
    else:  # the dense warm-up loss's own gradient on these scores
        scores = binding.indexer_scores(dev["q_idx"], dev["k_idx"], dev["w"], wl.q_pos0)
        target = target_weights(gen, (wl.B, wl.Tq, wl.L)).cuda()
        _, _, grad = binding.indexer_kl(scores, target, wl.q_pos0)
    dq, dk, dw = binding.indexer_backward(dev["q_idx"], dev["k_idx"], dev["w"], grad, wl.q_pos0)
    torch.cuda.synchronize()
    # bf16 G on the tensor-core path: 2^-8 of the absolute sums when g is not
    # exact in bf16; fp32 everywhere else
    rel = 2.0 ** -8 if (grad_kind == "kl" and wl.dtype == "bf16") else 1e-5
    _check_backward(wl, cpu, grad, dq, dk, dw, rel=rel)


def test_indexer_backward_partial_outputs(cuda):
    """Only dk, then only dq and dw: the same values as the full call."""
    wl = BWD_SHAPES["bwd_chunked"]
    dev = to_device(make_inputs(wl), "cuda")
    grad = _bf16_exact_grad(torch.Generator().manual_seed(5), (wl.B, wl.Tq, wl.L)).cuda()
    dq, dk, dw = binding.indexer_backward(dev["q_idx"], dev["k_idx"], dev["w"], grad, wl.q_pos0)
    _, dk2, _ = binding.indexer_backward(dev["q_idx"], dev["k_idx"], dev["w"], grad, wl.q_pos0, want=("dk",))
    dq2, _, dw2 = binding.indexer_backward(dev["q_idx"], dev["k_idx"], dev["w"], grad, wl.q_pos0,
                                           want=("dq", "dw"))
    torch.cuda.synchronize()
    assert torch.equal(dk, dk2) and torch.equal(dq, dq2) and torch.equal(dw, dw2)
    # keys after the last query row receive nothing
    assert not dk[:, wl.q_pos0 + wl.Tq:].any()


@pytest.mark.parametrize("name", ["prefill8k"])
def test_indexer_backward_full_size_sampled(cuda, name):
    """The training step's backward at full size (dense warm-up loss on the
    indexer's own scores, then dq, dk, dw on the tensor cores), checked on
    sampled query rows and keys against the oracle (G rounded to bf16:
    2^-8 of the absolute sums)."""
    wl = WORKLOADS[name]
    cpu = make_inputs(wl)
    dev = to_device(cpu, "cuda")
    scores = binding.indexer_scores(dev["q_idx"], dev["k_idx"], dev["w"], wl.q_pos0)
    gen = torch.Generator().manual_seed(77)
    target = target_weights(gen, (wl.B, wl.Tq, wl.L)).cuda()
    _, _, grad = binding.indexer_kl(scores, target, wl.q_pos0, want_sum=False)
    del scores, target
    dq, dk, dw = binding.indexer_backward(dev["q_idx"], dev["k_idx"], dev["w"], grad, wl.q_pos0)
    binding.device_error()
    n = wl.Tq
    rows = np.array([0, 1, 127, 128, n // 2 + 3, n - 2, n - 1])
    keys = np.array([0, 5, 127, 128, n // 3, n - 129, n - 1])
    g_rows = grad[0, torch.from_numpy(rows)].cpu().numpy()
    # the oracle needs g only on the sampled rows (dq, dw) and columns (dk)
    g = np.zeros((1, wl.Tq, wl.L), dtype=np.float32)
    g[0, rows] = g_rows
    g[0][:, keys] = grad[0][:, torch.from_numpy(keys)].cpu().numpy()
    _check_backward(wl, cpu, g, dq, dk, dw, rows=rows, keys=keys, rel=2.0 ** -8)
