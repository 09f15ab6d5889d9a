"""CPU oracle for the indexer's training loss and its backward pass --
TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU legs of ``bench.py``
may import this module. The CUDA library never calls it, and it shares no
code with the CUDA sources. Plain numpy in fp64, one query row at a time; a
matrix product is the only library step.

Sources (page title, section, equation):
  "DeepSeek Sparse Attention: Learned Token Selection from Scratch"
    §5.2, the two steps that build the target: sum the heads' attention
          weights, then L1-normalise along the keys     -> target_from_heads
    §5.4, boxed loss: sum over t of KL(p_t || Softmax(I_t)) over every
          candidate (dense warm-up)                      -> kl_rows (idx=None)
    §6.2, boxed loss restricted to the selected set S_t  -> kl_rows (idx)
    §6.4, the gradient reaches only the indexer's inputs -> indexer_backward_*
  "DeepSeek NSA and DSA: From Native Sparse Attention to Fine-Grained Token
   Selection" §3.3, the same two losses.
  The indexer score it differentiates is the one of "Learned Token
  Selection" §2.1: I[t,s] = sum_j w[t,j] ReLU(q[t,j] . k[s]).

Readings of points the pages leave open (also listed in the design notes):
  - the loss of one query row is KL(p_hat || q) over the row's set: s <= t
    for the dense loss, the valid entries of idx (not -1) for the restricted
    one; q = softmax of I over that set;
  - the target weights are L1-normalised over the set (§5.2, step 2), so the
    head sums a[t,s] or an already normalised p may be passed; restricting a
    dense target to S_t and renormalising is the reading of "the target
    distribution restricted to the selected set"; a row whose weights sum to
    0 contributes no loss and no gradient;
  - 0 * log 0 = 0: a target weight of 0 adds nothing to the loss;
  - the gradient of the summed loss with respect to I[t,s] is
    q[t,s] - p_hat[t,s] on the row's set and 0 elsewhere (s > t, or s not
    in S_t);
  - ReLU'(0) = 0 (a dot product of exactly 0 passes no gradient), the
    convention of common autograd libraries; integer-valued inputs hit it.

Parity pins (tests/test_oracle_kl_pins.py): the §5.3 numerical example
(p_{10,3} = 0.91 / 8 = 0.11375), closed forms (zero loss at I = log p + c,
log n - H(p) for equal scores, the cross-entropy LSE(I) - I[s*] for a
one-hot target), torch's kl_div on random rows, central differences of the
loss and of the C oracle's indexer scores, torch autograd in fp64 with its
ReLU'(0) = 0, and brute-force loops on tiny inputs.
"""
from __future__ import annotations

import numpy as np


def to_f64(a) -> np.ndarray:
    """float64 values of oracle inputs: float32 arrays, uint16 arrays holding
    bf16 bit patterns, or uint8 arrays holding e4m3 codes."""
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    if a.dtype == np.uint8:
        import oracle
        return oracle.e4m3_decode(a).reshape(a.shape)
    return a.astype(np.float64)


def target_from_heads(alpha) -> np.ndarray:
    """p[s] for one query row from the heads' attention weights alpha[h, s]
    ("Learned Token Selection" §5.2): a = sum over heads, p = a / sum(a)."""
    alpha = np.asarray(alpha, dtype=np.float64)
    a = alpha.sum(axis=0)
    return a / a.sum()


def kl_row(I_set, a_set):
    """(loss, grad) of one row over its set: KL(p_hat || softmax(I_set)) with
    p_hat = a_set / sum(a_set), and d loss / d I_set = softmax(I_set) - p_hat.
    """
    I = np.asarray(I_set, dtype=np.float64)
    a = np.asarray(a_set, dtype=np.float64)
    total = a.sum()
    if I.size == 0 or total == 0.0:
        return 0.0, np.zeros_like(I)
    p = a / total
    m = I.max()
    z = np.exp(I - m)
    Z = z.sum()
    q = z / Z
    log_q = (I - m) - np.log(Z)
    on = p > 0
    loss = float(np.sum(p[on] * (np.log(p[on]) - log_q[on])))
    return loss, q - p


def kl_rows(scores, target, row_t, idx=None):
    """Per-row indexer loss and its gradient.

    scores [R, L]: I[t, s] of each requested query row (entries s > t are
    ignored). Dense loss (idx None, §5.4): target [R, L], the row's set is
    s <= t. Restricted loss (§6.2): idx [R, k] int32 with -1 padding and
    target [R, k] aligned with idx; the row's set is its valid idx entries.
    Returns (loss [R] float64, grad [R, L] float64, zero outside the set).
    """
    scores = np.asarray(scores, dtype=np.float64)
    target = np.asarray(target, dtype=np.float64)
    row_t = np.asarray(row_t)
    R, L = scores.shape
    loss = np.zeros(R, dtype=np.float64)
    grad = np.zeros((R, L), dtype=np.float64)
    for r in range(R):
        t = int(row_t[r])
        if idx is None:
            pos = np.arange(t + 1)
            a = target[r, : t + 1]
        else:
            sel = np.asarray(idx[r])
            valid = sel >= 0
            pos = sel[valid].astype(np.int64)
            a = target[r][valid]
        loss[r], g = kl_row(scores[r, pos], a)
        grad[r, pos] = g
    return loss, grad


def _row_terms(q_row, keys, w_row, g_row):
    """x[j, s] = q[j] . k[s]; G[j, s] = g[s] w[j] [x > 0] (d I / d x times the
    incoming gradient); returns x, G."""
    x = q_row @ keys.T
    G = w_row[:, None] * (x > 0) * g_row[None, :]
    return x, G


def indexer_backward_rows(q_idx, k_idx, w, grad, row_b, row_t, row_i=None):
    """dq and dw of the requested query rows for the incoming gradient
    grad = d loss / d I ("Learned Token Selection" §2.1, §6.4):

      dw[t, j]  = sum_{s<=t} g[t,s] ReLU(x[t,j,s])
      dq[t, j]  = sum_{s<=t} g[t,s] w[t,j] [x[t,j,s] > 0] k[s]

    q_idx [B, Tq, H, d], k_idx [B, L, d], w [B, Tq, H], grad [B, Tq, L];
    row_b / row_i select the rows (row_i = row_t when q_pos0 = 0), row_t is
    each row's absolute position. Also returns the same sums of absolute
    values (the error scale of a computation that rounds G).
    Returns dict dq [R, H, d], dw [R, H], dq_abs, dw_abs (float64).
    """
    qf, kf, wf = to_f64(q_idx), to_f64(k_idx), np.asarray(w, dtype=np.float64)
    gf = np.asarray(grad, dtype=np.float64)
    row_i = row_t if row_i is None else row_i
    R = len(row_b)
    H, d = qf.shape[2], qf.shape[3]
    dq = np.zeros((R, H, d))
    dw = np.zeros((R, H))
    dq_abs = np.zeros((R, H, d))
    dw_abs = np.zeros((R, H))
    for r in range(R):
        b, i, t = int(row_b[r]), int(row_i[r]), int(row_t[r])
        keys = kf[b, : t + 1]
        g = gf[b, i, : t + 1]
        x, G = _row_terms(qf[b, i], keys, wf[b, i], g)
        relu = np.maximum(x, 0.0)
        dw[r] = (relu * g[None, :]).sum(axis=1)
        dw_abs[r] = (relu * np.abs(g)[None, :]).sum(axis=1)
        dq[r] = G @ keys
        dq_abs[r] = np.abs(G) @ np.abs(keys)
    return {"dq": dq, "dw": dw, "dq_abs": dq_abs, "dw_abs": dw_abs}


def indexer_backward_keys(q_idx, k_idx, w, grad, key_b, key_s, q_pos0: int):
    """dk of the requested keys: every query row t = q_pos0 + i >= s of the
    batch entry contributes

      dk[s] = sum_{t>=s} sum_j g[t,s] w[t,j] [x[t,j,s] > 0] q[t,j].

    Returns dict dk [R, d], dk_abs [R, d] (float64)."""
    qf, kf, wf = to_f64(q_idx), to_f64(k_idx), np.asarray(w, dtype=np.float64)
    gf = np.asarray(grad, dtype=np.float64)
    Tq = qf.shape[1]
    R, d = len(key_b), kf.shape[2]
    dk = np.zeros((R, d))
    dk_abs = np.zeros((R, d))
    for r in range(R):
        b, s = int(key_b[r]), int(key_s[r])
        i0 = max(0, s - q_pos0)  # first query row with t >= s
        q = qf[b, i0:]                                   # [rows, H, d]
        x = q @ kf[b, s]                                 # x[i, j] = q[i, j] . k[s]
        G = wf[b, i0:] * (x > 0) * gf[b, i0:, s][:, None]
        dk[r] = np.einsum("ij,ijd->d", G, q)
        dk_abs[r] = np.einsum("ij,ijd->d", np.abs(G), np.abs(q))
    return {"dk": dk, "dk_abs": dk_abs}


def indexer_backward(q_idx, k_idx, w, grad, q_pos0: int):
    """Full dq [B,Tq,H,d], dk [B,L,d], dw [B,Tq,H] (small problems)."""
    qf = to_f64(q_idx)
    B, Tq = qf.shape[0], qf.shape[1]
    L = np.asarray(k_idx).shape[1]
    rb = np.repeat(np.arange(B), Tq)
    ri = np.tile(np.arange(Tq), B)
    rows = indexer_backward_rows(q_idx, k_idx, w, grad, rb, ri + q_pos0, ri)
    kb = np.repeat(np.arange(B), L)
    ks = np.tile(np.arange(L), B)
    keys = indexer_backward_keys(q_idx, k_idx, w, grad, kb, ks, q_pos0)
    H, d = qf.shape[2], qf.shape[3]
    return {"dq": rows["dq"].reshape(B, Tq, H, d), "dw": rows["dw"].reshape(B, Tq, H),
            "dk": keys["dk"].reshape(B, L, d),
            "dq_abs": rows["dq_abs"].reshape(B, Tq, H, d), "dw_abs": rows["dw_abs"].reshape(B, Tq, H),
            "dk_abs": keys["dk_abs"].reshape(B, L, d)}
