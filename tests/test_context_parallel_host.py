"""The context-parallel decode step (learned_sparse_attention_dsa_b200.
context_parallel) on two and three gloo ranks on CPU.

The per-shard steps run as CPU stand-ins built on the oracle (its indexer,
top-k and attention rows) plus the definitions of the candidate gather, the
merge and the log-sum-exp combine written out here; the collectives are real
(gloo). The split step must reproduce the oracle's single-context result:
the same selected positions exactly (each member of the global top-k is in
its shard's top-k, and the merge keeps the tie rule), and the same attention
output up to fp32 rounding (the attention over S_t is the log-sum-exp merge
of the shards' partial attentions).
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle

B, L, P, H_I, D_I, K, HQ, HKV, D = 2, 72, 2, 4, 8, 7, 4, 1, 16


def _inputs():
    gen = torch.Generator().manual_seed(99)
    q_idx = torch.randint(-3, 4, (B, 1, H_I, D_I), generator=gen).float()
    k_idx = torch.randint(-3, 4, (B, L, D_I), generator=gen).float()
    w = torch.tensor([0.5, 1.0, 2.0])[torch.randint(0, 3, (B, 1, H_I), generator=gen)]
    q = torch.randn(B, 1, HQ, D, generator=gen)
    kc = torch.randn(B, L, HKV, D, generator=gen)
    vc = torch.randn(B, L, HKV, D, generator=gen)
    return q_idx, k_idx, w, q, kc, vc


class CpuOps:
    """CPU stand-ins for the library calls the context-parallel step makes."""

    @staticmethod
    def indexer_scores(q_idx, k_idx, w, q_pos0):
        rows = np.arange(q_idx.shape[0], dtype=np.int32)
        s = oracle.indexer_rows(q_idx[:, 0].numpy(), w[:, 0].numpy(), k_idx.numpy(), rows,
                                np.full(len(rows), q_pos0, dtype=np.int32))
        return torch.from_numpy(s)[:, None, :]

    @staticmethod
    def topk(scores, k, q_pos0):
        idx = oracle.topk_rows(scores[:, 0].numpy(), np.full(scores.shape[0], q_pos0, dtype=np.int32), k)
        return torch.from_numpy(idx)[:, None, :]

    @staticmethod
    def cp_select_candidates(scores, idx, key_pos0):
        s = scores.numpy()
        i = idx.numpy()
        cs = np.where(i >= 0, np.take_along_axis(s, np.maximum(i, 0), axis=-1), -np.inf).astype(np.float32)
        ci = np.where(i >= 0, i + key_pos0, -1).astype(np.int32)
        return torch.from_numpy(cs), torch.from_numpy(ci)

    @staticmethod
    def cp_merge(cs, ci, k):
        cs, ci = cs.numpy(), ci.numpy()                   # [P, B, 1, kc]
        out = np.full(cs.shape[1:-1] + (k,), -1, dtype=np.int32)
        for b in range(cs.shape[1]):
            cand = [(float(cs[p, b, 0, j]), int(ci[p, b, 0, j])) for p in range(cs.shape[0])
                    for j in range(cs.shape[3]) if ci[p, b, 0, j] >= 0]
            best = sorted(cand, key=lambda x: (-x[0], x[1]))[:k]
            sel = sorted(x[1] for x in best)
            out[b, 0, :len(sel)] = sel
        return torch.from_numpy(out)

    @staticmethod
    def cp_localize(idx, key_pos0, L_local):
        i = idx.numpy()
        return torch.from_numpy(np.where((i >= key_pos0) & (i < key_pos0 + L_local), i - key_pos0, -1)
                                .astype(np.int32))

    @staticmethod
    def sparse_attn(q, k_local, v_local, idx, scale, want_lse=True):
        out, lse = oracle.attn_rows(q[:, 0].numpy(), k_local.numpy(), v_local.numpy(), idx[:, 0].numpy(),
                                    np.arange(q.shape[0], dtype=np.int32), scale, want_lse=True)
        return torch.from_numpy(out)[:, None], torch.from_numpy(lse)[:, None]

    @staticmethod
    def cp_combine(parts, lse):
        parts, lse = parts.numpy(), lse.numpy()           # [P, B, 1, Hq, Dv], [P, B, 1, Hq]
        m = lse.max(axis=0)
        total = m + np.log(np.exp(lse - m).sum(axis=0))
        wgt = np.exp(lse - total)
        return torch.from_numpy((wgt[..., None] * parts).sum(axis=0))


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from learned_sparse_attention_dsa_b200 import context_parallel as cp
        q_idx, k_idx, w, qq, kc, vc = _inputs()
        Ll = L // world
        a = rank * Ll
        out, idx = cp.cp_decode(q_idx, k_idx[:, a:a + Ll].contiguous(), w, qq, kc[:, a:a + Ll].contiguous(),
                                vc[:, a:a + Ll].contiguous(), K, a, L, 1.0 / D ** 0.5, cp.TorchComm(), CpuOps)
        q.put((rank, idx.numpy(), out.numpy()))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world", [P, 3])
def test_context_parallel_decode_gloo_ranks(world):
    ctx = mp.get_context("spawn")
    qu = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, qu)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    res = {r: (i, o) for r, i, o in (qu.get(timeout=5) for _ in range(world))}
    # the single-context oracle
    q_idx, k_idx, w, qq, kc, vc = _inputs()
    rows = np.arange(B, dtype=np.int32)
    t = np.full(B, L - 1, dtype=np.int32)
    scores = oracle.indexer_rows(q_idx[:, 0].numpy(), w[:, 0].numpy(), k_idx.numpy(), rows, t)
    ref_idx = oracle.topk_rows(scores, t, K)
    ref_out = oracle.attn_rows(qq[:, 0].numpy(), kc.numpy(), vc.numpy(), ref_idx, rows, 1.0 / D ** 0.5)
    for r in range(world):
        idx, out = res[r]
        assert np.array_equal(idx[:, 0], ref_idx), f"rank {r}: selection differs"
        assert np.allclose(out[:, 0], ref_out, atol=1e-9, rtol=1e-9), f"rank {r}: output differs"
    # at least two shards contributed (the test would not exercise the merge otherwise)
    assert len(np.unique(ref_idx[ref_idx >= 0] // (L // world))) >= 2


def test_local_candidates_rejects_multi_row_queries():
    from learned_sparse_attention_dsa_b200 import context_parallel as cp
    q_idx, k_idx, w, *_ = _inputs()
    with pytest.raises(ValueError):
        cp.local_candidates(q_idx.repeat(1, 2, 1, 1), k_idx, w, K, 0, L, CpuOps)


def test_shard_after_the_query_has_no_candidates():
    from learned_sparse_attention_dsa_b200 import context_parallel as cp
    q_idx, k_idx, w, *_ = _inputs()
    cs, ci = cp.local_candidates(q_idx, k_idx[:, :8].contiguous(), w, K, 100, 50, CpuOps)
    assert torch.isneginf(cs).all() and (ci == -1).all()
