"""Context-parallel decode step: the context split by position over ranks.

Each rank holds positions [key_pos0, key_pos0 + L_local) of the indexer keys
and of the KV cache; every rank holds the query rows of the step (decode:
one row per batch entry, at position t = L_total - 1). The selection S_t
("DeepSeek Sparse Attention: Learned Token Selection from Scratch" §3.1) is
exact: each member of S_t is among the k best of its own shard, so the ranks
exchange only their local selections (k scores and k positions per row), and
the attention over S_t (§3.3) is a log-sum-exp merge of the ranks' partial
attentions. Per step:

  1. local indexer scores and top-k (dsa_indexer_scores, dsa_topk),
     as (score, global position) candidates (dsa_cp_select_candidates);
  2. all-gather of the candidates, 8 k bytes per row and rank;
  3. the merge into the global selection (dsa_cp_merge), the same on every
     rank;
  4. attention over the selected positions held locally (dsa_cp_localize,
     dsa_sparse_attn with the log-sum-exp);
  5. all-gather of (output, log-sum-exp) and the merge (dsa_cp_combine).

Ranks must be ordered by position (rank r holds the r-th block), so that the
gathered candidates come in ascending global position, which the merge's tie
rule relies on. The arithmetic runs in the CUDA library; this module only
sequences the calls and the collectives (NCCL through torch.distributed).
"""
from __future__ import annotations

import torch


class TorchComm:
    """All-gather over a torch.distributed group: returns [P, *shape]."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.size = dist.get_world_size(group)

    def all_gather(self, t: torch.Tensor) -> torch.Tensor:
        t = t.contiguous()
        out = torch.empty((self.size,) + tuple(t.shape), dtype=t.dtype, device=t.device)
        if t.is_cuda:
            self.dist.all_gather_into_tensor(out, t, group=self.group)
        else:  # gloo has no all_gather_into_tensor for every dtype
            parts = list(out.unbind(0))
            self.dist.all_gather(parts, t, group=self.group)
        return out


def _cuda_ops():
    from . import binding
    return binding


def local_candidates(q_idx, k_idx_local, w, k: int, key_pos0: int, L_total: int, ops=None):
    """Step 1 on this rank: ([B, 1, k] scores, [B, 1, k] global positions)
    of the local selection (-inf / -1 where the shard has fewer than k
    candidates, all of them when it lies after the query)."""
    ops = ops or _cuda_ops()
    B, Tq = q_idx.shape[0], q_idx.shape[1]
    if Tq != 1:
        raise ValueError("the context-parallel step is a decode step: one query row per batch entry")
    L_local = k_idx_local.shape[1]
    t = L_total - 1
    if t < key_pos0:  # every local position is after the query
        return (torch.full((B, 1, k), float("-inf"), dtype=torch.float32, device=q_idx.device),
                torch.full((B, 1, k), -1, dtype=torch.int32, device=q_idx.device))
    q_pos0_local = min(t - key_pos0, L_local - 1)
    scores = ops.indexer_scores(q_idx, k_idx_local, w, q_pos0_local)
    idx = ops.topk(scores, k, q_pos0_local)
    return ops.cp_select_candidates(scores, idx, key_pos0)


def merge(cand_scores, cand_idx, k: int, ops=None):
    """Step 3: [P, B, 1, kc] candidates -> the global selection [B, 1, k]."""
    ops = ops or _cuda_ops()
    return ops.cp_merge(cand_scores, cand_idx, k)


def local_attention(q, k_local, v_local, idx, key_pos0: int, scale: float, ops=None):
    """Step 4: this rank's partial attention over the selected positions it
    holds: (output [B, 1, Hq, Dv], log-sum-exp [B, 1, Hq])."""
    ops = ops or _cuda_ops()
    idx_local = ops.cp_localize(idx, key_pos0, k_local.shape[1])
    return ops.sparse_attn(q, k_local, v_local, idx_local, scale, want_lse=True)


def combine(parts, parts_lse, ops=None):
    """Step 5: [P, B, 1, Hq, Dv] partial outputs -> [B, 1, Hq, Dv]."""
    ops = ops or _cuda_ops()
    return ops.cp_combine(parts, parts_lse)


def cp_decode(q_idx, k_idx_local, w, q, k_local, v_local, k: int, key_pos0: int, L_total: int, scale: float,
              comm, ops=None):
    """One decode step with the context split over the ranks of `comm`.

    q_idx [B,1,H^I,d^I], w [B,1,H^I], q [B,1,Hq,Dqk]: the step's query rows
    (the same on every rank); k_idx_local [B,L_local,d^I] and the caches
    k_local / v_local [B,L_local,Hkv,D]: this rank's positions
    [key_pos0, key_pos0 + L_local). Returns (output [B,1,Hq,Dv], the global
    selection [B,1,k] int32), identical on every rank.
    """
    cand_scores, cand_idx = local_candidates(q_idx, k_idx_local, w, k, key_pos0, L_total, ops)
    idx = merge(comm.all_gather(cand_scores), comm.all_gather(cand_idx), k, ops)
    out, lse = local_attention(q, k_local, v_local, idx, key_pos0, scale, ops)
    return combine(comm.all_gather(out), comm.all_gather(lse), ops), idx
