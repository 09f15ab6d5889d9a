"""GPU parity of the context-parallel decode step, with the P ranks emulated
one after another on one GPU: each shard's local stages run on its own slice
of the caches, and the two all-gathers become stacks of the shards' results.
No kernel waits on another.

The split step must give the single-context selection bit for bit (and thus
the oracle's), and the attention output within the usual bf16 tolerance of
the fp64 oracle.
"""
import numpy as np
import pytest
import torch

from learned_sparse_attention_dsa_b200 import binding
from learned_sparse_attention_dsa_b200 import context_parallel as cp
from learned_sparse_attention_dsa_b200.inputs import WORKLOADS, Workload, make_inputs, to_device
from parity_helpers import assert_attn_close, oracle_forward

pytestmark = pytest.mark.gpu

CASES = {
    # decode32k's shapes at context 5,000 over four ranks
    "gqa_5000_p4": (Workload("gqa_5000_p4", B=3, Tq=1, L=5000, q_pos0=4999, H_I=64, d_I=128, k=2048, Hq=16,
                             Hkv=1, Dqk=128, Dv=128, seed=51), 4),
    # decode128k's latent rows at context 3,000 over three unequal ranks
    "latent_3000_p3": (Workload("latent_3000_p3", B=2, Tq=1, L=3000, q_pos0=2999, H_I=64, d_I=128, k=256,
                                Hq=128, Hkv=1, Dqk=576, Dv=512, kv_alias=True, seed=52), 3),
    # a budget larger than some shards, one KV head per query head
    "perhead_900_p2": (Workload("perhead_900_p2", B=2, Tq=1, L=900, q_pos0=899, H_I=64, d_I=128, k=600, Hq=8,
                                Hkv=8, Dqk=64, Dv=64, seed=53), 2),
}


def _bounds(L, P):
    step = -(-L // P)
    return [(a, min(L, a + step)) for a in range(0, L, step)]


def _emulated_step(wl, dev, P):
    parts = _bounds(wl.L, P)
    cands = [cp.local_candidates(dev["q_idx"], dev["k_idx"][:, a:b].contiguous(), dev["w"], wl.k, a, wl.L)
             for a, b in parts]
    idx = cp.merge(torch.stack([c[0] for c in cands]), torch.stack([c[1] for c in cands]), wl.k)
    outs, lses = [], []
    for a, b in parts:
        kc = dev["k_cache"][:, a:b].contiguous()
        vc = kc[..., : wl.Dv] if wl.kv_alias else dev["v_cache"][:, a:b].contiguous()
        o, l = cp.local_attention(dev["q"], kc, vc, idx, a, wl.scale)
        outs.append(o)
        lses.append(l)
    out = cp.combine(torch.stack(outs), torch.stack(lses))
    binding.device_error()
    return idx, out


@pytest.mark.parametrize("name", sorted(CASES))
def test_context_parallel_decode_emulated(cuda, name):
    wl, P = CASES[name]
    cpu = make_inputs(wl)
    dev = to_device(cpu, "cuda")
    idx, out = _emulated_step(wl, dev, P)
    # the single-GPU forward on the whole context
    idx_full = torch.empty((wl.B, 1, wl.k), dtype=torch.int32, device="cuda")
    out_full = binding.forward(dev["q_idx"], dev["k_idx"], dev["w"], dev["q"], dev["k_cache"], dev["v_cache"],
                               wl.k, wl.q_pos0, wl.scale, idx_out=idx_full)
    torch.cuda.synchronize()
    assert torch.equal(idx, idx_full), "selection differs from the single-context one"
    rows = list(range(wl.B))
    _, o_idx, o_out = oracle_forward(wl, cpu, rows)
    assert np.array_equal(idx.cpu().numpy()[:, 0], o_idx)
    assert_attn_close(out.float().cpu().numpy()[:, 0], o_out, name)
    # every shard took part in the selection
    sel = idx.cpu().numpy()
    for a, b in _bounds(wl.L, P):
        assert ((sel >= a) & (sel < b)).any()


def _merge_reference(cs, ci, k):
    P, R, kc = cs.shape
    out = np.full((R, k), -1, dtype=np.int32)
    for r in range(R):
        cand = [(float(cs[p, r, j]), int(ci[p, r, j])) for p in range(P) for j in range(kc) if ci[p, r, j] >= 0]
        sel = sorted(x[1] for x in sorted(cand, key=lambda x: (-x[0], x[1]))[:k])
        out[r, :len(sel)] = sel
    return out


@pytest.mark.parametrize("P,R,kc,k", [(3, 40, 50, 30), (2, 5, 2048, 2048), (4, 7, 6, 30), (8, 3, 2048, 1000)])
def test_cp_merge_against_definition(cuda, P, R, kc, k):
    """Random candidates with many ties and invalid entries: the merge is the
    k best by (score, then lower position), in ascending position."""
    gen = torch.Generator().manual_seed(P * 1000 + kc)
    cs = torch.randint(-5, 6, (P, R, kc), generator=gen).float()
    # each rank's positions ascending and disjoint, rank r below rank r+1
    ci = torch.sort(torch.randperm(kc * 3, generator=gen)[:kc])[0].to(torch.int32)
    ci = torch.stack([ci + p * kc * 3 for p in range(P)])[:, None, :].repeat(1, R, 1).contiguous()
    drop = torch.rand(P, R, kc, generator=gen) < 0.3
    ci[drop] = -1
    cs[drop] = float("-inf")
    got = binding.cp_merge(cs.cuda(), ci.cuda(), k)
    torch.cuda.synchronize()
    assert np.array_equal(got.cpu().numpy(), _merge_reference(cs.numpy(), ci.numpy(), k))


def test_cp_combine_and_localize(cuda):
    gen = torch.Generator().manual_seed(3)
    P, R, H, Dv = 3, 5, 4, 40
    parts = torch.randn(P, R, H, Dv, generator=gen)
    lse = torch.randn(P, R, H, generator=gen) * 3
    lse[1, 2] = float("-inf")          # a part that selected nothing
    parts[1, 2] = float("nan")         # whose output must be ignored
    lse[:, 4, 1] = float("-inf")       # a pair with no part at all
    out, tot = binding.cp_combine(parts.cuda(), lse.cuda(), want_lse=True)
    out, tot = out.cpu(), tot.cpu()
    l64, p64 = lse.double(), torch.nan_to_num(parts.double())
    ref_tot = torch.logsumexp(l64, dim=0)
    wgt = torch.where(torch.isneginf(l64), torch.zeros_like(l64), torch.exp(l64 - ref_tot))
    ref = (wgt[..., None] * p64).sum(0)
    ok = ~torch.isneginf(ref_tot)
    assert torch.allclose(out.double()[ok], ref[ok], atol=1e-5, rtol=1e-5)
    assert torch.allclose(tot.double()[ok], ref_tot[ok], atol=1e-5)
    assert torch.isneginf(tot[4, 1]) and not out[4, 1].any()
    idx = torch.tensor([[5, 17, 30, -1, 99]], dtype=torch.int32, device="cuda")
    loc = binding.cp_localize(idx, 10, 25)
    assert loc.tolist() == [[-1, 7, 20, -1, -1]]
