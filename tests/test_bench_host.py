"""Host-side logic of the benchmark: algorithmic work per stage, the
closed-form counts it relies on, and the max-over-ranks timing reduction on
two gloo ranks."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from learned_sparse_attention_dsa_b200.inputs import WORKLOADS


def test_selected_rows_closed_form():
    """sum_t min(t+1, k) = k(k+1)/2 + (n-k)k ("DeepSeek Sparse Attention ..." §7.2)."""
    for name, expect in (("prefill8k", 14_681_088), ("prefill32k", 65_012_736)):
        wl = WORKLOADS[name]
        n, k = wl.L, wl.k
        assert wl.selected_rows() == k * (k + 1) // 2 + (n - k) * k == expect
    wl = WORKLOADS["toy16"]
    assert wl.selected_rows() == 45  # §7.3
    assert WORKLOADS["decode32k"].selected_rows() == 32 * 2048


def test_causal_pairs():
    wl = WORKLOADS["prefill32k"]
    assert wl.causal_pairs() == 32768 * 32769 // 2
    wl = WORKLOADS["decode128k"]
    assert wl.causal_pairs() == 8 * 131072


def test_stage_work_figures():
    w = bench.stage_work(WORKLOADS["decode32k"])
    idx_bytes, idx_flops = w["indexer"]
    # K^I cache 32 x 32768 x 128 bf16 = 268 MB dominates
    assert abs(idx_bytes - 268.4e6) / 268.4e6 < 0.03
    assert abs(idx_flops - 17.18e9) / 17.18e9 < 0.01
    attn_bytes, attn_flops = w["attn"]
    assert abs(attn_bytes - 33.5e6) / 33.5e6 < 0.05
    p4 = bench.stage_work(WORKLOADS["prefill32k"])
    assert abs(p4["indexer"][1] - 8.80e12) / 8.80e12 < 0.01
    assert abs(p4["topk"][0] - 2.15e9) / 2.15e9 < 0.15
    p3 = bench.stage_work(WORKLOADS["prefill8k"])
    assert abs(p3["indexer"][1] - 5.50e11) / 5.50e11 < 0.01
    d5 = bench.stage_work(WORKLOADS["decode128k"])
    # latent rows: V is a view of the 576-wide K row and adds no bytes
    assert abs(d5["attn"][0] - (8 * 2048 * 1152 + 8 * 128 * (576 + 512) * 2 + 8 * 2048 * 4)) < 1


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench._max_over_ranks(1.5 + rank, world, torch.device("cpu"))
        bench._barrier(world)
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=5) for _ in range(2))
    assert res == {0: 2.5, 1: 2.5}


def test_units_and_metric():
    units, unit = bench._units(WORKLOADS["decode32k"], 10)
    assert (units, unit) == (10.0, "decode steps/s")
    units, unit = bench._units(WORKLOADS["prefill8k"], 2)
    assert (units, unit) == (2 * 8192.0, "prefill tokens/s")


def test_oracle_timing_helpers():
    """The CPU-baseline legs: a bounded sample of rows, timed on one thread,
    scaled to a whole step."""
    import oracle
    oracle.build()
    wl = WORKLOADS["toy16"]
    cpu = bench.make_inputs(wl)
    rows = bench._sample_rows_for(wl, 0.2, 1, cpu)
    assert 1 <= rows <= wl.B * wl.Tq
    sec, r, pairs = bench.time_oracle(wl, cpu, rows, 1)
    assert r == rows and sec >= 0.0
    assert pairs == bench.sample_pairs(wl, bench.sample_rows(wl, rows))
    # rows holding a quarter of toy16's causal pairs in 2 s: a full step
    # takes 8 s, 16 tokens / 8 s
    assert bench._oracle_rate(wl, 2.0, wl.causal_pairs() // 4) == pytest.approx(2.0)
    dec = WORKLOADS["decode32k"]
    # 8 of 32 decode rows (32768 pairs each) in 1 s: a step takes 4 s
    assert bench._oracle_rate(dec, 1.0, 8 * 32768) == pytest.approx(0.25)


def test_oracle_row_sample_and_pair_count():
    wl = WORKLOADS["prefill32k"]
    flat = bench.sample_rows(wl, 512, tail=256)
    assert len(flat) == 512 and len(set(flat.tolist())) == 512
    assert flat[-256:].tolist() == list(range(32768 - 256, 32768))
    assert flat[0] == 0
    # sum of t + 1 over the rows, by brute force
    assert bench.sample_pairs(wl, flat) == sum(int(t) + 1 for t in flat)
    assert bench.sample_pairs(wl, range(wl.Tq)) == wl.causal_pairs()
    dec = WORKLOADS["decode128k"]
    assert bench.sample_pairs(dec, [0, 7]) == 2 * 131072


def test_traffic_entries_expire_when_their_kernel_changes(monkeypatch):
    files = ["indexer_tc.cu", "sm100.cuh"]
    entry = {"bytes": 1.0e6, "sources": files, "digest": bench._sources_digest(files), "profile": "x"}
    monkeypatch.setitem(bench.DRAM_TRAFFIC_PER_LAUNCH, ("w", "indexer"), entry)
    assert bench.dram_traffic("w", "indexer") == 1.0e6
    monkeypatch.setitem(bench.DRAM_TRAFFIC_PER_LAUNCH, ("w", "indexer"), dict(entry, digest="0" * 16))
    assert bench.dram_traffic("w", "indexer") is None
    assert bench.dram_traffic("w", "topk") is None


def test_traffic_entries_name_their_profile():
    """Every committed traffic figure names the profile summary it came from."""
    for (wl, stage), e in bench.DRAM_TRAFFIC_PER_LAUNCH.items():
        assert os.path.exists(os.path.join(bench.ROOT, e["profile"])), (wl, stage)


def test_union_rows_counts_each_group_once():
    """The rows a grouped attention fetches: distinct valid positions per
    group of consecutive query rows (padding and out-of-range entries not
    counted), the plain valid count for groups of one."""
    import torch
    import bench
    idx = torch.tensor([[[0, 1, 2, -1], [1, 2, 3, -1], [5, 6, -1, -1]],
                        [[7, 7, -1, -1], [0, 9, -1, -1], [-1, -1, -1, -1]]], dtype=torch.int32)
    assert bench.union_rows(idx, 1, 8) == 3 + 3 + 2 + 2 + 1 + 0  # 9 is out of range, 7 counted twice
    assert bench.union_rows(idx, 2, 8) == 4 + 2 + 2 + 0          # {0..3}, {5, 6}, {0, 7}, {}
    assert bench.union_rows(idx, 4, 8) == 6 + 2


def test_union_rows_matches_brute_force():
    """union_rows against a plain set union on random selections with padding,
    out-of-range entries and ragged last groups."""
    import torch
    import bench
    gen = torch.Generator().manual_seed(7)
    for B, Tq, k, L, group in ((2, 37, 9, 50, 8), (1, 16, 5, 20, 16), (3, 10, 4, 12, 4)):
        idx = torch.randint(-2, L + 3, (B, Tq, k), generator=gen, dtype=torch.int32)
        expect = 0
        for b in range(B):
            for g0 in range(0, Tq, group):
                rows = idx[b, g0:g0 + group].reshape(-1).tolist()
                expect += len({s for s in rows if 0 <= s < L})
        assert bench.union_rows(idx, group, L) == expect
