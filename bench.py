"""Benchmark of the DSA forward path (indexer -> top-k -> sparse attention).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step is one dsa_forward call over one batch of synthetic input: the
lightning-indexer scores, the top-k selection and the attention over the
selected rows. The default workload is the decode step of 32 sequences at
context 32,768 with k = 2048 (16 query heads sharing one 128-wide KV head);
its unit is decode steps per second. Prefill workloads report tokens per
second. Rank 0 prints one JSON line.

Timing: W untimed warm-up steps, then exactly K steps between two CUDA events
on the launching stream, bracketed by a barrier and a device synchronize,
max over ranks. Every step streams the 268 MB indexer-key cache (larger than
the 126 MB L2), so L2 is not flushed between steps. Per-stage times (for the
roofline) are taken the same way in separate loops after the main region.
--impl reference times the CPU oracle on the host cores instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from learned_sparse_attention_dsa_b200.inputs import WORKLOADS, make_inputs, to_device  # noqa: E402

METRIC = "prefill tokens/s and decode steps/s at k=2048; % HBM/tensor roofline per stage"

# dram__bytes_read.sum + dram__bytes_write.sum per launch of a stage's kernel,
# from an ncu capture (the profiles/ summary named here holds its command and
# figures), with the SHA-256 prefix of the kernel sources it was taken on.
# dram_traffic() reports an entry only while those sources are unchanged, so
# a kernel edit turns its traffic into null until it is captured again.
_IDX = ["indexer_tc.cu", "sm100.cuh", "common.cuh", "tma_map.cu"]
_TOPK = ["topk.cu", "topk_block.cu", "common.cuh"]
DRAM_TRAFFIC_PER_LAUNCH = {
    ("decode32k", "indexer"): {"bytes": 271.96e6, "sources": _IDX, "digest": "73a556a5f522a639",
                               "profile": "profiles/dram_stages_decode32k.md"},
    ("decode32k", "topk"): {"bytes": 4.27e6, "sources": _TOPK, "digest": "65454fadbee778ff",
                            "profile": "profiles/dram_stages_decode32k.md"},
    ("decode32k", "attn"): {"bytes": 34.02e6, "sources": ["attn_tc.cu", "common.cuh"],
                            "digest": "dc4d1f57bbd48356", "profile": "profiles/dram_stages_decode32k.md"},
    ("decode128k", "indexer"): {"bytes": 271.42e6, "sources": _IDX, "digest": "73a556a5f522a639",
                                "profile": "profiles/dram_stages_decode128k.md"},
    ("decode128k", "topk"): {"bytes": 4.27e6, "sources": _TOPK, "digest": "65454fadbee778ff",
                             "profile": "profiles/dram_stages_decode128k.md"},
    # the stage's two kernels: the attention and the combine of its split partials
    ("decode128k", "attn"): {"bytes": 28.65e6, "sources": ["attn_mla_tc.cu", "sm100.cuh", "common.cuh", "tma_map.cu"],
                             "digest": "398fd6177746f459", "profile": "profiles/dram_stages_decode128k.md"},
    ("prefill8k", "indexer"): {"bytes": 219.44e6, "sources": _IDX, "digest": "73a556a5f522a639",
                               "profile": "profiles/dram_stages_prefill8k.md"},
    ("decode32k_fp8", "indexer"): {"bytes": 135.96e6, "sources": _IDX, "digest": "73a556a5f522a639",
                                   "profile": "profiles/indexer_tc_e4m3_decode32k.md"},
    ("decode32k_fp8", "topk"): {"bytes": 4.27e6, "sources": _TOPK, "digest": "65454fadbee778ff",
                                "profile": "profiles/indexer_tc_e4m3_decode32k.md"},
    ("prefill8k", "topk"): {"bytes": 170.64e6, "sources": _TOPK, "digest": "65454fadbee778ff",
                            "profile": "profiles/dram_stages_prefill8k.md"},
    ("prefill8k", "attn"): {"bytes": 92.45e6, "sources": ["attn_perhead.cu", "common.cuh"],
                            "digest": "f553d8ec079b5f95", "profile": "profiles/dram_stages_prefill8k.md"},
}


def _sources_digest(files):
    import hashlib
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "learned_sparse_attention_dsa_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def dram_traffic(workload, stage):
    e = DRAM_TRAFFIC_PER_LAUNCH.get((workload, stage))
    if e is None:
        return None
    try:
        if _sources_digest(e["sources"]) != e["digest"]:
            return None
    except OSError:
        return None
    return e["bytes"]


# ------------------------------------------------------------------ helpers

def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


def _tensor_peak(wl, stage, peaks):
    """Dense tensor peak for the stage's input type: the measured bf16 peak,
    times 2 for the e4m3 indexer (4.5 / 2.25 PFLOP/s nominal dense)."""
    if stage == "indexer" and wl.idx_dtype == "e4m3":
        return 2.0 * peaks["bf16_tflops"]
    return peaks["bf16_tflops"]


def stage_work(wl, attn_rows=None):
    """Algorithmic bytes and flops per forward pass, per stage.

    indexer: reads K^I once, q^I and w once, writes one fp32 score per causal
             pair; flops = 2 * H_I * d_I per causal pair (the contraction).
    top-k:   reads one fp32 score per causal pair, writes k int32 per row.
    attn:    reads each selected KV row once per KV head (K and V; a V that is
             a view of the K row adds nothing), Q once, writes the output;
             flops = 2 * Hq * (Dqk + Dv) per selected row. attn_rows, when
             given, replaces the selected rows in the bytes: the rows the
             kernel has to fetch when query rows share the gathers of the
             union of their selections (each union row once per group).
    """
    eb = 4 if wl.dtype == "f32" else 2
    ieb = 1 if wl.idx_dtype == "e4m3" else eb  # indexer input element bytes
    rows = wl.B * wl.Tq
    pairs = wl.causal_pairs()
    sel = wl.selected_rows()
    idx_bytes = (wl.B * wl.L * wl.d_I * ieb + rows * wl.H_I * wl.d_I * ieb + rows * wl.H_I * 4
                 + pairs * 4)
    idx_flops = 2.0 * wl.H_I * wl.d_I * pairs
    topk_bytes = pairs * 4 + rows * wl.k * 4
    kv_row = wl.Hkv * (wl.Dqk if wl.kv_alias else wl.Dqk + wl.Dv) * eb
    attn_bytes = (sel if attn_rows is None else attn_rows) * kv_row + rows * wl.Hq * (wl.Dqk + wl.Dv) * eb \
        + rows * wl.k * 4
    attn_flops = 2.0 * wl.Hq * (wl.Dqk + wl.Dv) * sel
    return {"indexer": (idx_bytes, idx_flops), "topk": (topk_bytes, 0.0), "attn": (attn_bytes, attn_flops)}


class ClockSampler:
    """Polls NVML for SM clock and throttle reasons on a background thread."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown", 0x1: "gpu_idle",
               0x2: "applications_clocks_setting"}

    def __init__(self, device_index: int, period_s: float = 0.002):
        self.samples = []
        self.period = period_s
        self._stop = threading.Event()
        self._thread = None
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:  # NVML missing: no clock record
            self._nvml = None

    def _run(self):
        nv = self._nvml
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                self.samples.append((time.perf_counter(), mhz, reasons))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self._nvml is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self):
        if self._thread is not None:
            self._stop.set()
            self._thread.join()

    def summary(self, t0: float, t1: float):
        if self._nvml is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "NVML unavailable"}
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        note = "sampled during the timed region"
        if not inside:  # region shorter than the polling period: nearest samples
            inside = sorted(self.samples, key=lambda s: min(abs(s[0] - t0), abs(s[0] - t1)))[:3]
            note = "timed region shorter than the polling period; nearest samples"
        mhz = [s[1] for s in inside]
        mask = 0
        for s in inside:
            mask |= int(s[2])
        reasons = [name for bit, name in self.REASONS.items() if mask & bit and name != "gpu_idle"]
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(inside), "note": note}


def _dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def _max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def _units(wl, steps: int) -> tuple[float, str]:
    if wl.is_decode:
        return float(steps), "decode steps/s"
    return float(steps * wl.B * wl.Tq), "prefill tokens/s"


# ------------------------------------------------------------------ oracle timing

def sample_rows(wl, n_rows: int, tail: int = 0) -> np.ndarray:
    """Flat query-row ids of an oracle sample: n_rows - tail rows spread
    evenly over the batch, plus the last `tail` rows (the longest prefill
    rows), without repeats."""
    total = wl.B * wl.Tq
    n_rows = min(n_rows, total)
    tail = min(tail, n_rows)
    spread = np.linspace(0, total - 1 - tail, num=n_rows - tail).round().astype(np.int64) if n_rows > tail \
        else np.zeros(0, dtype=np.int64)
    last = np.arange(total - tail, total, dtype=np.int64)
    return np.unique(np.concatenate([spread, last]))


def sample_pairs(wl, flat) -> int:
    """Causal (query, key) pairs of the sampled rows: sum of t + 1."""
    flat = np.asarray(flat, dtype=np.int64)
    return int(((flat % wl.Tq) + wl.q_pos0 + 1).sum())


def bits(t):
    """A CPU tensor as the oracle reads it: fp32 values, raw bf16 bits
    (uint16) or e4m3 codes (uint8)."""
    t = t.contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float8_e4m3fn:
        return t.view(torch.uint8).numpy()
    return t.numpy()


def time_oracle(wl, cpu, n_rows: int, nthreads: int = 0, tail: int = 0):
    """Run the CPU oracle (all three stages) on a sample of n_rows query rows
    (sample_rows) and return (seconds, rows, causal pairs of those rows)."""
    import oracle


    flat = sample_rows(wl, n_rows, tail)
    row_b = (flat // wl.Tq).astype(np.int32)
    row_i = (flat % wl.Tq).astype(np.int32)
    row_t = row_i + wl.q_pos0
    q_idx = bits(cpu["q_idx"][row_b, row_i])
    w = cpu["w"][row_b, row_i].numpy()
    q = bits(cpu["q"][row_b, row_i])
    kc = cpu["k_cache"]
    kbuf = bits(kc)
    ks = (kc.shape[1] * kc.shape[2] * kc.shape[3], kc.shape[2] * kc.shape[3], kc.shape[3])
    if wl.kv_alias:
        vbuf, vs = kbuf, ks
    else:
        vc = cpu["v_cache"]
        vbuf = bits(vc)
        vs = (vc.shape[1] * vc.shape[2] * vc.shape[3], vc.shape[2] * vc.shape[3], vc.shape[3])
    k_idx = bits(cpu["k_idx"])
    t0 = time.perf_counter()
    scores = oracle.indexer_rows(q_idx, w, k_idx, row_b, row_t, nthreads)
    idx = oracle.topk_rows(scores, row_t, wl.k, nthreads)
    oracle.attn_rows(q, kbuf, vbuf, idx, row_b, wl.scale, k_strides=ks, v_strides=vs, Hkv=wl.Hkv,
                     Dv=wl.Dv, nthreads=nthreads)
    return time.perf_counter() - t0, len(flat), sample_pairs(wl, flat)


def _oracle_rate(wl, seconds: float, pairs: int) -> float:
    """Metric value of the oracle (decode steps/s or prefill tokens/s) from
    `seconds` spent on rows holding `pairs` causal pairs: the whole step is
    extrapolated by the exact pair count (every decode row has the same
    count; in prefill the indexer's work per row grows with t)."""
    step_seconds = seconds * wl.causal_pairs() / pairs
    if wl.is_decode:
        return 1.0 / step_seconds
    return wl.B * wl.Tq / step_seconds


def _sample_rows_for(wl, budget_s: float, nthreads: int, cpu) -> int:
    """Rows of the oracle that fit a wall-clock budget (probe with a few rows)."""
    probe = max(1, min(wl.B * wl.Tq, max(8, nthreads)))
    sec, rows, _ = time_oracle(wl, cpu, probe, nthreads)
    per_row = sec / rows
    return int(max(1, min(wl.B * wl.Tq, budget_s / per_row)))


# ------------------------------------------------------------------ reference arm

def run_reference(args, wl):
    world, rank, _ = _dist()
    if rank != 0:
        return
    import oracle
    oracle.build()
    cpu = make_inputs(wl)
    nthreads = oracle.max_threads()
    # Size each step so that the whole run ends within a few minutes.
    budget = max(0.5, 150.0 / max(1, args.steps + args.warmup))
    rows = _sample_rows_for(wl, budget, nthreads, cpu)
    for _ in range(args.warmup):
        time_oracle(wl, cpu, rows, nthreads)
    secs = []
    for _ in range(args.steps):
        s, r, pairs = time_oracle(wl, cpu, rows, nthreads)
        secs.append(s)
    mean_s = sum(secs) / len(secs)
    value = _oracle_rate(wl, mean_s, pairs)
    _, unit = _units(wl, 1)
    sample = (f"{rows} of {wl.B * wl.Tq} query rows per step (all three stages), extrapolated to a full "
              f"step by the exact causal-pair count")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": unit, "n_gpus": 0,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * mean_s * wl.causal_pairs() / pairs,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": _config(wl, world),
        "cpu_baseline": {"value": value, "unit": unit, "cores": nthreads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def _config(wl, world):
    return {"workload": wl.name, "global_batch": wl.B * world, "seq_len": wl.L, "query_rows": wl.Tq,
            "k": wl.k, "indexer_heads": wl.H_I, "indexer_dim": wl.d_I, "q_heads": wl.Hq,
            "kv_heads": wl.Hkv, "d_qk": wl.Dqk, "d_v": wl.Dv, "kv_alias": wl.kv_alias,
            "parallelism": f"replicas{world}",
            "l2": "no flush: every step streams the indexer-key cache "
                  f"({wl.B * wl.L * wl.d_I * (1 if wl.idx_dtype == 'e4m3' else 4 if wl.dtype == 'f32' else 2) / 1e6:.0f} MB), "
                  "larger than the 126 MB L2"}


# ------------------------------------------------------------------ our arm

# The other configurations measured by the default run, each reported under
# "workloads" in the same JSON line (the headline workload is decode32k).
EXTRA_WORKLOADS = ("toy16", "prefill8k", "prefill32k", "decode128k", "decode32k_fp8")
# Minimum length of the window of identical back-to-back steps over which
# clocks are sampled (the steps queued right before the timed ones, then the
# timed ones).
CLOCK_WINDOW_S = 0.5


def union_rows(idx, group: int, L: int) -> int:
    """KV rows a grouped attention fetches: for every batch entry and every
    group of `group` consecutive query rows, the number of distinct valid
    positions in their selections (group 1: the valid entries)."""
    B, Tq, k = idx.shape
    if group <= 1:
        return int(((idx >= 0) & (idx < L)).sum())
    ng = (Tq + group - 1) // group
    x = idx
    if ng * group != Tq:
        x = torch.cat([x, torch.full((B, ng * group - Tq, k), -1, dtype=idx.dtype, device=idx.device)], 1)
    x = x.reshape(B * ng, group * k).long()
    x = torch.where((x >= 0) & (x < L), x, torch.full_like(x, L))  # padding -> an extra column
    total = 0
    for c in range(0, x.shape[0], 64):
        xs = x[c:c + 64]
        m = torch.zeros((xs.shape[0], L + 1), dtype=torch.bool, device=x.device)
        m.scatter_(1, xs, True)
        total += int(m[:, :L].sum())
    return total


def _stage_report(wl, stages, peaks, attn_info=None):
    work = stage_work(wl, attn_info["gathered_rows"] if attn_info and attn_info.get("row_group", 1) > 1 else None)
    report = {}
    for name, ms in stages.items():
        nbytes, flops = work[name]
        sec_s = ms / 1000.0
        gbs = nbytes / sec_s / 1e9
        entry = {"ms": ms, "GB/s": gbs, "hbm_frac": gbs / peaks["hbm_gbs"],
                 "algorithmic_bytes": nbytes, "algorithmic_flops": flops,
                 "dram_traffic": dram_traffic(wl.name, name)}
        if flops:
            entry["TFLOP/s"] = flops / sec_s / 1e12
            entry["tensor_frac"] = entry["TFLOP/s"] / _tensor_peak(wl, name, peaks)
        report[name] = entry
    if attn_info and attn_info.get("row_group", 1) > 1:
        report["attn"]["row_group"] = attn_info["row_group"]
        report["attn"]["gathered_rows"] = attn_info["gathered_rows"]
        report["attn"]["selected_rows"] = wl.selected_rows()
        report["attn"]["note_rows"] = (f"groups of {attn_info['row_group']} consecutive query rows share the gathers "
                                       "of the union of their selections: algorithmic_bytes count each union row "
                                       "once per group (selected_rows is the per-row count)")
    return report


def _roofline(wl, stage_report, peaks):
    """The dominant stage against its bound: tensor for the prefill indexer,
    HBM for every other stage."""
    dominant = max(stage_report, key=lambda n: stage_report[n]["ms"])
    d = stage_report[dominant]
    traffic = dram_traffic(wl.name, dominant)
    if dominant == "indexer" and not wl.is_decode:
        tpeak = _tensor_peak(wl, dominant, peaks)
        return {"bound": "tensor", "kernel": dominant, "achieved": d["TFLOP/s"], "peak": tpeak,
                "unit": "TFLOP/s", "frac": d["TFLOP/s"] / tpeak, "traffic": traffic,
                "peak_source": peaks["source"] + ("" if tpeak == peaks["bf16_tflops"] else
                                                  " bf16 x 2 (nominal fp8 / bf16 dense ratio)")}
    return {"bound": "hbm", "kernel": dominant, "achieved": d["GB/s"], "peak": peaks["hbm_gbs"],
            "unit": "GB/s", "frac": d["GB/s"] / peaks["hbm_gbs"], "traffic": traffic,
            "peak_source": peaks["source"]}


def _timed_steps(run, steps, stream, device, world, local, step_s_estimate):
    """Exactly `steps` calls of run() between two CUDA events on the launching
    stream, barrier and synchronize on both sides, max over ranks. Identical
    steps are queued right before the first event so that the clock sampler
    sees at least CLOCK_WINDOW_S of this load; they are not timed.
    Returns (seconds, clocks)."""
    pre = int(min(100000, max(0, (CLOCK_WINDOW_S - steps * step_s_estimate) / max(step_s_estimate, 1e-7))))
    sampler = ClockSampler(local)
    sampler.start()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    _barrier(world)
    torch.cuda.synchronize(device)
    h0 = time.perf_counter()
    for _ in range(pre):
        run()
    ev0.record(stream)
    for _ in range(steps):
        run()
    ev1.record(stream)
    torch.cuda.synchronize(device)
    h1 = time.perf_counter()
    _barrier(world)
    sampler.stop()
    sec = _max_over_ranks(ev0.elapsed_time(ev1) / 1000.0, world, device)
    clocks = sampler.summary(h0, h1)
    clocks["window"] = (f"{pre} identical steps queued before the {steps} timed ones, then the timed ones "
                        f"({h1 - h0:.2f} s)")
    return sec, clocks


def measure_forward(wl, args, binding, device, world, rank, local, peaks):
    """Device throughput of dsa_forward on one workload: CUDA-graph replays of
    one forward per step, plus per-stage times and their roofline fractions.
    Returns (report, context) where context holds what the e2e and CPU legs
    reuse."""
    cpu = make_inputs(wl, seed=wl.seed + rank)
    dev = to_device(cpu, device)
    out = torch.empty((wl.B, wl.Tq, wl.Hq, wl.Dv), dtype=dev["q"].dtype, device=device)
    fargs = binding.forward_args(dev["q_idx"], dev["k_idx"], dev["w"], dev["q"], dev["k_cache"],
                                 dev["v_cache"], wl.k, wl.q_pos0, wl.scale, out=out)
    ws_bytes = binding.forward_workspace_bytes(fargs)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)

    def step():  # one dsa_forward on the current stream
        binding.forward(dev["q_idx"], dev["k_idx"], dev["w"], dev["q"], dev["k_cache"], dev["v_cache"],
                        wl.k, wl.q_pos0, wl.scale, out=out, ws=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)

    # The step is captured once in a CUDA graph; each timed step is one replay
    # (the kernels of one dsa_forward), so host launch overhead stays out of
    # the device timeline. The eager rate (one C-ABI call per step) is kept
    # as `eager` for comparison.
    graph, launches_per_step = _capture(step, binding, device)
    run = graph.replay if graph is not None else step
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.warmup):
        run()
    e1.record(stream)
    torch.cuda.synchronize(device)
    est = e0.elapsed_time(e1) / 1000.0 / max(1, args.warmup)

    launches0 = binding.kernel_launch_count()
    sec_max, clocks = _timed_steps(run, args.steps, stream, device, world, local, est)
    launches = (launches_per_step * args.steps if graph is not None
                else binding.kernel_launch_count() - launches0)
    units, unit = _units(wl, args.steps)
    value = units * world / sec_max

    # eager: the same K steps as direct C-ABI calls from Python
    _barrier(world)
    torch.cuda.synchronize(device)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(device)
    eager_sec = _max_over_ranks(e0.elapsed_time(e1) / 1000.0, world, device)
    eager = {"value": units * world / eager_sec, "unit": unit, "ms_per_step": 1000.0 * eager_sec / args.steps,
             "note": "one dsa_forward call per step from Python, no graph"}

    # per-stage timing (same stream, separate loops) for the roofline
    # the L2-served prefill gathers (large selections over a KV cache that fits
    # in L2) are also compared with the gather of the same rows alone
    kv_row = wl.Hkv * (wl.Dqk + (0 if wl.kv_alias else wl.Dv)) * (4 if wl.dtype == "f32" else 2)
    ceiling = {} if (not wl.is_decode and wl.selected_rows() * kv_row > 126e6
                     and wl.Hkv * max(wl.Dqk, wl.Dv) * (4 if wl.dtype == "f32" else 2) <= 1024) else None
    attn_info = {}
    stages = stage_timings(wl, dev, binding, stream, max(3, min(args.steps, 50)), gather_ceiling=ceiling,
                           attn_info=attn_info)
    stage_report = _stage_report(wl, stages, peaks, attn_info)
    report = {"metric": METRIC, "value": value, "unit": unit, "ms_per_step": 1000.0 * sec_max / args.steps,
              "steps": args.steps, "warmup": args.warmup, "config": _config(wl, world),
              "roofline": _roofline(wl, stage_report, peaks), "stages": stage_report,
              "gpu_launches": int(launches), "clocks": clocks, "eager": eager,
              "timing": "CUDA-graph replay of one dsa_forward per step" if graph is not None
              else "eager dsa_forward calls"}
    if ceiling:
        # prefill: the KV cache fits in L2 and every row is selected by many
        # queries, so the gathers are served by L2; the attention is compared
        # with the gather of the same rows alone
        att = report["stages"]["attn"]
        gathered = attn_info.get("gathered_rows", wl.selected_rows()) * kv_row
        gbs = gathered / (att["ms"] / 1e3) / 1e9
        att["gather"] = {"gathered_bytes": gathered, "GB/s": gbs,
                         "ceiling_GB/s": ceiling["GB/s"], "frac_of_ceiling": gbs / ceiling["GB/s"],
                         "ceiling": "builder-measured: the rate at which every query row's selected K and V rows "
                                    "are gathered into shared memory with no arithmetic (dsa_diag_gather, 16-byte "
                                    "cp.async; fastest of 8-, 16- and 32-row tiles: "
                                    f"{ceiling['tile_rows']}; {ceiling['ms']:.3f} ms for "
                                    f"{ceiling['gathered_bytes'] / 1e9:.1f} GB); gathered_bytes are the rows this "
                                    "attention fetches (the union rows of each group when rows share gathers)"}
        att["note"] = ("the gathered rows are mostly served by L2 (the KV cache is smaller than L2 and each row "
                       "is selected by many queries): hbm_frac compares them with the HBM copy rate, "
                       "gather.frac_of_ceiling with the gather alone")
    return report, {"cpu": cpu, "stream": stream}


def cpu_baseline_for(wl, cpu, budget_s, repeat: bool):
    """The oracle (all three stages) on a bounded sample of the workload's
    query rows on every host core, sized to about budget_s seconds and
    extrapolated to a whole step by the exact causal-pair count; for prefill
    half of the sample is the longest (last) rows, the other half spread
    evenly over the rest (at most 512 rows)."""
    import oracle
    oracle.build()
    nthreads = oracle.max_threads()
    _, unit = _units(wl, 1)
    prefill = wl.Tq >= 1024
    # the probe's rows are spread evenly (average cost); a sample that is half
    # last rows costs about 1.5 times as much per row in prefill
    rows = _sample_rows_for(wl, budget_s / (1.5 if prefill else 1.0), nthreads, cpu)
    if prefill:
        rows = max(16, min(512, rows))
    tail = rows // 2 if prefill else 0
    total_s, total_pairs, total_rows, reps = 0.0, 0, 0, 0
    while reps == 0 or (repeat and total_s < 0.66 * budget_s and reps < 50):
        secs, r, pairs = time_oracle(wl, cpu, rows, nthreads, tail=tail)
        total_s += secs
        total_pairs += pairs
        total_rows += r
        reps += 1
    sample = (f"{r} of {wl.B * wl.Tq} query rows"
              + (f" (the last {tail} and {r - tail} spread evenly)" if tail else "")
              + f", all three stages, {reps} repetition(s), {total_s:.1f} s in total, "
              + "extrapolated to a full step by the exact causal-pair count")
    return {"value": _oracle_rate(wl, total_s, total_pairs), "unit": unit, "cores": nthreads, "kind": "oracle",
            "sample": sample}


def run_ours(args, wl):
    from learned_sparse_attention_dsa_b200 import binding

    world, rank, local = _dist()
    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    binding.load_library()
    peaks = _peaks()

    report, ctx = measure_forward(wl, args, binding, device, world, rank, local, peaks)
    cpu = ctx["cpu"]

    # ---- end to end through the public API with host buffers
    e2e = run_e2e(wl, cpu, binding, device, ctx["stream"], max(1, min(args.steps, args.e2e_steps)), world)

    # ---- CPU baseline: the oracle on a bounded sample (rank 0, N = 1 only)
    cpu_baseline = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu_baseline = cpu_baseline_for(wl, cpu, args.cpu_budget, repeat=True)
        # the same oracle on one core, on a smaller sample of the same rows
        rows1 = _sample_rows_for(wl, args.cpu_budget / 4, 1, cpu)
        secs1, r1, pairs1 = time_oracle(wl, cpu, rows1, 1)
        cpu_baseline["single_core"] = {"value": _oracle_rate(wl, secs1, pairs1), "unit": report["unit"],
                                       "cores": 1, "sample": f"{r1} query rows, {secs1:.1f} s, extrapolated "
                                                             "to a full step"}
    del cpu, ctx
    torch.cuda.empty_cache()

    # ---- the other configurations: device throughput, per-stage roofline
    # fractions, clocks and an oracle baseline on a bounded row sample each
    workloads = {}
    extra = [] if args.workloads == "none" else (
        [w for w in EXTRA_WORKLOADS if w != wl.name] if args.workloads == "all" else args.workloads.split(","))
    for name in extra:
        xwl = WORKLOADS[name]
        xrep, xctx = measure_forward(xwl, args, binding, device, world, rank, local, peaks)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            xrep["cpu_baseline"] = cpu_baseline_for(xwl, xctx["cpu"], args.cpu_budget / 3, repeat=True)
        workloads[name] = xrep
        del xctx
        torch.cuda.empty_cache()

    if rank == 0:
        line = {
            "metric": METRIC, "value": report["value"], "unit": report["unit"], "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": report["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if wl.dtype == "bf16" else "f32", "data": "synthetic", "config": report["config"],
            "roofline": report["roofline"], "stages": report["stages"], "cpu_baseline": cpu_baseline, "e2e": e2e,
            "gpu_launches": report["gpu_launches"], "clocks": report["clocks"], "eager": report["eager"],
            "timing": report["timing"], "workloads": workloads,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


def _capture(fn, binding, device):
    """Capture fn() into a CUDA graph; returns (graph, kernels per call) or
    (None, 0) when capture is not possible."""
    side = torch.cuda.Stream(device)
    side.wait_stream(torch.cuda.current_stream(device))
    with torch.cuda.stream(side):
        fn()
    torch.cuda.current_stream(device).wait_stream(side)
    torch.cuda.synchronize(device)
    g = torch.cuda.CUDAGraph()
    n0 = binding.kernel_launch_count()
    try:
        with torch.cuda.graph(g, capture_error_mode="thread_local"):
            fn()
    except RuntimeError as exc:  # pragma: no cover - reported, eager timing used
        print(f"graph capture failed, timing eager calls: {exc}", file=sys.stderr)
        return None, 0
    return g, binding.kernel_launch_count() - n0


def stage_timings(wl, dev, binding, stream, iters, gather_ceiling=None, attn_info=None):
    """Average device time (ms) per launch of each stage: the stage call is
    captured in a CUDA graph and replayed `iters` times between CUDA events on
    the launching stream. The indexer writes the causal entries only
    (DSA_INDEXER_CAUSAL_ONLY), as the fused forward does; the top-k reads no
    other entry."""
    device = dev["q"].device
    scores = torch.empty((wl.B, wl.Tq, wl.L), dtype=torch.float32, device=device)
    idx = torch.empty((wl.B, wl.Tq, wl.k), dtype=torch.int32, device=device)
    out = torch.empty((wl.B, wl.Tq, wl.Hq, wl.Dv), dtype=dev["q"].dtype, device=device)
    sh = binding.attn_shape(dev["q"], dev["k_cache"], dev["v_cache"], wl.k, wl.scale)
    import ctypes
    ws_bytes = binding.load_library().dsa_sparse_attn_workspace_bytes(ctypes.byref(sh),
                                                                      binding._dt(dev["q"]))
    ws = torch.empty(max(int(ws_bytes), 1), dtype=torch.uint8, device=device)

    def t_of(fn):
        for _ in range(3):
            fn()
        g, _ = _capture(fn, binding, device)
        run = g.replay if g is not None else fn
        for _ in range(3):
            run()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(iters):
            run()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / iters

    res = {}
    res["indexer"] = t_of(lambda: binding.indexer_scores(dev["q_idx"], dev["k_idx"], dev["w"], wl.q_pos0,
                                                         scores=scores, causal_only=True))
    res["topk"] = t_of(lambda: binding.topk(scores, wl.k, wl.q_pos0, idx=idx))
    res["attn"] = t_of(lambda: binding.sparse_attn(dev["q"], dev["k_cache"], dev["v_cache"], idx, wl.scale,
                                                   out=out, ws=ws))
    if attn_info is not None:
        group = binding.sparse_attn_row_group(dev["q"], dev["k_cache"], dev["v_cache"], wl.k)
        attn_info["row_group"] = group
        attn_info["gathered_rows"] = union_rows(idx, group, wl.L)
    if gather_ceiling is not None and wl.B == 1:
        # the gather of the same selected K and V rows alone (dsa_diag_gather)
        sink = torch.zeros(1, dtype=torch.int32, device=device)
        kc, vc = dev["k_cache"], dev["v_cache"]
        krow, vrow = wl.Hkv * wl.Dqk * kc.element_size(), wl.Hkv * wl.Dv * vc.element_size()
        flat = idx.reshape(-1)

        def gather_kv(tile_rows):
            binding.diag_gather(kc, krow, wl.L, flat, sink, pitch_bytes=kc.stride(1) * kc.element_size(),
                                tile_rows=tile_rows)
            if not wl.kv_alias:
                binding.diag_gather(vc, vrow, wl.L, flat, sink, pitch_bytes=vc.stride(1) * vc.element_size(),
                                    tile_rows=tile_rows)

        # the fastest of three tile sizes (more CTAs per SM with smaller tiles)
        trial = {tr: t_of(lambda tr=tr: gather_kv(tr)) for tr in (8, 16, 32)}
        best = min(trial, key=trial.get)
        ms = trial[best]
        gathered = wl.selected_rows() * (krow + (0 if wl.kv_alias else vrow))
        gather_ceiling.update({"ms": ms, "GB/s": gathered / (ms / 1e3) / 1e9, "gathered_bytes": gathered,
                               "tile_rows": best, "ms_by_tile_rows": trial})
    return res


def run_e2e(wl, cpu, binding, device, stream, steps, world):
    """Same metric through dsa_forward with inputs in pinned host memory:
    every step copies all of its inputs host->device and reads the output
    back device->host inside the timed region."""
    host = {k: v.contiguous().pin_memory() for k, v in cpu.items() if k != "v_cache"}
    if not wl.kv_alias:
        host["v_cache"] = cpu["v_cache"].contiguous().pin_memory()
    dev = {k: torch.empty_like(v, device=device) for k, v in host.items()}
    v_dev = dev["k_cache"][..., : wl.Dv] if wl.kv_alias else dev["v_cache"]
    out = torch.empty((wl.B, wl.Tq, wl.Hq, wl.Dv), dtype=dev["q"].dtype, device=device)
    out_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    fargs = binding.forward_args(dev["q_idx"], dev["k_idx"], dev["w"], dev["q"], dev["k_cache"], v_dev,
                                 wl.k, wl.q_pos0, wl.scale, out=out)
    ws = torch.empty(max(binding.forward_workspace_bytes(fargs), 1), dtype=torch.uint8, device=device)
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = out.numel() * out.element_size()

    def step():
        for k2, v in host.items():
            dev[k2].copy_(v, non_blocking=True)
        binding.forward(dev["q_idx"], dev["k_idx"], dev["w"], dev["q"], dev["k_cache"], v_dev, wl.k,
                        wl.q_pos0, wl.scale, out=out, ws=ws, stream=stream)
        out_host.copy_(out, non_blocking=True)

    for _ in range(2):
        step()
    _barrier(world)
    torch.cuda.synchronize(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(device)
    sec = _max_over_ranks(e0.elapsed_time(e1) / 1000.0, world, device)
    units, unit = _units(wl, steps)
    return {"value": units * world / sec, "unit": unit, "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "steps": steps,
            "note": "all step inputs copied from pinned host memory, output read back, every step"}


def run_stage(args, wl):
    """Eager launches of one stage only (for profiler captures): W warm-up
    calls then K timed calls; prints the average device time per call.
    --tail-rows R keeps only the last R query rows of the workload (a small
    case of the same kernel for full profiler captures)."""
    from learned_sparse_attention_dsa_b200 import binding
    if args.tail_rows:
        R = min(args.tail_rows, wl.Tq)
        wl = wl.replace(name=f"{wl.name}_tail{R}", Tq=R, q_pos0=wl.q_pos0 + wl.Tq - R)
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    dev = to_device(make_inputs(wl), device)
    scores = torch.empty((wl.B, wl.Tq, wl.L), dtype=torch.float32, device=device)
    idx = torch.empty((wl.B, wl.Tq, wl.k), dtype=torch.int32, device=device)
    out = torch.empty((wl.B, wl.Tq, wl.Hq, wl.Dv), dtype=dev["q"].dtype, device=device)
    binding.indexer_scores(dev["q_idx"], dev["k_idx"], dev["w"], wl.q_pos0, scores=scores, causal_only=True)
    binding.topk(scores, wl.k, wl.q_pos0, idx=idx)
    calls = {
        "indexer": lambda: binding.indexer_scores(dev["q_idx"], dev["k_idx"], dev["w"], wl.q_pos0,
                                                  scores=scores, causal_only=True),
        "topk": lambda: binding.topk(scores, wl.k, wl.q_pos0, idx=idx),
        "attn": lambda: binding.sparse_attn(dev["q"], dev["k_cache"], dev["v_cache"], idx, wl.scale, out=out),
    }
    fn = calls[args.stage]
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    print(json.dumps({"stage": args.stage, "workload": wl.name, "calls": args.steps,
                      "ms_per_call": e0.elapsed_time(e1) / args.steps}))


# ------------------------------------------------------------------ training side

TRAIN_METRIC = ("indexer training tokens/s (scores, dense KL loss and backward); "
                "% tensor/HBM roofline per stage")


def train_work(wl):
    """Algorithmic bytes and flops per training step, per stage.

    scores:   as the forward indexer stage (2 H d flops per causal pair).
    kl:       reads one fp32 score and one fp32 target weight per causal pair,
              writes the fp32 gradient of every (row, key) entry (zeros above
              the diagonal) and one loss per row.
    backward: two products per side (x recomputed, then G times the other
              operand) on the query side (dq, dw) and on the key side (dk):
              8 H d flops per causal pair; reads q, k, w and one fp32
              gradient per causal pair, writes dq, dk, dw in fp32.
    """
    rows = wl.B * wl.Tq
    pairs = wl.causal_pairs()
    eb = 2
    idx_bytes = (wl.B * wl.L * wl.d_I * eb + rows * wl.H_I * wl.d_I * eb + rows * wl.H_I * 4 + pairs * 4)
    kl_bytes = pairs * 8 + rows * wl.L * 4 + rows * 4
    bwd_bytes = (wl.B * wl.L * wl.d_I * eb + rows * wl.H_I * wl.d_I * eb + rows * wl.H_I * 4 + pairs * 4
                 + rows * wl.H_I * wl.d_I * 4 + wl.B * wl.L * wl.d_I * 4 + rows * wl.H_I * 4)
    return {"scores": (idx_bytes, 2.0 * wl.H_I * wl.d_I * pairs), "kl": (kl_bytes, 0.0),
            "backward": (bwd_bytes, 8.0 * wl.H_I * wl.d_I * pairs)}


def _train_buffers(wl, dev, binding):
    device = dev["q_idx"].device
    f32 = dict(dtype=torch.float32, device=device)
    bufs = {
        "scores": torch.empty((wl.B, wl.Tq, wl.L), **f32),
        "grad": torch.empty((wl.B, wl.Tq, wl.L), **f32),
        "loss_rows": torch.empty(wl.B * wl.Tq, **f32),
        "loss_sum": torch.empty(1, **f32),
        "dq": torch.empty((wl.B, wl.Tq, wl.H_I, wl.d_I), **f32),
        "dk": torch.empty((wl.B, wl.L, wl.d_I), **f32),
        "dw": torch.empty((wl.B, wl.Tq, wl.H_I), **f32),
    }
    nbytes = binding.indexer_backward_workspace_bytes(dev["q_idx"], dev["k_idx"], wl.q_pos0)
    bufs["ws"] = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=device)
    return bufs


def _train_calls(wl, dev, target, bufs, binding):
    def scores():
        binding.indexer_scores(dev["q_idx"], dev["k_idx"], dev["w"], wl.q_pos0, scores=bufs["scores"])

    def kl():
        binding.indexer_kl(bufs["scores"], target, wl.q_pos0, loss_rows=bufs["loss_rows"],
                           loss_sum=bufs["loss_sum"], grad=bufs["grad"])

    def backward():
        binding.indexer_backward(dev["q_idx"], dev["k_idx"], dev["w"], bufs["grad"], wl.q_pos0, dq=bufs["dq"],
                                 dk=bufs["dk"], dw=bufs["dw"], ws=bufs["ws"])

    return {"scores": scores, "kl": kl, "backward": backward}


def time_train_oracle(wl, cpu, target, n_rows: int, nthreads: int = 0):
    """The oracle on a sample: scores, loss and dq/dw of n_rows query rows,
    dk of n_rows keys (rows and keys spread evenly). Returns (seconds, rows,
    keys); a full step is rows_total / rows times the row part plus
    keys_total / keys times the key part, both already in the seconds."""
    import oracle
    from oracle import kl as okl


    total = wl.B * wl.Tq
    flat = np.linspace(0, total - 1, num=min(n_rows, total)).round().astype(np.int64)
    rb, ri = (flat // wl.Tq).astype(np.int32), (flat % wl.Tq).astype(np.int32)
    rt = ri + wl.q_pos0
    q_all, k_all, w_all = bits(cpu["q_idx"]), bits(cpu["k_idx"]), cpu["w"].numpy()
    tg = target.numpy()
    t0 = time.perf_counter()
    sc = oracle.indexer_rows(q_all[rb, ri], w_all[rb, ri], k_all, rb, rt, nthreads)
    _, g = okl.kl_rows(sc, tg[rb, ri], rt)
    grad = np.zeros((wl.B, wl.Tq, wl.L), dtype=np.float64) if total * wl.L <= 1 << 26 else None
    if grad is not None:
        grad[rb, ri] = g
        okl.indexer_backward_rows(q_all, k_all, w_all, grad, rb, rt, ri)
    t_rows = time.perf_counter() - t0
    # key part: dk of sampled keys needs g[t, s] for every t >= s of those keys
    keys = np.linspace(0, wl.B * wl.L - 1, num=min(n_rows, wl.B * wl.L)).round().astype(np.int64)
    kb, ks = keys // wl.L, keys % wl.L
    t1 = time.perf_counter()
    gk = np.zeros((wl.B, wl.Tq, wl.L), dtype=np.float64) if total * wl.L <= 1 << 26 else None
    if gk is not None:
        okl.indexer_backward_keys(q_all, k_all, w_all, gk, kb, ks, wl.q_pos0)
    t_keys = time.perf_counter() - t1
    sec = t_rows * total / len(flat) + t_keys * (wl.B * wl.L) / len(keys)
    return sec, len(flat), len(keys), t_rows + t_keys


def run_train(args, wl):
    from learned_sparse_attention_dsa_b200 import binding
    from learned_sparse_attention_dsa_b200.inputs import target_weights

    world, rank, local = _dist()
    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    binding.load_library()
    cpu = make_inputs(wl, seed=wl.seed + rank)
    target_cpu = target_weights(torch.Generator().manual_seed(wl.seed + 7 + rank), (wl.B, wl.Tq, wl.L))
    dev = to_device(cpu, device)
    target = target_cpu.to(device)
    bufs = _train_buffers(wl, dev, binding)
    calls = _train_calls(wl, dev, target, bufs, binding)
    stream = torch.cuda.current_stream(device)

    def step():
        calls["scores"]()
        calls["kl"]()
        calls["backward"]()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    graph, launches_per_step = _capture(step, binding, device)
    run = graph.replay if graph is not None else step
    for _ in range(args.warmup):
        run()
    torch.cuda.synchronize(device)

    sampler = ClockSampler(local)
    sampler.start()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    _barrier(world)
    torch.cuda.synchronize(device)
    launches0 = binding.kernel_launch_count()
    h0 = time.perf_counter()
    ev0.record(stream)
    for _ in range(args.steps):
        run()
    ev1.record(stream)
    torch.cuda.synchronize(device)
    h1 = time.perf_counter()
    launches = (launches_per_step * args.steps if graph is not None
                else binding.kernel_launch_count() - launches0)
    _barrier(world)
    sampler.stop()
    sec_max = _max_over_ranks(ev0.elapsed_time(ev1) / 1000.0, world, device)
    units = float(args.steps * wl.B * wl.Tq)
    unit = "training tokens/s"
    value = units * world / sec_max
    clocks = sampler.summary(h0, h1)

    # ---- per-stage timing for the roofline (graph replays, launching stream)
    peaks = _peaks()
    work = train_work(wl)
    iters = max(3, min(args.steps, 20))
    stage_report = {}
    for name, fn in calls.items():
        g, _ = _capture(fn, binding, device)
        r = g.replay if g is not None else fn
        for _ in range(3):
            r()
        torch.cuda.synchronize(device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(iters):
            r()
        e1.record(stream)
        torch.cuda.synchronize(device)
        ms = e0.elapsed_time(e1) / iters
        nbytes, flops = work[name]
        entry = {"ms": ms, "GB/s": nbytes / (ms / 1e3) / 1e9, "algorithmic_bytes": nbytes,
                 "algorithmic_flops": flops}
        entry["hbm_frac"] = entry["GB/s"] / peaks["hbm_gbs"]
        if flops:
            entry["TFLOP/s"] = flops / (ms / 1e3) / 1e12
            entry["tensor_frac"] = entry["TFLOP/s"] / peaks["bf16_tflops"]
        stage_report[name] = entry
    dominant = max(stage_report, key=lambda n: stage_report[n]["ms"])
    d = stage_report[dominant]
    if d["algorithmic_flops"]:
        roofline = {"bound": "tensor", "kernel": dominant, "achieved": d["TFLOP/s"], "peak": peaks["bf16_tflops"],
                    "unit": "TFLOP/s", "frac": d["tensor_frac"], "traffic": None, "peak_source": peaks["source"]}
    else:
        roofline = {"bound": "hbm", "kernel": dominant, "achieved": d["GB/s"], "peak": peaks["hbm_gbs"],
                    "unit": "GB/s", "frac": d["hbm_frac"], "traffic": None, "peak_source": peaks["source"]}

    # ---- end to end: inputs and target from pinned host memory, loss read back
    host = {"q_idx": cpu["q_idx"].contiguous().pin_memory(), "k_idx": cpu["k_idx"].contiguous().pin_memory(),
            "w": cpu["w"].contiguous().pin_memory(), "target": target_cpu.contiguous().pin_memory()}
    dst = {"q_idx": dev["q_idx"], "k_idx": dev["k_idx"], "w": dev["w"], "target": target}
    loss_host = torch.empty(1, dtype=torch.float32).pin_memory()
    e2e_steps = max(1, min(args.steps, args.e2e_steps))

    def e2e_step():
        for k2, v in host.items():
            dst[k2].copy_(v, non_blocking=True)
        step()
        loss_host.copy_(bufs["loss_sum"], non_blocking=True)

    e2e_step()
    _barrier(world)
    torch.cuda.synchronize(device)
    ev0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    ev1.record(stream)
    torch.cuda.synchronize(device)
    e2e_sec = _max_over_ranks(ev0.elapsed_time(ev1) / 1000.0, world, device)
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    e2e = {"value": e2e_steps * wl.B * wl.Tq * world / e2e_sec, "unit": unit, "h2d_bytes_per_step": int(h2d),
           "d2h_bytes_per_step": 4, "steps": e2e_steps,
           "note": "indexer inputs and the target copied from pinned host memory, the summed loss read back, "
                   "every step"}

    cpu_baseline = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        nthreads = oracle.max_threads()
        _, _, _, probe = time_train_oracle(wl, cpu, target_cpu, 4, nthreads)
        n = int(min(256, max(4, 4 * args.cpu_budget / max(probe, 1e-6))))
        sec, r, k, _ = time_train_oracle(wl, cpu, target_cpu, n, nthreads)
        cpu_baseline = {"value": wl.B * wl.Tq / sec, "unit": unit, "cores": nthreads, "kind": "oracle",
                        "sample": f"{r} query rows (scores, loss, dq, dw) and {k} keys (dk), scaled to a full "
                                  f"step ({sec:.1f} s extrapolated)"}

    if rank == 0:
        line = {
            "metric": TRAIN_METRIC, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1000.0 * sec_max / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": dict(_config(wl, world), **{"pass": "train", "target": "log-normal weights, 10% zeros"}),
            "roofline": roofline, "stages": stage_report, "cpu_baseline": cpu_baseline, "e2e": e2e,
            "gpu_launches": int(launches), "clocks": clocks,
            "timing": "CUDA-graph replay of one training step" if graph is not None else "eager calls",
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


# ------------------------------------------------------------------ context parallelism

def run_cp(args, wl):
    """The context-parallel decode step with its P shards emulated one after
    another on one GPU: every shard's indexer, top-k and candidate gather,
    the merge, every shard's attention over its part of the selection, and
    the log-sum-exp combine. Each shard writes into its slot of the buffers an
    all-gather would fill, so the step runs the library's kernels only (no
    collective: one GPU)."""
    from learned_sparse_attention_dsa_b200 import binding

    world, rank, _ = _dist()
    if world > 1:
        raise SystemExit("--pass cp emulates the shards on one GPU; run it with --gpus 1")
    if not wl.is_decode:
        raise SystemExit("--pass cp is a decode step (one query row per batch entry)")
    P = args.shards
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    binding.load_library()
    cpu = make_inputs(wl)
    dev = to_device(cpu, device)
    step_len = -(-wl.L // P)
    bounds = [(a, min(wl.L, a + step_len)) for a in range(0, wl.L, step_len)]
    P = len(bounds)
    shards = []
    for a, b in bounds:
        kc = dev["k_cache"][:, a:b].contiguous()
        shards.append({"a": a, "L": b - a, "k_idx": dev["k_idx"][:, a:b].contiguous(), "k": kc,
                       "v": kc[..., : wl.Dv] if wl.kv_alias else dev["v_cache"][:, a:b].contiguous(),
                       "scores": torch.empty((wl.B, 1, b - a), dtype=torch.float32, device=device),
                       "idx": torch.empty((wl.B, 1, wl.k), dtype=torch.int32, device=device),
                       "idx_local": torch.empty((wl.B, 1, wl.k), dtype=torch.int32, device=device)})
    del dev["k_cache"], dev["v_cache"], dev["k_idx"]
    f32 = dict(dtype=torch.float32, device=device)
    cand_s = torch.empty((P, wl.B, 1, wl.k), **f32)
    cand_i = torch.empty((P, wl.B, 1, wl.k), dtype=torch.int32, device=device)
    idx = torch.empty((wl.B, 1, wl.k), dtype=torch.int32, device=device)
    parts = torch.empty((P, wl.B, 1, wl.Hq, wl.Dv), dtype=dev["q"].dtype, device=device)
    lses = torch.empty((P, wl.B, 1, wl.Hq), **f32)
    out = torch.empty((wl.B, 1, wl.Hq, wl.Dv), dtype=dev["q"].dtype, device=device)
    t = wl.L - 1

    def step():
        for r, sh in enumerate(shards):
            q0 = min(t - sh["a"], sh["L"] - 1)
            binding.indexer_scores(dev["q_idx"], sh["k_idx"], dev["w"], q0, scores=sh["scores"])
            binding.topk(sh["scores"], wl.k, q0, idx=sh["idx"])
            binding.cp_select_candidates(sh["scores"], sh["idx"], sh["a"], cand_scores=cand_s[r],
                                         cand_idx=cand_i[r])
        binding.cp_merge(cand_s, cand_i, wl.k, idx=idx)
        for r, sh in enumerate(shards):
            binding.cp_localize(idx, sh["a"], sh["L"], out=sh["idx_local"])
            binding.sparse_attn(dev["q"], sh["k"], sh["v"], sh["idx_local"], wl.scale, out=parts[r], lse=lses[r])
        binding.cp_combine(parts, lses, out=out)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    graph, launches_per_step = _capture(step, binding, device)
    run = graph.replay if graph is not None else step
    for _ in range(args.warmup):
        run()
    stream = torch.cuda.current_stream(device)
    sampler = ClockSampler(0)
    sampler.start()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(device)
    h0 = time.perf_counter()
    ev0.record(stream)
    for _ in range(args.steps):
        run()
    ev1.record(stream)
    torch.cuda.synchronize(device)
    h1 = time.perf_counter()
    sampler.stop()
    sec = ev0.elapsed_time(ev1) / 1000.0
    line = {
        "metric": "context-parallel decode steps/s (shards emulated on one GPU)", "value": args.steps / sec,
        "unit": "decode steps/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * sec / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(_config(wl, 1), **{"pass": "cp", "shards": P, "shard_len": step_len}),
        "gpu_launches": int(launches_per_step * args.steps) if graph is not None else None,
        "clocks": sampler.summary(h0, h1),
        "timing": "CUDA-graph replay of one emulated step" if graph is not None else "eager calls",
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--stage", choices=["indexer", "topk", "attn"], default=None,
                    help="launch only this stage (profiler captures); prints its time")
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default=None, choices=sorted(WORKLOADS),
                    help="default: decode32k (forward), prefill8k (train)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--workloads", default="all",
                    help="other configurations reported under \"workloads\": all (default), none, or a "
                         "comma-separated list of names")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle wall time")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--pass", dest="pass_", default="forward", choices=["forward", "train", "cp"],
                    help="train: indexer scores, dense KL loss and indexer backward per step; "
                         "cp: the context-parallel decode step with its shards emulated on one GPU")
    ap.add_argument("--shards", type=int, default=8, help="--pass cp: number of context shards")
    ap.add_argument("--tail-rows", type=int, default=0,
                    help="--stage: keep only the last R query rows (small profiler cases)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)  # at least three untimed warm-up steps
    if args.workload is None:
        args.workload = "prefill8k" if args.pass_ == "train" else "decode32k"
    wl = WORKLOADS[args.workload]
    if args.pass_ == "train" and args.impl == "ours" and args.stage is None:
        run_train(args, wl)
    elif args.pass_ == "cp" and args.impl == "ours" and args.stage is None:
        run_cp(args, wl)
    elif args.stage is not None:
        run_stage(args, wl)
    elif args.impl == "reference":
        run_reference(args, wl)
    else:
        run_ours(args, wl)


if __name__ == "__main__":
    main()
