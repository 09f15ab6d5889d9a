"""Seeded synthetic inputs for the DSA forward path.

This module holds no arithmetic of the method: it only draws random tensors
with the shapes and value distributions of the workloads, so that the CUDA
path and the CPU oracle can be fed identical data. Both sides receive the
tensors it returns; neither side's arithmetic lives here.

Value recipes (the pages fix the indexer inputs to small integers and the
weights to powers of two so that every score is exact in fp32):
  toy16       n=16 worked-example scale ("DeepSeek Sparse Attention: Learned
              Token Selection from Scratch", running example): q^I, k^I
              integers uniform in [-4, 4] as fp32, w in {0.5, 1, 2}; Q/K/V
              N(0, 1) fp32; H^I=2, d^I=2, k=3, 8 heads of width 64.
  decode32k   decode step, 32 sequences, context 32,768: q^I, k^I integers
              uniform in [-8, 8] as bf16, w = +-2^j with j uniform in
              {-3..0}; Q/K/V N(0, 1) bf16; 16 query heads over one KV head,
              width 128.
  prefill8k   prefill of 8,192 tokens; indexer as decode32k; 8 heads of width
              64, one KV head per query head.
  prefill32k  prefill of 32,768 tokens; indexer as decode32k; 16 query heads
              over one latent KV head, QK width 192, V width 128.
  decode128k  decode step, 8 sequences, context 131,072; indexer as
              decode32k; 128 query heads over one 576-wide latent row whose
              first 512 columns are also the value.
The indexer shape H^I=64, d^I=128 and the budget k=2048 are the public
configuration values quoted on "DeepSeek NSA and DSA" §3.2.
"""
from __future__ import annotations

import dataclasses
import math
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Tq: int
    L: int
    q_pos0: int
    H_I: int
    d_I: int
    k: int
    Hq: int
    Hkv: int
    Dqk: int
    Dv: int
    dtype: str = "bf16"        # "f32" or "bf16" for q^I/k^I and Q/K/V
    idx_range: int = 8         # indexer integers uniform in [-idx_range, idx_range]
    w_kind: str = "pow2"       # "pow2": +-2^j, j in -3..0; "set": {0.5, 1, 2}
    kv_alias: bool = False     # V = first Dv columns of each K row
    idx_dtype: str = ""        # q^I/k^I storage: "" = as dtype, "e4m3" = 8-bit FP8 codes
    seed: int = 1234

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.Dqk)

    @property
    def is_decode(self) -> bool:
        return self.Tq == 1

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    def selected_rows(self) -> int:
        """sum over query rows of min(t+1, k): KV rows the attention reads."""
        total = 0
        for i in range(self.Tq):
            total += min(self.q_pos0 + i + 1, self.k)
        return total * self.B

    def causal_pairs(self) -> int:
        """sum over query rows of (t+1): indexer (query, key) pairs."""
        t0 = self.q_pos0
        t1 = self.q_pos0 + self.Tq - 1
        return self.B * ((t1 + 1) * (t1 + 2) // 2 - t0 * (t0 + 1) // 2)


WORKLOADS = {
    "toy16": Workload("toy16", B=1, Tq=16, L=16, q_pos0=0, H_I=2, d_I=2, k=3,
                      Hq=8, Hkv=8, Dqk=64, Dv=64, dtype="f32", idx_range=4,
                      w_kind="set", seed=1235),
    "decode32k": Workload("decode32k", B=32, Tq=1, L=32768, q_pos0=32767, H_I=64,
                          d_I=128, k=2048, Hq=16, Hkv=1, Dqk=128, Dv=128, seed=1236),
    "prefill8k": Workload("prefill8k", B=1, Tq=8192, L=8192, q_pos0=0, H_I=64,
                          d_I=128, k=2048, Hq=8, Hkv=8, Dqk=64, Dv=64, seed=1237),
    "prefill32k": Workload("prefill32k", B=1, Tq=32768, L=32768, q_pos0=0, H_I=64,
                           d_I=128, k=2048, Hq=16, Hkv=1, Dqk=192, Dv=128, seed=1238),
    "decode128k": Workload("decode128k", B=8, Tq=1, L=131072, q_pos0=131071, H_I=64,
                           d_I=128, k=2048, Hq=128, Hkv=1, Dqk=576, Dv=512,
                           kv_alias=True, seed=1239),
    # a context no longer than the budget: every row keeps all of its
    # candidates, so the forward skips the indexer and the top-k
    # decode32k with the indexer inputs in e4m3 (half the key bytes)
    "decode32k_fp8": Workload("decode32k_fp8", B=32, Tq=1, L=32768, q_pos0=32767, H_I=64,
                              d_I=128, k=2048, Hq=16, Hkv=1, Dqk=128, Dv=128, idx_dtype="e4m3", seed=1236),
    "prefill2k": Workload("prefill2k", B=1, Tq=2048, L=2048, q_pos0=0, H_I=64,
                          d_I=128, k=2048, Hq=16, Hkv=1, Dqk=192, Dv=128, seed=1240),
}


def _dtype(wl: Workload) -> torch.dtype:
    return torch.float32 if wl.dtype == "f32" else torch.bfloat16


def _ints(gen, shape, r, dtype, chunk_dim0=True):
    out = torch.empty(shape, dtype=dtype)
    if chunk_dim0 and len(shape) > 1:
        for i in range(shape[0]):
            out[i] = torch.randint(-r, r + 1, shape[1:], generator=gen, dtype=torch.int16).to(dtype)
    else:
        out.copy_(torch.randint(-r, r + 1, shape, generator=gen, dtype=torch.int16).to(dtype))
    return out


def _normal(gen, shape, dtype):
    out = torch.empty(shape, dtype=dtype)
    for i in range(shape[0]):
        out[i] = torch.randn(shape[1:], generator=gen, dtype=torch.float32).to(dtype)
    return out


def _weights(gen, shape, kind):
    if kind == "set":
        table = torch.tensor([0.5, 1.0, 2.0], dtype=torch.float32)
        return table[torch.randint(0, 3, shape, generator=gen)]
    if kind == "pow2":
        j = torch.randint(-3, 1, shape, generator=gen).to(torch.float32)
        sign = torch.randint(0, 2, shape, generator=gen).to(torch.float32) * 2.0 - 1.0
        return sign * torch.pow(2.0, j)
    raise ValueError(kind)


def make_inputs(wl: Workload, seed: int | None = None) -> dict:
    """Draw every input tensor of one forward pass on the CPU.

    Keys: q_idx [B,Tq,H_I,d_I], k_idx [B,L,d_I], w [B,Tq,H_I] fp32,
    q [B,Tq,Hq,Dqk], k_cache [B,L,Hkv,Dqk], v_cache [B,L,Hkv,Dv]
    (for kv_alias workloads v_cache is a strided view of k_cache).
    """
    gen = torch.Generator().manual_seed(wl.seed if seed is None else seed)
    dt = _dtype(wl)
    q_idx = _ints(gen, (wl.B, wl.Tq, wl.H_I, wl.d_I), wl.idx_range, dt)
    k_idx = _ints(gen, (wl.B, wl.L, wl.d_I), wl.idx_range, dt)
    if wl.idx_dtype == "e4m3":  # the same integers, exact in e4m3 up to 16
        q_idx = q_idx.to(torch.float8_e4m3fn)
        k_idx = k_idx.to(torch.float8_e4m3fn)
    w = _weights(gen, (wl.B, wl.Tq, wl.H_I), wl.w_kind)
    q = _normal(gen, (wl.B, wl.Tq, wl.Hq, wl.Dqk), dt)
    k_cache = _normal(gen, (wl.B, wl.L, wl.Hkv, wl.Dqk), dt)
    if wl.kv_alias:
        if wl.Dv > wl.Dqk:
            raise ValueError("kv_alias needs Dv <= Dqk")
        v_cache = k_cache[..., : wl.Dv]
    else:
        v_cache = _normal(gen, (wl.B, wl.L, wl.Hkv, wl.Dv), dt)
    return dict(q_idx=q_idx, k_idx=k_idx, w=w, q=q, k_cache=k_cache, v_cache=v_cache)


def to_device(inputs: dict, device) -> dict:
    """Copy a make_inputs() dict to a device, keeping the K/V alias."""
    out = {}
    for key in ("q_idx", "k_idx", "w", "q", "k_cache"):
        out[key] = inputs[key].to(device)
    v = inputs["v_cache"]
    if v.data_ptr() == inputs["k_cache"].data_ptr() and v.shape != inputs["k_cache"].shape:
        out["v_cache"] = out["k_cache"][..., : v.shape[-1]]
    else:
        out["v_cache"] = v.to(device)
    return out


def target_weights(gen: torch.Generator, shape, sigma: float = 2.0, zero_frac: float = 0.1) -> torch.Tensor:
    """Non-negative fp32 target weights a[t, s] for the indexer's training
    loss: log-normal exp(sigma * N(0, 1)), a peaked spread like that of
    attention weights summed over heads, with a fraction of exact zeros.
    The loss normalises them itself."""
    a = torch.exp(sigma * torch.randn(shape, generator=gen, dtype=torch.float32))
    a[torch.rand(shape, generator=gen) < zero_frac] = 0.0
    return a


def random_score_rows(gen: torch.Generator, n_rows: int, L: int, kind: str) -> torch.Tensor:
    """fp32 score rows for exercising the selector on its own.

    kind: "int" small integers (heavy ties), "equal" all equal,
    "normal" continuous, "neg" non-positive integers, "mixed" a mix of
    exact duplicates, -0.0/+0.0 and -inf entries.
    """
    if kind == "int":
        return torch.randint(-6, 7, (n_rows, L), generator=gen).to(torch.float32)
    if kind == "equal":
        return torch.full((n_rows, L), 1.5, dtype=torch.float32)
    if kind == "normal":
        return torch.randn((n_rows, L), generator=gen, dtype=torch.float32)
    if kind == "neg":
        return -torch.randint(0, 40, (n_rows, L), generator=gen).to(torch.float32)
    if kind == "mixed":
        base = torch.randint(-3, 4, (n_rows, L), generator=gen).to(torch.float32) * 0.125
        pick = torch.randint(0, 10, (n_rows, L), generator=gen)
        base[pick == 0] = -0.0
        base[pick == 1] = float("-inf")
        base[pick == 2] = 1.0e30
        return base
    raise ValueError(kind)
