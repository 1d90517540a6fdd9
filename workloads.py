"""Seeded synthetic inputs for the Gated DeltaNet mixer workloads.

This module draws random inputs and nothing else: it holds none of the
mixer's arithmetic, so that both the CUDA path and the fp64 oracle can be
fed the very same bits. Inputs are drawn on the CPU with ``torch.Generator``
(fp32 normals rounded to bf16 by round-to-nearest-even where the workload is
bf16); gates are drawn in fp64 and rounded once to fp32.

Gate convention: the decay alpha = sigmoid(x), x ~ N(3, 1), is passed as its
logarithm g = log(alpha) (fp32, <= 0); the update strength beta = sigmoid(y),
y ~ N(0, 1), is passed as is (fp32). Both are per token per value head.

Workloads (sizes of a Qwen3.5-style hybrid model's linear-attention layers):

  tiny        1 sequence, T=64, 2 q/k heads and 2 v heads, d_k=d_v=16, fp32 I/O,
              chunk 16, zero initial state
  prefill     1 sequence, T=4096, 16 q/k and 16 v heads, d=128, bf16, chunk 64,
              zero initial state (a 0.8B-class layer)
  decode      64 sequences, one token each, 16 q/k and 32 v heads, d=128, bf16,
              fp32 state ~ N(0, 0.05^2), run for 1000 consecutive steps
  long        1 sequence, T=32768 (and 81920), 16 q/k and 32 v heads, d=128,
              bf16, zero initial state
  varlen      8 sequences, lengths uniform in [128, 8192], packed token-major,
              16 q/k and 32 v heads, d=128, bf16, per-sequence fp32 initial
              states ~ N(0, 0.05^2)
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

# seeds: workload i uses 1000+i for tokens and 2000+i for states; decode step s
# uses 3_000_000+s; varlen lengths use 5005.
SEED_TOKENS = 1000
SEED_STATES = 2000
SEED_DECODE_STEP = 3_000_000
SEED_VARLEN_LENGTHS = 5005


@dataclass
class Workload:
    name: str
    index: int                 # 0..4, fixes the seeds
    kind: str                  # "prefill" or "decode"
    lengths: list = field(default_factory=list)   # prefill: tokens per sequence
    batch: int = 0             # decode: sequences
    steps: int = 0             # decode: consecutive steps
    Hqk: int = 16
    Hv: int = 16
    d: int = 128
    dtype: str = "bf16"        # dtype of q, k, v, o ("bf16", "f16" or "f32")
    chunk: int = 64
    state_std: float = 0.0     # 0 => zero initial state
    tol_o: float = 2e-2        # max abs error vs the fp64 oracle
    tol_state: float = 1e-2

    @property
    def total_tokens(self) -> int:
        return sum(self.lengths)

    @property
    def torch_dtype(self):
        return {"bf16": torch.bfloat16, "f16": torch.float16, "f32": torch.float32}[self.dtype]


def varlen_lengths(n: int = 8, lo: int = 128, hi: int = 8192, seed: int = SEED_VARLEN_LENGTHS):
    g = torch.Generator().manual_seed(seed)
    return [int(x) for x in torch.randint(lo, hi + 1, (n,), generator=g)]


def workload(name: str, T: int | None = None, dtype: str | None = None) -> Workload:
    """The named workload; ``T`` overrides the length of single-sequence prefill
    and ``dtype`` the input type of a 16-bit workload ("f16": the same draws
    rounded to IEEE half instead of bfloat16)."""
    w = _workload(name, T)
    if dtype is not None:
        w.dtype = dtype
    return w


def _workload(name: str, T: int | None = None) -> Workload:
    if name == "tiny":
        return Workload("tiny", 0, "prefill", lengths=[64], Hqk=2, Hv=2, d=16,
                        dtype="f32", chunk=16, tol_o=1e-4, tol_state=1e-4)
    if name == "prefill":
        return Workload("prefill", 1, "prefill", lengths=[T or 4096], Hqk=16, Hv=16)
    if name == "decode":
        return Workload("decode", 2, "decode", batch=64, steps=1000, Hqk=16, Hv=32,
                        state_std=0.05)
    if name == "long":
        return Workload("long", 3, "prefill", lengths=[T or 32768], Hqk=16, Hv=32,
                        tol_o=3e-2, tol_state=2e-2)
    if name == "varlen":
        return Workload("varlen", 4, "prefill", lengths=varlen_lengths(), Hqk=16, Hv=32,
                        state_std=0.05)
    raise KeyError(name)


ALL = ("tiny", "prefill", "decode", "long", "varlen")


def _gates(gen: torch.Generator, shape):
    x = torch.randn(shape, generator=gen, dtype=torch.float64) + 3.0
    y = torch.randn(shape, generator=gen, dtype=torch.float64)
    g = torch.nn.functional.logsigmoid(x).to(torch.float32)
    beta = torch.sigmoid(y).to(torch.float32)
    return g, beta


def log_sigmoid_gates(gen: torch.Generator, shape, mean: float, std: float):
    """g = log sigmoid(x), x ~ N(mean, std^2) drawn in fp64, rounded once to fp32
    (mean 3, std 1 is the workloads' own decay; negative means decay strongly)."""
    x = torch.randn(shape, generator=gen, dtype=torch.float64) * std + mean
    return torch.nn.functional.logsigmoid(x).to(torch.float32)


def shifted_log_decay(gen: torch.Generator, shape, mean: float, std: float):
    """g ~ N(mean, std^2) drawn in fp64, rounded once to fp32 (no sigmoid: with a
    mean of -5 every token decays the state by about e^-5)."""
    return (torch.randn(shape, generator=gen, dtype=torch.float64) * std + mean).to(torch.float32)


def prefill_inputs(lengths, Hqk, Hv, d, dtype=torch.bfloat16, seed=SEED_TOKENS + 1,
                   state_std=0.0, state_seed=None, dv=None):
    """Packed prefill inputs on the CPU.

    Returns dict(q, k, v [T, H, d] in ``dtype``; g, beta [T, Hv] fp32;
    cu_seqlens [N+1] int32; state_in [N, Hv, dv, d] fp32 or None).
    """
    dv = dv or d
    T = int(sum(lengths))
    gen = torch.Generator().manual_seed(seed)
    q = torch.randn(T, Hqk, d, generator=gen).to(dtype)
    k = torch.randn(T, Hqk, d, generator=gen).to(dtype)
    v = torch.randn(T, Hv, dv, generator=gen).to(dtype)
    g, beta = _gates(gen, (T, Hv))
    cu = torch.zeros(len(lengths) + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(torch.tensor(lengths, dtype=torch.int64), 0).to(torch.int32)
    state = None
    if state_std > 0:
        sg = torch.Generator().manual_seed(state_seed if state_seed is not None else seed + 1000)
        state = torch.randn(len(lengths), Hv, dv, d, generator=sg) * state_std
    return dict(q=q, k=k, v=v, g=g, beta=beta, cu_seqlens=cu, state_in=state)


def decode_step_inputs(step, B, Hqk, Hv, d, dtype=torch.bfloat16, dv=None):
    """Inputs of decode step ``step`` (fresh seeded tokens each step); q, k, v
    are drawn in fp32 and rounded to ``dtype`` (bf16, f16, or kept fp32)."""
    dv = dv or d
    gen = torch.Generator().manual_seed(SEED_DECODE_STEP + step)
    q = torch.randn(B, Hqk, d, generator=gen).to(dtype)
    k = torch.randn(B, Hqk, d, generator=gen).to(dtype)
    v = torch.randn(B, Hv, dv, generator=gen).to(dtype)
    g, beta = _gates(gen, (B, Hv))
    return dict(q=q, k=k, v=v, g=g, beta=beta)


def decode_state(B, Hv, d, std=0.05, seed=SEED_STATES + 2, dv=None):
    dv = dv or d
    gen = torch.Generator().manual_seed(seed)
    return torch.randn(B, Hv, dv, d, generator=gen) * std


def inputs_for(w: Workload):
    """Prefill inputs of a prefill workload, with its seeds."""
    assert w.kind == "prefill"
    return prefill_inputs(w.lengths, w.Hqk, w.Hv, w.d, w.torch_dtype,
                          seed=SEED_TOKENS + w.index, state_std=w.state_std,
                          state_seed=SEED_STATES + w.index)
