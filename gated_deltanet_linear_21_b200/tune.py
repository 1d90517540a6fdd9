"""Measured choice of the tensor-core prefill's launch plan, with a correctness gate.

The library picks the plan of its tensor-core prefill -- the state-slice width
DVP (32, 64 or 128 state rows per state-carrying CTA) and the number of
state-carrying CTAs -- from a cost model. ``tune_prefill`` measures instead and
checks every candidate before trusting its time, as the pages' engine does
after it once kept a fast but wrong kernel ("One level down: #004 the same
compiler on Apple's chips", section "The night the engine chose wrong": each
candidate is compared with a kernel already trusted, on a full and a partial
block, and dropped beyond 1/64 of the largest value):

* each candidate plan runs the caller's problem with that plan passed to the
  call (gdn_prefill_ex), timed with CUDA events over a few calls after a
  warm-up;
* its outputs must match the default plan's within 1/64 of the largest value,
  on the caller's problem and on a check problem of one full and one partial
  64-token chunk entering a non-zero state. The pages zero the output first;
  here it is filled with NaN, which shows an unwritten element whatever value
  was expected there;
* the fastest plan that passes is returned; pass ``(best.dvp, best.nc)`` as
  ``plan=`` to ``prefill`` to run with it.

Only the plan differs between candidates: every run goes through the library's
kernels, and the default plan is the one the parity tests hold to the oracle.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch

_SLICE_WIDTHS = (32, 64, 128)


@dataclass
class PlanResult:
    dvp: int
    nc: int
    ms: float          # per call, CUDA events
    err: float         # largest difference from the default plan (o, state, check problem)
    ok: bool
    reason: str = ""


def candidate_plans(n_chains: int, sms: int = 148, max_positions: int = 74):
    """(dvp, nc) candidates for `n_chains` sequence-heads: every slice width, with
    as many chains per round as fit and with the chains split into 2, 3 or 4
    rounds. nc is a multiple of the slices per chain and leaves at least 8 CTAs
    for preparation; the library applies the same limits."""
    plans = []
    for dvp in _SLICE_WIDTHS:
        slices = 128 // dvp
        p_max = min(n_chains, max_positions, (sms - 8) // slices)
        if p_max < 1:
            continue
        positions = {p_max} | {min(p_max, math.ceil(n_chains / r)) for r in (2, 3, 4)}
        for p in sorted(positions, reverse=True):
            if p >= 1 and (dvp, p * slices) not in plans:
                plans.append((dvp, p * slices))
    return plans


def gate(out: torch.Tensor, ref: torch.Tensor, rel_tol: float = 1 / 64):
    """(ok, err, reason): `out` fully written (no NaN) and within rel_tol of the
    largest magnitude of `ref`."""
    o = out.detach().to(torch.float64)
    r = ref.detach().to(torch.float64)
    if o.shape != r.shape:
        return False, math.inf, f"shape {tuple(o.shape)} != {tuple(r.shape)}"
    if o.numel() == 0:
        return True, 0.0, ""
    if torch.isnan(o).any():
        return False, math.inf, "unwritten (NaN) elements"
    err = float((o - r).abs().max())
    bound = rel_tol * float(r.abs().max()) + 1e-7
    if err > bound:
        return False, err, f"max difference {err:.3e} > {bound:.3e}"
    return True, err, ""


def select_plan(results):
    """The fastest plan that passed its gate; ValueError if none did."""
    good = [r for r in results if r.ok]
    if not good:
        raise ValueError("no launch plan passed the correctness gate: "
                         + "; ".join(f"({r.dvp}, {r.nc}): {r.reason}" for r in results))
    return min(good, key=lambda r: r.ms)


def check_problem(Hqk, Hv, dk, dv, dtype, device, seed=1234):
    """One sequence of 64 + 37 tokens (a full and a partial chunk) entering a
    non-zero state, drawn like the benchmark inputs."""
    gen = torch.Generator().manual_seed(seed)
    T = 64 + 37
    q = torch.randn(T, Hqk, dk, generator=gen).to(dtype)
    k = torch.randn(T, Hqk, dk, generator=gen).to(dtype)
    v = torch.randn(T, Hv, dv, generator=gen).to(dtype)
    g = torch.nn.functional.logsigmoid(torch.randn(T, Hv, generator=gen, dtype=torch.float64) + 3.0).float()
    beta = torch.sigmoid(torch.randn(T, Hv, generator=gen, dtype=torch.float64)).float()
    state = (0.05 * torch.randn(1, Hv, dv, dk, generator=gen)).float()
    cu = torch.tensor([0, T], dtype=torch.int32)
    return tuple(t.to(device) for t in (q, k, v, g, beta, state, cu))


def _device_runner(args, plan, reps):
    """Run the prefill of `args` under `plan` (None: the default); returns
    (o, state_out, ms per call) with o, state_out from a call into NaN-filled
    buffers and ms from `reps` further calls (nan if reps == 0)."""
    from . import device_error, prefill

    q, k, v, g, beta, state_in, cu = args
    T, _, dk = q.shape
    Hv, dv = v.shape[1], v.shape[2]
    N = cu.numel() - 1
    ms = math.nan
    if reps > 0:
        prefill(q, k, v, g, beta, state_in, cu, plan=plan)   # warm-up
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(reps):
            prefill(q, k, v, g, beta, state_in, cu, plan=plan)
        b.record()
        torch.cuda.synchronize()
        ms = a.elapsed_time(b) / reps
    o = torch.full((T, Hv, dv), math.nan, dtype=q.dtype, device=q.device)
    s = torch.full((N, Hv, dv, dk), math.nan, dtype=torch.float32, device=q.device)
    prefill(q, k, v, g, beta, state_in, cu, o=o, state_out=s, plan=plan)
    device_error()
    return o, s, ms


def tune_prefill(q, k, v, g, beta, state_in=None, cu_seqlens=None, *, plans=None, reps=5,
                 rel_tol=1 / 64, runner=None):
    """Measure the candidate launch plans on this problem (arguments as for
    ``prefill``) and return (best PlanResult, all results). `runner(args, plan,
    reps) -> (o, state_out, ms)` runs one plan (the default one for plan=None);
    it is replaceable for tests."""
    runner = runner or _device_runner
    T, Hqk, dk = q.shape
    Hv, dv = v.shape[1], v.shape[2]
    if q.dtype != torch.bfloat16 or dk != 128 or dv != 128:
        raise ValueError("launch plans belong to the tensor-core kernel (bf16, d_k = d_v = 128); "
                         "other shapes run on the fp32 SIMT kernel, which has none")
    if cu_seqlens is None:
        cu_seqlens = torch.tensor([0, T], dtype=torch.int32, device=q.device)
    N = cu_seqlens.numel() - 1
    args = (q, k, v, g, beta, state_in, cu_seqlens)
    chk = check_problem(Hqk, Hv, dk, dv, q.dtype, q.device)
    if plans is None:
        plans = candidate_plans(N * Hv)
    ref_o, ref_s, _ = runner(args, None, 0)
    chk_o, chk_s, _ = runner(chk, None, 0)
    for name, t in (("o", ref_o), ("state", ref_s), ("check o", chk_o), ("check state", chk_s)):
        if torch.isnan(t.detach().float()).any():
            raise RuntimeError(f"the default plan left {name} elements unwritten")
    results = []
    for dvp, nc in plans:
        try:
            o, s, ms = runner(args, (dvp, nc), reps)
            co, cs, _ = runner(chk, (dvp, nc), 0)
        except Exception as e:  # a plan the library rejects or whose waits ran out
            results.append(PlanResult(dvp, nc, math.inf, math.inf, False, f"{type(e).__name__}: {e}"))
            continue
        ok, err, why = True, 0.0, ""
        for name, out, ref in (("o", o, ref_o), ("state", s, ref_s), ("check o", co, chk_o),
                               ("check state", cs, chk_s)):
            good, e, reason = gate(out, ref, rel_tol)
            err = max(err, e)
            if not good and ok:
                ok, why = False, f"{name}: {reason}"
        results.append(PlanResult(dvp, nc, ms, err, ok, why))
    return select_plan(results), results
