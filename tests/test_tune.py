"""Host logic of the measured launch-plan choice (gated_deltanet_linear_21_b200.tune):
the candidate grid, the correctness gate, the override context and the selection,
with a fake runner in place of the device (no GPU needed)."""
import math
import os

import pytest
import torch

from gated_deltanet_linear_21_b200 import tune


def test_candidate_plans_cover_every_width_within_the_limits():
    for chains in (1, 3, 16, 32, 74, 500):
        plans = tune.candidate_plans(chains)
        assert {d for d, _ in plans} == {32, 64, 128}
        assert len(plans) == len(set(plans))
        for dvp, nc in plans:
            slices = 128 // dvp
            assert nc % slices == 0
            assert 1 <= nc // slices <= min(chains, 74)
            assert nc <= 148 - 8
    # the 4096-token layer (16 chains): one round at each width is among them
    assert {(32, 64), (64, 32), (128, 16)} <= set(tune.candidate_plans(16))
    assert (128, 74) in tune.candidate_plans(500) and (32, 140) in tune.candidate_plans(500)


def test_gate_rejects_unwritten_and_distant_outputs():
    ref = torch.linspace(-2.0, 2.0, 64).reshape(8, 8)
    assert tune.gate(ref.clone(), ref)[0]
    ok, err, _ = tune.gate(ref + 2.0 / 64 * 0.99, ref)      # just inside 1/64 of max |ref| = 2
    assert ok and err == pytest.approx(2.0 / 64 * 0.99, rel=1e-5)   # (float32 sums)
    ok, err, why = tune.gate(ref + 2.0 / 64 * 1.01, ref)
    assert not ok and "max difference" in why
    bad = ref.clone()
    bad[3, 4] = math.nan
    ok, err, why = tune.gate(bad, ref)
    assert not ok and math.isinf(err) and "NaN" in why
    assert not tune.gate(ref[:4], ref)[0]
    assert tune.gate(torch.empty(0, 8), torch.empty(0, 8))[0]


def test_check_problem_has_a_full_and_a_partial_chunk_and_a_state():
    q, k, v, g, beta, s, cu = tune.check_problem(2, 4, 128, 128, torch.bfloat16, "cpu")
    assert q.shape == (101, 2, 128) and v.shape == (101, 4, 128) and q.dtype == torch.bfloat16
    assert cu.tolist() == [0, 101] and 101 // 64 == 1 and 101 % 64 == 37
    assert (g <= 0).all() and ((beta > 0) & (beta < 1)).all()
    assert s.shape == (1, 4, 128, 128) and float(s.abs().max()) > 0


def _fake_problem():
    gen = torch.Generator().manual_seed(7)
    T, Hqk, Hv, d = 130, 2, 4, 128
    q = torch.randn(T, Hqk, d, generator=gen).to(torch.bfloat16)
    k = torch.randn(T, Hqk, d, generator=gen).to(torch.bfloat16)
    v = torch.randn(T, Hv, d, generator=gen).to(torch.bfloat16)
    g = -torch.rand(T, Hv, generator=gen)
    beta = torch.rand(T, Hv, generator=gen)
    return q, k, v, g, beta


class FakeRunner:
    """Stands in for the device: a deterministic 'result' per problem, spoiled
    for some plans, and a time per plan."""
    TIMES = {(32, 64): 2.0, (64, 32): 1.0, (128, 16): 0.5, (64, 16): 0.4, (32, 32): 0.3}

    def __init__(self):
        self.calls = []

    def __call__(self, args, plan, reps):
        self.calls.append((plan, reps, args[0].shape[0]))
        q, k, v, g, beta, s_in, cu = args
        T, _, dk = q.shape
        Hv, dv = v.shape[1], v.shape[2]
        o = v.float() * 0.5 + 0.25
        s = torch.ones(cu.numel() - 1, Hv, dv, dk)
        if plan == (32, 32):
            raise RuntimeError("a bounded device wait ran out")
        if plan == (128, 16):            # fastest of the valid-looking ones, but wrong
            o = o + 0.1 * float(o.abs().max())
        if plan == (64, 16) and T < 128:  # leaves an element unwritten on the check problem only
            o = o.clone()
            o[-1, 0, 0] = math.nan
        ms = self.TIMES.get(plan, 9.0) if reps else math.nan
        return o, s, ms


def test_tune_keeps_the_fastest_plan_that_passes_the_gate():
    q, k, v, g, beta = _fake_problem()
    run = FakeRunner()
    plans = list(FakeRunner.TIMES)
    best, results = tune.tune_prefill(q, k, v, g, beta, plans=plans, runner=run)
    assert (best.dvp, best.nc) == (64, 32) and best.ok and best.ms == 1.0
    by = {(r.dvp, r.nc): r for r in results}
    assert by[(32, 64)].ok
    assert not by[(128, 16)].ok and "o:" in by[(128, 16)].reason
    assert not by[(64, 16)].ok and "check o" in by[(64, 16)].reason and "NaN" in by[(64, 16)].reason
    assert not by[(32, 32)].ok and "RuntimeError" in by[(32, 32)].reason and math.isinf(by[(32, 32)].ms)
    # the default plan ran first on both problems, untimed; each candidate was timed on
    # the caller's problem and checked, untimed, on the check problem
    assert run.calls[0] == (None, 0, 130) and run.calls[1] == (None, 0, 101)
    assert (plans[0], 5, 130) in run.calls and (plans[0], 0, 101) in run.calls


def test_tune_raises_when_no_plan_passes():
    q, k, v, g, beta = _fake_problem()
    with pytest.raises(ValueError, match="no launch plan passed"):
        tune.tune_prefill(q, k, v, g, beta, plans=[(128, 16), (32, 32)], runner=FakeRunner())


def test_tune_refuses_a_default_plan_that_leaves_elements_unwritten():
    q, k, v, g, beta = _fake_problem()

    def broken(args, plan, reps):
        o, s, ms = FakeRunner()(args, plan, reps)
        if plan is None:
            s = s.clone()
            s[0, 0, 0, 0] = math.nan
        return o, s, ms

    with pytest.raises(RuntimeError, match="default plan left state"):
        tune.tune_prefill(q, k, v, g, beta, plans=[(64, 32)], runner=broken)


def test_tune_refuses_shapes_without_launch_plans():
    q, k, v, g, beta = _fake_problem()
    with pytest.raises(ValueError, match="tensor-core kernel"):
        tune.tune_prefill(q.float(), k.float(), v.float(), g, beta, plans=[(64, 32)], runner=FakeRunner())
    with pytest.raises(ValueError, match="tensor-core kernel"):
        tune.tune_prefill(q[..., :64], k[..., :64], v[..., :64], g, beta, plans=[(64, 32)], runner=FakeRunner())


def test_device_runner_applies_the_plan_times_and_fills_fresh_outputs(monkeypatch):
    """The device leg's own lines, with the library call, the error check and the
    CUDA events replaced by stand-ins (no GPU): the plan is passed to every
    call (no process state), the gated outputs come from a call into NaN-filled
    buffers, and the time is the events' over the timed calls."""
    import gated_deltanet_linear_21_b200 as pkg
    seen = []

    def fake_prefill(q, k, v, g, beta, state_in=None, cu_seqlens=None, *, o=None, state_out=None, plan=None,
                     **kw):
        seen.append((plan, o is not None))
        T, Hv, dv = v.shape
        N = cu_seqlens.numel() - 1
        if o is not None:
            assert torch.isnan(o).all() and torch.isnan(state_out).all()   # fresh NaN buffers
            o.copy_(v.float() * 2)
            state_out.fill_(3.0)
            return o, state_out
        return v * 2, torch.full((N, Hv, dv, q.shape[2]), 3.0)

    class FakeEvent:
        def __init__(self, enable_timing=False):
            pass

        def record(self, stream=None):
            pass

        def elapsed_time(self, other):
            return 6.0

    monkeypatch.setattr(pkg, "prefill", fake_prefill)
    monkeypatch.setattr(pkg, "device_error", lambda stream=None: None)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a, **k: None)
    monkeypatch.setattr(torch.cuda, "Event", FakeEvent)
    q, k, v, g, beta = _fake_problem()
    cu = torch.tensor([0, 130], dtype=torch.int32)
    o, s, ms = tune._device_runner((q, k, v, g, beta, None, cu), (64, 32), 3)
    assert ms == pytest.approx(2.0)                                   # 6 ms over 3 timed calls
    assert o.dtype == torch.bfloat16 and o.shape == v.shape and torch.equal(o.float(), (v.float() * 2).to(o.dtype).float())
    assert s.shape == (1, 4, 128, 128) and bool((s == 3.0).all())
    assert seen == [((64, 32), False)] * 4 + [((64, 32), True)]  # warm-up, 3 timed, the gated call
    seen.clear()
    o, s, ms = tune._device_runner((q, k, v, g, beta, None, cu), None, 0)   # the default plan, untimed
    assert math.isnan(ms) and seen == [(None, True)]
    # and the whole selection through the device leg
    best, results = tune.tune_prefill(q, k, v, g, beta, None, cu, plans=[(32, 16), (128, 4)], reps=2)
    assert all(r.ok for r in results) and (best.dvp, best.nc) == (32, 16)


@pytest.mark.gpu
def test_tune_prefill_on_the_device_returns_a_gated_plan_that_matches_the_oracle():
    """The tuner's whole device leg on a B200: two 700-token sequences, 4 q/k and
    8 value heads. Every candidate plan is timed and gated against the default
    plan; the chosen plan must have passed, and its output must also match the
    fp64 oracle at the bf16 prefill tolerances and the 1/64 rule."""
    import numpy as np

    import gated_deltanet_linear_21_b200 as gdn
    import oracle
    import workloads

    x = workloads.prefill_inputs([700, 700], Hqk=4, Hv=8, d=128, seed=8800, state_std=0.05)
    d = {kk: (vv.to("cuda") if isinstance(vv, torch.Tensor) else vv) for kk, vv in x.items()}
    args = (d["q"], d["k"], d["v"], d["g"], d["beta"], d["state_in"], d["cu_seqlens"])
    best, results = tune.tune_prefill(*args, reps=3)
    assert best.ok and math.isfinite(best.ms) and best.ms > 0
    assert len(results) >= 3 and all(r.ok for r in results), [r.reason for r in results if not r.ok]
    o, s = gdn.prefill(*args, plan=(best.dvp, best.nc))
    o_def, s_def = gdn.prefill(*args)
    torch.cuda.synchronize()
    gdn.device_error()
    ro, rs = oracle.prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], x["state_in"], x["cu_seqlens"])
    for got, ref, tol in ((o, ro, 2e-2), (s, rs, 1e-2), (o_def, ro, 2e-2), (s_def, rs, 1e-2)):
        a = got.double().cpu().numpy()
        err = float(np.abs(a - ref).max())
        assert err <= tol and err <= np.abs(ref).max() / 64
    print("plans:", [(r.dvp, r.nc, round(r.ms, 4), f"{r.err:.1e}") for r in results], "best", (best.dvp, best.nc))
