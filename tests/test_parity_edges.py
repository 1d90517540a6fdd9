"""GPU parity at the method's edges: gate values and inputs the benchmark
draws never produce.

The benchmark's gates (alpha = sigmoid(N(3,1)), beta = sigmoid(N(0,1))) keep a
chunk's decay range at a few units, so every chunk of the tensor-core kernel
takes its factored decay path (exp(G_r - m) exp(m - G_s) around the middle of
the range). These cases drive the other branches and the degenerate values of
the gated delta rule through the same kernels and compare them with the fp64
oracle, element by element, every head:

  strong_decay    g ~ -5 per token: a chunk's decay range is ~320 > 160, so the
                  exact per-entry decay path runs; alpha -> 0 (the state is
                  nearly replaced by each token's write)
  logsig_neg3     g = log sigmoid(N(-3, 2)): strong, uneven decay; chunks fall
                  on both sides of the range limit
  no_decay        g = 0 (alpha = 1) on every token: nothing decays
  beta_0_1        beta = 0 on even chunks (no write), beta = 1 on odd chunks
                  (full replacement along k)
  positive_g      a few tokens with g > 0 (alpha > 1): the "all g <= 0" test of
                  the factored path fails for their chunks
  zero_qk         all-zero q and k rows: the normalisation reduces to the
                  epsilon inside the square root (q^ = 0, k^ = 0)
  mixed_chunks    one chunk of each kind in a row: strong decay, then alpha = 1
                  with beta = 1, then beta = 0, then ordinary gates

Each at 64, 65 and 197 tokens (one full chunk, a full and a one-token chunk,
three full and a partial chunk), entering a non-zero state, with grouped heads
(2 q/k heads, 4 value heads). Gates: the bf16 prefill tolerances (o <= 2e-2,
state <= 1e-2) and 1/64 of the largest reference value; the fp32 SIMT kernel
at 1e-4.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads

gdn = pytest.importorskip("gated_deltanet_linear_21_b200")

pytestmark = pytest.mark.gpu
DEV = "cuda"
C = 64

KINDS = ("strong_decay", "logsig_neg3", "no_decay", "beta_0_1", "positive_g", "zero_qk", "mixed_chunks")


def edge_inputs(kind, L, d=128, dtype=torch.bfloat16, seed=0):
    """One sequence of L tokens (2 q/k heads, 4 value heads, head size d) with the
    gates or rows of `kind` written over the ordinary seeded draws."""
    x = workloads.prefill_inputs([L], Hqk=2, Hv=4, d=d, dtype=dtype, seed=6100 + seed + L, state_std=0.05)
    gen = torch.Generator().manual_seed(6200 + seed + L)
    g, beta, q, k = x["g"], x["beta"], x["q"], x["k"]
    chunk = torch.arange(L) // C
    if kind == "strong_decay":
        g[:] = workloads.shifted_log_decay(gen, g.shape, -5.0, 0.5)
    elif kind == "logsig_neg3":
        g[:] = workloads.log_sigmoid_gates(gen, g.shape, -3.0, 2.0)
    elif kind == "no_decay":
        g[:] = 0.0
    elif kind == "beta_0_1":
        beta[chunk % 2 == 0] = 0.0
        beta[chunk % 2 == 1] = 1.0
    elif kind == "positive_g":
        for t in (3, 40, 64, 100, 150):
            if t < L:
                g[t] = torch.tensor([0.25, 0.1, 0.4, 0.05])
    elif kind == "zero_qk":
        for t, which in ((5, "q"), (9, "k"), (64, "qk"), (130, "k"), (0, "q")):
            if t < L:
                if "q" in which:
                    q[t, t % 2] = 0
                if "k" in which:
                    k[t, (t + 1) % 2] = 0
    elif kind == "mixed_chunks":
        first = chunk == 0
        g[first] = workloads.shifted_log_decay(gen, g[first].shape, -5.0, 0.5)
        g[chunk == 1] = 0.0
        beta[chunk == 1] = 1.0
        beta[chunk == 2] = 0.0
    else:
        raise KeyError(kind)
    return x


def _run(x, chunk=0):
    d = {kk: (vv.to(DEV) if isinstance(vv, torch.Tensor) else vv) for kk, vv in x.items()}
    T, Hv, dv = d["v"].shape
    N = d["cu_seqlens"].numel() - 1
    dk = d["q"].shape[2]
    o = torch.full((T, Hv, dv), float("nan"), dtype=d["q"].dtype, device=DEV)
    s = torch.full((N, Hv, dv, dk), float("nan"), dtype=torch.float32, device=DEV)
    gdn.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state_in"], d["cu_seqlens"], chunk=chunk,
                o=o, state_out=s)
    torch.cuda.synchronize()
    gdn.device_error()
    ro, rs = oracle.prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], x["state_in"], x["cu_seqlens"])
    return o, s, ro, rs


def _compare(name, gpu, ref, tol):
    a = gpu.detach().to("cpu", torch.float64).numpy()
    assert not np.isnan(a).any(), f"{name}: kernel left unwritten (NaN) elements"
    assert np.isfinite(ref).all(), f"{name}: the oracle's values are not finite"
    err = float(np.abs(a - ref).max())
    ref_max = float(np.abs(ref).max())
    print(f"{name}: max abs error {err:.3e} (max |ref| {ref_max:.3e})")
    assert err <= tol, f"{name}: max abs error {err:.3e} > {tol:.1e}"
    assert err <= ref_max / 64 + 1e-7, f"{name}: max abs error {err:.3e} > 1/64 of {ref_max:.3e}"


@pytest.mark.parametrize("L", [64, 65, 197])
@pytest.mark.parametrize("kind", KINDS)
def test_tensor_core_prefill_edges(kind, L):
    x = edge_inputs(kind, L)
    o, s, ro, rs = _run(x)
    _compare(f"{kind} L={L} o", o, ro, 2e-2)
    _compare(f"{kind} L={L} state", s, rs, 1e-2)


@pytest.mark.parametrize("kind", ("strong_decay", "no_decay", "positive_g", "zero_qk", "mixed_chunks"))
def test_tensor_core_prefill_edges_f16(kind):
    """The f16 instantiation of the tensor-core kernel on the same edges (its
    operands have a narrower exponent range than bf16: tiny decayed terms
    flush to zero)."""
    x = edge_inputs(kind, 197, dtype=torch.float16)
    o, s, ro, rs = _run(x)
    _compare(f"{kind} f16 o", o, ro, 2e-2)
    _compare(f"{kind} f16 state", s, rs, 1e-2)


@pytest.mark.parametrize("kind", KINDS)
def test_simt_prefill_edges_fp32(kind):
    x = edge_inputs(kind, 197, d=64, dtype=torch.float32)
    o, s, ro, rs = _run(x, chunk=64)
    _compare(f"{kind} fp32 o", o, ro, 1e-4)
    _compare(f"{kind} fp32 state", s, rs, 1e-4)


@pytest.mark.parametrize("kind", ("strong_decay", "no_decay", "beta_0_1", "positive_g", "zero_qk"))
def test_decode_edges(kind):
    """Three decode steps on the same edge inputs, token by token (the decode
    kernel takes no chunk path, but alpha -> 0, alpha = 1, alpha > 1, beta in
    {0, 1} and zero rows still reach its arithmetic)."""
    x = edge_inputs(kind, 197)
    B = 1
    st = x["state_in"].clone()
    ref = st.double().numpy().copy()
    sd = st.to(DEV)
    for t in (0, 3, 5, 9, 40, 64, 100, 130, 150):
        sl = {n: x[n][t:t + 1].contiguous() for n in ("q", "k", "v", "g", "beta")}
        o = gdn.decode(*(sl[n].to(DEV) for n in ("q", "k", "v", "g", "beta")), sd)
        ro, ref = oracle.decode(sl["q"], sl["k"], sl["v"], sl["g"], sl["beta"], ref)
        assert o.shape[0] == B
        _compare(f"{kind} decode t={t} o", o, ro, 2e-2)
    _compare(f"{kind} decode state", sd, ref, 1e-2)
