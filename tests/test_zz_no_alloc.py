"""GPU test of gdn_prefill_noalloc, the allocation-free prefill entry point.

Callers that cannot allocate device memory (pre-planned runtime memory,
framework plugins that own every allocation, real-time loops) use the
library's built-in scratch array instead of a workspace. This file is named
to be collected last, so that a run stopping at its first failure has
already run every other test; it passes both alone and after them.

The entry point is called through the C ABI, twice in a row with different
inputs (the shared scratch keeps the previous call's contents, so each call
must clear what has to start at zero), and each result is compared with the
existing gdn_prefill entry point on the same inputs. Both run the same kernel
with the same launch plan, and every package and state step is computed in a
fixed order whichever CTA takes it, so the results must be identical bit for
bit: a stale flag or package left in the scratch by the previous call would
show as a difference however small.
"""
import ctypes

import pytest
import torch

import workloads

gdn = pytest.importorskip("gated_deltanet_linear_21_b200")

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _call_noalloc(x, o, s):
    lib = gdn.lib()
    T, Hqk, dk = x["q"].shape
    Hv, dv = x["v"].shape[1], x["v"].shape[2]
    N = x["cu_seqlens"].numel() - 1
    st = x["state_in"]
    status = lib.gdn_prefill_noalloc(
        x["q"].data_ptr(), x["k"].data_ptr(), x["v"].data_ptr(), x["g"].data_ptr(), x["beta"].data_ptr(),
        st.data_ptr() if st is not None else None, x["cu_seqlens"].data_ptr(), N, T, Hqk, Hv, dk, dv,
        ctypes.c_float(0.0), 0, gdn.GDN_BF16, o.data_ptr(), s.data_ptr(),
        torch.cuda.current_stream().cuda_stream)
    assert status == gdn.GDN_OK, lib.gdn_last_error().decode()


@pytest.mark.parametrize("call", [0, 1])
def test_noalloc_prefill_matches_workspace_prefill_twice(call):
    for rep, (lengths, seed) in enumerate([([1000, 37], 41), ([300, 64, 129], 42)]):
        x = workloads.prefill_inputs(lengths, Hqk=4, Hv=8, d=128, seed=seed + 10 * call, state_std=0.05)
        x = {kk: (vv.to(DEV) if isinstance(vv, torch.Tensor) else vv) for kk, vv in x.items()}
        T, Hv, N = x["v"].shape[0], x["v"].shape[1], x["cu_seqlens"].numel() - 1
        o_ref, s_ref = gdn.prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], x["state_in"], x["cu_seqlens"])
        o = torch.full((T, Hv, 128), float("nan"), dtype=torch.bfloat16, device=DEV)
        s = torch.full((N, Hv, 128, 128), float("nan"), device=DEV)
        _call_noalloc(x, o, s)
        torch.cuda.synchronize()
        gdn.device_error()
        assert not torch.isnan(o.float()).any() and not torch.isnan(s).any()
        assert torch.equal(o, o_ref), f"call {rep}: o differs by {(o.float() - o_ref.float()).abs().max().item():.3e}"
        assert torch.equal(s, s_ref), f"call {rep}: state differs by {(s - s_ref).abs().max().item():.3e}"


def test_noalloc_python_wrapper_checks_and_matches():
    """gdn.prefill_noalloc (the binding) validates its tensors like gdn.prefill and
    returns the same bits."""
    x = workloads.prefill_inputs([200, 65], Hqk=2, Hv=4, d=128, seed=4711, state_std=0.05)
    x = {kk: (vv.to(DEV) if isinstance(vv, torch.Tensor) else vv) for kk, vv in x.items()}
    args = (x["q"], x["k"], x["v"], x["g"], x["beta"], x["state_in"], x["cu_seqlens"])
    o_ref, s_ref = gdn.prefill(*args)
    o, s = gdn.prefill_noalloc(*args)
    torch.cuda.synchronize()
    gdn.device_error()
    assert torch.equal(o, o_ref) and torch.equal(s, s_ref)
    with pytest.raises(TypeError):   # a bf16 state_in would be read as twice the bytes
        gdn.prefill_noalloc(*args[:5], x["state_in"].to(torch.bfloat16), x["cu_seqlens"])
    with pytest.raises(ValueError):  # wrong number of sequences in state_in
        gdn.prefill_noalloc(*args[:5], x["state_in"][:1].contiguous(), x["cu_seqlens"])


def test_noalloc_scratch_covers_every_workspace_and_rejects_other_kernels():
    lib = gdn.lib()
    # the workspace is bounded however many sequences there are, so the
    # built-in scratch (sized for the largest) serves every problem
    assert lib.gdn_prefill_workspace_bytes(10000, 32, 128, 128, gdn.GDN_BF16) == \
        lib.gdn_prefill_workspace_bytes(100000, 64, 128, 128, gdn.GDN_BF16)
    P = 0x10000   # never dereferenced: argument checks fail first
    status = lib.gdn_prefill_noalloc(P, P, P, P, P, None, P, 1, 64, 2, 2, 128, 128,
                                     ctypes.c_float(0.0), 0, gdn.GDN_F32, P, P, None)
    assert status == gdn.GDN_ERR_UNSUPPORTED
    status = lib.gdn_prefill_noalloc(P, P, P, P, P, None, P, 1, 64, 2, 2, 128, 128,
                                     ctypes.c_float(0.0), 32, gdn.GDN_BF16, P, P, None)
    assert status == gdn.GDN_ERR_UNSUPPORTED
