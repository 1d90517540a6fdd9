"""The GDN_DEBUG build (libgdn_debug.so): the same kernels with device-side
index checks on the ring positions and slots, sequence bounds, token and head
coordinates and state offsets of the tensor-core prefill. A failed check
records GDN_ERR_DEVICE_CHECK in the device error word and stops the CTA's
work instead of touching memory out of bounds; it never traps.

The CPU test checks that both builds load and say which they are. The GPU
test runs the small parity cases -- ragged lengths, several sequences, every
state-slice width, multi-round splits, a ring-wrapping chain, f16 -- through
the debug build's C ABI, requires every check to pass (gdn_device_error
clear), and compares the results with the fp64 oracle at the bf16 prefill
tolerances.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads

gdn = pytest.importorskip("gated_deltanet_linear_21_b200")
DEV = "cuda"


def test_both_builds_load_and_say_which_they_are():
    from gated_deltanet_linear_21_b200 import build as gdn_build
    gdn_build.build()
    assert gdn.lib().gdn_debug_checks() == 0
    assert gdn.debug_lib().gdn_debug_checks() == 1


def _prefill_debug(lib, x, plan=None):
    q, k, v = x["q"], x["k"], x["v"]
    T, Hqk, dk = q.shape
    Hv, dv = v.shape[1], v.shape[2]
    N = x["cu_seqlens"].numel() - 1
    dtype = gdn.GDN_F16 if q.dtype == torch.float16 else gdn.GDN_BF16
    o = torch.full((T, Hv, dv), float("nan"), dtype=q.dtype, device=DEV)
    s = torch.full((N, Hv, dv, dk), float("nan"), device=DEV)
    ws_bytes = lib.gdn_prefill_workspace_bytes(N, Hv, dk, dv, dtype)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=DEV)
    st = x["state_in"]
    status = lib.gdn_prefill_ex(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), x["g"].data_ptr(), x["beta"].data_ptr(),
        st.data_ptr() if st is not None else None, x["cu_seqlens"].data_ptr(), N, T, Hqk, Hv, dk, dv,
        ctypes.c_float(0.0), 0, dtype, o.data_ptr(), s.data_ptr(), ws.data_ptr(), ws_bytes,
        ctypes.byref(gdn.GdnPlan(*plan)) if plan else None, torch.cuda.current_stream().cuda_stream)
    assert status == gdn.GDN_OK, lib.gdn_last_error().decode()
    status = lib.gdn_device_error(torch.cuda.current_stream().cuda_stream)
    assert status == gdn.GDN_OK, lib.gdn_last_error().decode()
    return o, s


CASES = [
    ([65], 2, 4, None, torch.bfloat16),
    ([197], 2, 4, None, torch.bfloat16),
    ([5, 130, 1, 64, 77], 2, 4, None, torch.bfloat16),
    ([300, 129, 64, 1], 4, 8, (32, 0), torch.bfloat16),
    ([300, 129, 64, 1], 4, 8, (64, 6), torch.bfloat16),
    ([300, 129, 64, 1], 4, 8, (128, 3), torch.bfloat16),
    ([2500], 2, 4, (64, 2), torch.bfloat16),
    ([0, 40, 0], 2, 4, None, torch.bfloat16),
    ([197, 70], 2, 4, None, torch.float16),
]


@pytest.mark.gpu
@pytest.mark.parametrize("lengths,Hqk,Hv,plan,dtype", CASES)
def test_debug_build_runs_the_small_cases_with_every_check_passing(lengths, Hqk, Hv, plan, dtype):
    lib = gdn.debug_lib()
    assert lib.gdn_debug_checks() == 1
    x = workloads.prefill_inputs(lengths, Hqk=Hqk, Hv=Hv, d=128, dtype=dtype, seed=3300 + sum(lengths),
                                 state_std=0.05)
    xd = {kk: (vv.to(DEV) if isinstance(vv, torch.Tensor) else vv) for kk, vv in x.items()}
    o, s = _prefill_debug(lib, xd, plan)
    torch.cuda.synchronize()
    ro, rs = oracle.prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], x["state_in"], x["cu_seqlens"])
    a = o.double().cpu().numpy()
    b = s.double().cpu().numpy()
    assert not np.isnan(a).any() and not np.isnan(b).any()
    assert np.abs(a - ro).max() <= 2e-2
    assert np.abs(b - rs).max() <= 1e-2
