"""Host-side tests of the C ABI (no GPU needed).

The library must load, export every function include/gdn.h declares, and
reject bad arguments with the documented status before touching the device.
Every call here fails host validation, so nothing is ever launched (the fake
pointers are never dereferenced).
"""
import ctypes
import os
import re

import pytest
import torch

import gated_deltanet_linear_21_b200 as gdn
from gated_deltanet_linear_21_b200 import build as gdn_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
P = 0x10000  # a 16-byte aligned fake device address (never dereferenced)


def declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"\b(gdn_[a-z_0-9]+)\s*\(", text)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    gdn_build.build()
    return gdn.lib()


def test_library_exports_every_declared_function(lib):
    names = declared_functions()
    assert {"gdn_prefill", "gdn_decode", "gdn_prefill_workspace_bytes", "gdn_last_error",
            "gdn_device_error", "gdn_version"} <= set(names)
    handle = ctypes.CDLL(gdn.library_path)
    for name in names:
        assert hasattr(handle, name), f"{name} declared in include/ but not exported"
    assert set(names) >= set(gdn.SIGNATURES), "binding names a function the header lacks"


def test_version(lib):
    assert lib.gdn_version() >= 1


def _prefill(lib, **kw):
    a = dict(q=P, k=P, v=P, g=P, beta=P, state_in=None, cu=P, n_seqs=1, total_T=64, Hqk=2, Hv=4,
             dk=128, dv=128, scale=0.0, chunk=0, dtype=gdn.GDN_BF16, o=P, state_out=P, ws=None,
             ws_bytes=0, stream=None)
    a.update(kw)
    return lib.gdn_prefill(a["q"], a["k"], a["v"], a["g"], a["beta"], a["state_in"], a["cu"],
                           a["n_seqs"], a["total_T"], a["Hqk"], a["Hv"], a["dk"], a["dv"], a["scale"],
                           a["chunk"], a["dtype"], a["o"], a["state_out"], a["ws"], a["ws_bytes"],
                           a["stream"])


def _decode(lib, **kw):
    a = dict(q=P, k=P, v=P, g=P, beta=P, state=P, B=4, Hqk=2, Hv=4, dk=128, dv=128, scale=0.0,
             dtype=gdn.GDN_BF16, o=P, stream=None)
    a.update(kw)
    return lib.gdn_decode(a["q"], a["k"], a["v"], a["g"], a["beta"], a["state"], a["B"], a["Hqk"],
                          a["Hv"], a["dk"], a["dv"], a["scale"], a["dtype"], a["o"], a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(o=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(cu=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(state_out=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(Hv=3), gdn.GDN_ERR_INVALID_ARG),
    (dict(Hqk=0), gdn.GDN_ERR_INVALID_ARG),
    (dict(n_seqs=-1), gdn.GDN_ERR_INVALID_ARG),
    (dict(total_T=-5), gdn.GDN_ERR_INVALID_ARG),
    (dict(total_T=1 << 31), gdn.GDN_ERR_INVALID_ARG),
    (dict(dk=96), gdn.GDN_ERR_UNSUPPORTED),
    (dict(dv=256), gdn.GDN_ERR_UNSUPPORTED),
    (dict(dtype=7), gdn.GDN_ERR_INVALID_ARG),
    (dict(q=P + 8), gdn.GDN_ERR_INVALID_ARG),
    (dict(state_in=P + 4), gdn.GDN_ERR_INVALID_ARG),
    (dict(g=P + 2), gdn.GDN_ERR_INVALID_ARG),
    (dict(chunk=48), gdn.GDN_ERR_UNSUPPORTED),
])
def test_prefill_rejects_bad_arguments(lib, kw, status):
    assert _prefill(lib, **kw) == status
    assert lib.gdn_last_error().decode().startswith("gdn_prefill")


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(state=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(Hv=5), gdn.GDN_ERR_INVALID_ARG),
    (dict(B=-1), gdn.GDN_ERR_INVALID_ARG),
    (dict(dk=100), gdn.GDN_ERR_UNSUPPORTED),
    (dict(dtype=3), gdn.GDN_ERR_INVALID_ARG),
    (dict(state=P + 4), gdn.GDN_ERR_INVALID_ARG),
    (dict(beta=P + 1), gdn.GDN_ERR_INVALID_ARG),
])
def test_decode_rejects_bad_arguments(lib, kw, status):
    assert _decode(lib, **kw) == status
    assert lib.gdn_last_error().decode().startswith("gdn_decode")


def test_empty_problems_are_no_ops(lib):
    assert _prefill(lib, n_seqs=0, q=None, k=None, v=None, o=None, cu=None, state_out=None) == gdn.GDN_OK
    assert _decode(lib, B=0, q=None, state=None, o=None) == gdn.GDN_OK
    assert lib.gdn_last_error() == b""


def test_workspace_query_is_pure(lib):
    a = lib.gdn_prefill_workspace_bytes(8, 32, 128, 128, gdn.GDN_BF16)
    b = lib.gdn_prefill_workspace_bytes(8, 32, 128, 128, gdn.GDN_BF16)
    assert a == b


# ------------------------------------------------------------- launch plan ---

def test_prefill_plan_for_the_benchmark_workloads():
    """The cost model's choices (a 148-SM B200 given explicitly: no GPU needed)."""
    # 4096 tokens x 16 heads: 16 chains of 4 slices of 32 state rows, 84 preparing CTAs
    assert gdn.prefill_plan(1, 4096, 16, sm_count=148) == (32, 64, 1)
    # long prompts x 32 heads: 32 chains of one 128-row slice, 116 preparing CTAs
    assert gdn.prefill_plan(1, 32768, 32, sm_count=148) == (128, 32, 1)
    assert gdn.prefill_plan(1, 81920, 32, sm_count=148) == (128, 32, 1)
    # f16 inputs run the same kernel with the same plans and workspace
    assert gdn.prefill_plan(1, 4096, 16, dtype=torch.float16, sm_count=148) == (32, 64, 1)
    assert gdn.prefill_workspace_bytes(1, 16, 128, 128, torch.float16) == \
        gdn.prefill_workspace_bytes(1, 16, 128, 128, torch.bfloat16) > 0


@pytest.mark.parametrize("n_seqs,total_T,Hv", [(8, 37000, 32), (300, 45000, 8), (3, 500, 8), (64, 64 * 300, 16)])
def test_prefill_plan_keeps_rounds_to_whole_sequences(n_seqs, total_T, Hv):
    """With several sequences a round runs whole sequences (positions a multiple
    of Hv) or equal parts of one (a divisor of Hv); every plan leaves CTAs to
    prepare and covers every sequence-head."""
    dvp, nc, rounds = gdn.prefill_plan(n_seqs, total_T, Hv, sm_count=148)
    slices = 128 // dvp
    positions = nc // slices
    assert dvp in (32, 64, 128) and nc % slices == 0 and nc <= 148 - 8
    assert positions % Hv == 0 or Hv % positions == 0
    assert positions <= min(n_seqs * Hv, 74)
    assert rounds == -(-(n_seqs * Hv) // positions)


def test_prefill_plan_applies_and_clamps_a_requested_plan():
    plan = lambda req: gdn.prefill_plan(1, 4096, 16, sm_count=148, requested=req)
    assert plan((64, 7)) == (64, 6, 6)           # rounded down to whole chains of 2 slices
    assert plan((64, 1000)) == (64, 32, 1)       # no more chain CTAs than slices to run
    assert plan((0, 0)) == plan(None) == (32, 64, 1)
    assert plan((128, 0)) == (128, 16, 1)        # another width keeps the model's 16 chains per round
    assert plan((0, 8)) == (32, 8, 8)            # a count alone keeps the model's width
    assert gdn.prefill_plan(1, 81920, 32, sm_count=148, requested=(32, 500)) == (32, 128, 1)   # 74 positions max
    for bad in ((48, 0), (0, -1)):                # not a slice width; a negative count
        with pytest.raises(gdn.GdnError) as e:
            plan(bad)
        assert e.value.status == gdn.GDN_ERR_INVALID_ARG


def test_concurrent_prefill_plans_do_not_leak_between_threads():
    """The plan is an argument of the call, not process state: host threads asking
    with different plans at the same time each get their own."""
    import threading
    errors = []

    def worker(req, want):
        for _ in range(2000):
            got = gdn.prefill_plan(1, 4096, 16, sm_count=148, requested=req)
            if got != want:
                errors.append((req, got))
                return

    cases = [((64, 6), (64, 6, 6)), ((128, 3), (128, 3, 6)), (None, (32, 64, 1)), ((32, 16), (32, 16, 4))]
    threads = [threading.Thread(target=worker, args=c) for c in cases]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors


def test_prefill_ex_rejects_an_invalid_plan_before_any_launch(lib):
    for dvp, nc in ((48, 0), (64, -2)):
        status = lib.gdn_prefill_ex(P, P, P, P, P, None, P, 1, 64, 2, 4, 128, 128, ctypes.c_float(0.0), 0,
                                    gdn.GDN_BF16, P, P, P, 1 << 26, ctypes.byref(gdn.GdnPlan(dvp, nc)), None)
        assert status == gdn.GDN_ERR_INVALID_ARG
        assert "plan" in lib.gdn_last_error().decode()


def test_prefill_plan_rejects_what_the_kernel_does_not_run(lib):
    with pytest.raises(gdn.GdnError) as e:
        gdn.prefill_plan(1, 4096, 16, dk=64, dv=64, sm_count=148)
    assert e.value.status == gdn.GDN_ERR_UNSUPPORTED
    with pytest.raises(gdn.GdnError) as e:
        gdn.prefill_plan(1, 4096, 16, dtype=torch.float32, sm_count=148)
    assert e.value.status == gdn.GDN_ERR_UNSUPPORTED
    for bad in (dict(n_seqs=0), dict(Hv=0), dict(total_T=-1), dict(sm_count=8)):
        a = dict(n_seqs=1, total_T=4096, Hv=16, sm_count=148)
        a.update(bad)
        with pytest.raises(gdn.GdnError) as e:
            gdn.prefill_plan(a["n_seqs"], a["total_T"], a["Hv"], sm_count=a["sm_count"])
        assert e.value.status == gdn.GDN_ERR_INVALID_ARG
    out = ctypes.c_int(0)
    assert lib.gdn_prefill_plan(1, 4096, 16, 128, 128, gdn.GDN_BF16, 148, None, None, ctypes.byref(out),
                                ctypes.byref(out)) == gdn.GDN_ERR_INVALID_ARG
