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
