"""Pins for the fp64 oracle (CPU only).

The oracle is checked against things other than itself: an explicit-matrix
brute force, an independently written chunked (WY) formulation, closed forms
of the gated delta rule, a hand-worked example, invariants (varlen packing,
continuation from a state, decode == prefill) -- and each pin's power is
shown by planting typical mistakes in a copy of the oracle's C source and
checking that some pin fails.
"""
import ctypes
import json
import os
import subprocess

import numpy as np
import pytest
import torch

import oracle
import workloads
from tests import _brute

HERE = os.path.dirname(os.path.abspath(__file__))


def _rand_inputs(lengths, Hqk, Hv, dk, dv, seed, state=True):
    gen = torch.Generator().manual_seed(seed)
    T = sum(lengths)
    q = torch.randn(T, Hqk, dk, generator=gen, dtype=torch.float64)
    k = torch.randn(T, Hqk, dk, generator=gen, dtype=torch.float64)
    v = torch.randn(T, Hv, dv, generator=gen, dtype=torch.float64)
    g = torch.nn.functional.logsigmoid(torch.randn(T, Hv, generator=gen, dtype=torch.float64) + 1.0)
    beta = torch.sigmoid(torch.randn(T, Hv, generator=gen, dtype=torch.float64))
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    s0 = torch.randn(len(lengths), Hv, dv, dk, generator=gen, dtype=torch.float64) * 0.3 if state else None
    return q, k, v, g, beta, s0, cu


def test_matches_explicit_matrix_brute_force():
    # d_k != d_v, GQA 2:1, varlen with an empty and a one-token sequence, nonzero state
    args = _rand_inputs([5, 17, 0, 1, 9], Hqk=2, Hv=4, dk=8, dv=6, seed=1)
    o, s = oracle.prefill(*args)
    ob, sb = _brute.brute_prefill(*args)
    np.testing.assert_allclose(o, ob, rtol=0, atol=1e-12)
    np.testing.assert_allclose(s, sb, rtol=0, atol=1e-12)


@pytest.mark.parametrize("C", [1, 4, 16, 64])
def test_chunked_wy_form_matches_sequential(C):
    args = _rand_inputs([37, 16, 5, 64, 65], Hqk=1, Hv=2, dk=16, dv=12, seed=2)
    o, s = oracle.prefill(*args)
    oc, sc = _brute.chunked_prefill(*args, C=C)
    np.testing.assert_allclose(o, oc, rtol=0, atol=1e-10)
    np.testing.assert_allclose(s, sc, rtol=0, atol=1e-10)


def test_handworked_example():
    with open(os.path.join(HERE, "golden", "handworked_d2_t2.json")) as f:
        gold = json.load(f)
    q = np.array(gold["q"])[:, None, :]
    k = np.array(gold["k"])[:, None, :]
    v = np.array(gold["v"])[:, None, :]
    g = np.log(np.array(gold["alpha"]))[:, None]
    beta = np.array(gold["beta"])[:, None]
    o, s = oracle.prefill(q, k, v, g, beta, None, [0, 2], scale=gold["scale"], eps=gold["eps"])
    np.testing.assert_allclose(o[:, 0, :], gold["o"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(s[0, 0], gold["S_final"], rtol=0, atol=1e-14)


def test_closed_form_pure_decay_when_beta_zero():
    q, k, v, g, beta, s0, cu = _rand_inputs([23], 1, 1, 8, 8, seed=3)
    beta = torch.zeros_like(beta)
    o, s = oracle.prefill(q, k, v, g, beta, s0, cu)
    G = np.cumsum(g.numpy()[:, 0])
    S0 = s0.numpy()[0, 0]
    np.testing.assert_allclose(s[0, 0], np.exp(G[-1]) * S0, rtol=1e-13, atol=0)
    qn = q.numpy()[:, 0]
    qh = qn / np.sqrt((qn ** 2).sum(1, keepdims=True) + oracle.EPS) * 8 ** -0.5
    expect = np.exp(G)[:, None] * (qh @ S0.T)
    np.testing.assert_allclose(o[:, 0], expect, rtol=1e-12, atol=1e-15)


def test_closed_form_associative_recall_orthonormal_keys():
    # alpha = beta = 1, keys e_0..e_{d-1}, S_0 = 0: S = sum_t v_t e_t^T, and the
    # query e_s reads back v_s exactly (times the query scale).
    d = 8
    T = d
    k = np.eye(d)[:, None, :]
    v = np.random.default_rng(4).normal(size=(T, 1, d))
    q = np.eye(d)[[3, 0, 7, 5, 1, 2, 6, 4]][:, None, :]
    g = np.zeros((T, 1))
    beta = np.ones((T, 1))
    o, s = oracle.prefill(q, k, v, g, beta, None, [0, T], scale=1.0, eps=0.0)
    np.testing.assert_allclose(s[0, 0], v[:, 0, :].T, atol=1e-15)
    # at the last token every key has been written: query e_s returns v_s
    assert np.allclose(o[-1, 0], v[4, 0], atol=1e-15)


def test_closed_form_repeated_key_overwrites():
    # alpha = beta = 1 and one key k repeated: S_T = S_0 (I - k k^T) + v_T k^T
    d = 6
    rng = np.random.default_rng(5)
    kk = rng.normal(size=d)
    T = 4
    k = np.tile(kk, (T, 1))[:, None, :]
    v = rng.normal(size=(T, 1, d))
    q = rng.normal(size=(T, 1, d))
    S0 = rng.normal(size=(1, 1, d, d))
    o, s = oracle.prefill(q, k, v, np.zeros((T, 1)), np.ones((T, 1)), S0, [0, T], eps=0.0)
    kh = kk / np.linalg.norm(kk)
    expect = S0[0, 0] @ (np.eye(d) - np.outer(kh, kh)) + np.outer(v[-1, 0], kh)
    np.testing.assert_allclose(s[0, 0], expect, atol=1e-13)


def test_closed_form_single_token_from_zero_state():
    # T = 1, S_0 = 0: o = beta (k^ . q^) v
    q, k, v, g, beta, _, cu = _rand_inputs([1], 1, 1, 16, 16, seed=6, state=False)
    o, s = oracle.prefill(q, k, v, g, beta, None, cu)
    qn, kn = q.numpy()[0, 0], k.numpy()[0, 0]
    qh = qn / np.sqrt(qn @ qn + oracle.EPS) * 16 ** -0.5
    kh = kn / np.sqrt(kn @ kn + oracle.EPS)
    expect = beta.numpy()[0, 0] * (kh @ qh) * v.numpy()[0, 0]
    np.testing.assert_allclose(o[0, 0], expect, rtol=1e-13)


def test_gqa_value_heads_share_query_key_heads_in_contiguous_groups():
    # Hqk=2, Hv=4: value heads 0,1 read q/k head 0; heads 2,3 read head 1.
    q, k, v, g, beta, s0, cu = _rand_inputs([11], Hqk=2, Hv=4, dk=8, dv=8, seed=7)
    o, s = oracle.prefill(q, k, v, g, beta, s0, cu)
    for h in range(4):
        hq = h // 2
        oh, sh = oracle.prefill(q[:, hq:hq + 1], k[:, hq:hq + 1], v[:, h:h + 1], g[:, h:h + 1],
                                beta[:, h:h + 1], s0[:, h:h + 1], cu)
        np.testing.assert_array_equal(o[:, h:h + 1], oh)
        np.testing.assert_array_equal(s[:, h:h + 1], sh)


def test_varlen_packing_equals_separate_runs():
    lengths = [7, 1, 30, 12]
    q, k, v, g, beta, s0, cu = _rand_inputs(lengths, 2, 4, 8, 8, seed=8)
    o, s = oracle.prefill(q, k, v, g, beta, s0, cu)
    for n in range(len(lengths)):
        a, b = cu[n], cu[n + 1]
        on, sn = oracle.prefill(q[a:b], k[a:b], v[a:b], g[a:b], beta[a:b], s0[n:n + 1], [0, b - a])
        np.testing.assert_array_equal(o[a:b], on)
        np.testing.assert_array_equal(s[n:n + 1], sn)


def test_continuation_from_state_equals_one_run():
    q, k, v, g, beta, s0, cu = _rand_inputs([40], 1, 2, 8, 8, seed=9)
    o, s = oracle.prefill(q, k, v, g, beta, s0, cu)
    o1, s1 = oracle.prefill(q[:17], k[:17], v[:17], g[:17], beta[:17], s0, [0, 17])
    o2, s2 = oracle.prefill(q[17:], k[17:], v[17:], g[17:], beta[17:], s1, [0, 23])
    np.testing.assert_allclose(np.concatenate([o1, o2]), o, atol=1e-14)
    np.testing.assert_allclose(s2, s, atol=1e-14)


def test_decode_steps_equal_prefill():
    T = 12
    q, k, v, g, beta, s0, cu = _rand_inputs([T], 2, 4, 8, 8, seed=10)
    o, s = oracle.prefill(q, k, v, g, beta, s0, cu)
    state = s0.numpy().copy()
    for t in range(T):
        ot, state = oracle.decode(q[t:t + 1], k[t:t + 1], v[t:t + 1], g[t:t + 1], beta[t:t + 1], state)
        np.testing.assert_allclose(ot[0], o[t], atol=1e-14)
    np.testing.assert_allclose(state, s, atol=1e-14)


def test_head_subset_matches_full_run():
    q, k, v, g, beta, s0, cu = _rand_inputs([9, 4], 2, 4, 8, 8, seed=11)
    o, s = oracle.prefill(q, k, v, g, beta, s0, cu)
    op, sp = oracle.prefill(q, k, v, g, beta, s0, cu, heads=(1, 3))
    np.testing.assert_array_equal(op[:, 1:3], o[:, 1:3])
    np.testing.assert_array_equal(sp[:, 1:3], s[:, 1:3])
    assert np.isnan(op[:, 0]).all() and np.isnan(op[:, 3]).all()


def test_norm_bound_invariant():
    # |I - beta k^ k^^T|_2 = 1 for beta in [0,1], |k^| = 1 (eps = 0), so
    # |S_t|_2 <= alpha_t |S_{t-1}|_2 + beta_t |v_t|.
    q, k, v, g, beta, s0, cu = _rand_inputs([1], 1, 1, 8, 8, seed=12)
    S = s0.numpy().copy()
    gen = np.random.default_rng(12)
    for t in range(50):
        qq, kk, vv = (gen.normal(size=(1, 1, 8)) for _ in range(3))
        gg = np.log(gen.uniform(0.2, 1.0, size=(1, 1)))
        bb = gen.uniform(0, 1, size=(1, 1))
        prev = np.linalg.norm(S[0, 0], 2)
        _, S = oracle.decode(qq, kk, vv, gg, bb, S, eps=0.0)
        bound = np.exp(gg[0, 0]) * prev + bb[0, 0] * np.linalg.norm(vv)
        assert np.linalg.norm(S[0, 0], 2) <= bound * (1 + 1e-12)


def test_workload_tiny_oracle_agrees_with_brute_force():
    w = workloads.workload("tiny")
    x = workloads.inputs_for(w)
    o, s = oracle.prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], x["state_in"], x["cu_seqlens"])
    ob, sb = _brute.brute_prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], x["state_in"],
                                  x["cu_seqlens"])
    np.testing.assert_allclose(o, ob, atol=1e-12)
    np.testing.assert_allclose(s, sb, atol=1e-12)


# ---------------------------------------------------------------------------
# planted mistakes: each mutant of the oracle's C source must fail some pin

MUTANTS = {
    "dropped_write_term": ("row[j] = alpha * (row[j] - a * kh[j]) + b * kh[j];",
                           "row[j] = alpha * (row[j] - a * kh[j]);"),
    "wrong_delta_sign": ("row[j] = alpha * (row[j] - a * kh[j]) + b * kh[j];",
                         "row[j] = alpha * (row[j] + a * kh[j]) + b * kh[j];"),
    "decay_not_applied": ("double alpha = exp(g);", "double alpha = 1.0 + 0.0 * g;"),
    "transposed_readout": ("for (int j = 0; j < dk; ++j) acc += row[j] * qh[j];",
                           "for (int j = 0; j < dk; ++j) acc += S[(size_t)j * dk + i] * qh[j];"),
    "query_not_scaled": ("l2_normalise(q, dk, eps, scale, qh);", "l2_normalise(q, dk, eps, 1.0, qh);"),
    "gqa_modulo_mapping": ("int hq = h / group;\n            size_t sbase",
                           "int hq = h % Hqk;\n            size_t sbase"),
    "key_not_normalised": ("l2_normalise(k, dk, eps, 1.0, kh);",
                           "for (int j = 0; j < dk; ++j) kh[j] = k[j];"),
}


def _build_mutant(tmp_path, name):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "gdn_oracle.c")).read()
    old, new = MUTANTS[name]
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    path_c = tmp_path / f"{name}.c"
    path_c.write_text(src.replace(old, new, 1))
    path_so = tmp_path / f"{name}.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-o", str(path_so),
                    str(path_c), "-lm"], check=True)
    return ctypes.CDLL(str(path_so))


def _pins_pass(lib, monkeypatch):
    """Run the sharpest pins against a given compiled oracle; True if all pass."""
    dp = ctypes.POINTER(ctypes.c_double)
    lib.gdn_oracle_prefill.restype = ctypes.c_int
    lib.gdn_oracle_prefill.argtypes = [dp] * 6 + [ctypes.POINTER(ctypes.c_int64)] + \
        [ctypes.c_int] * 5 + [ctypes.c_double] * 2 + [ctypes.c_int] * 2 + [dp, dp, ctypes.c_int]
    lib.gdn_oracle_decode.restype = ctypes.c_int
    lib.gdn_oracle_decode.argtypes = [dp] * 6 + [ctypes.c_int] * 5 + [ctypes.c_double] * 2 + \
        [ctypes.c_int] * 2 + [dp, ctypes.c_int]
    lib.gdn_oracle_max_threads.restype = ctypes.c_int
    monkeypatch.setattr(oracle, "_lib", lib)
    try:
        test_matches_explicit_matrix_brute_force()
        test_handworked_example()
    except AssertionError:
        return False
    return True


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, tmp_path, monkeypatch):
    lib = _build_mutant(tmp_path, name)
    assert not _pins_pass(lib, monkeypatch), f"mutant {name} passed every pin"


def test_unmutated_copy_passes_pins(tmp_path, monkeypatch):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "gdn_oracle.c")).read()
    (tmp_path / "same.c").write_text(src)
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-o",
                    str(tmp_path / "same.so"), str(tmp_path / "same.c"), "-lm"], check=True)
    assert _pins_pass(ctypes.CDLL(str(tmp_path / "same.so")), monkeypatch)


# ------------------------------------------------- bf16-state decode variant ---

def test_round_bf16_is_round_to_nearest_even_through_float():
    """Pinned against torch's float -> bfloat16 conversion (round to nearest
    even) on values of every magnitude, exact ties, subnormals and specials."""
    import torch
    rng = np.random.default_rng(7)
    x = rng.standard_normal(50000) * 10.0 ** rng.uniform(-40, 38, 50000)
    ties = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8), 2.0 ** -130, 0.0, -0.0])
    x = np.concatenate([x, ties])
    got = oracle.round_bf16(x)
    ref = torch.tensor(x).to(torch.float32).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(got, ref)
    # ties go to even: 1 + 2^-8 lies halfway between 1 and 1 + 2^-7 -> 1
    assert got[-6] == 1.0 and got[-5] == 1.0 + 2.0 ** -6
    sp = oracle.round_bf16(np.array([np.inf, -np.inf, np.nan]))
    assert sp[0] == np.inf and sp[1] == -np.inf and np.isnan(sp[2])


def test_bf16_state_decode_reads_o_before_rounding_and_stores_bf16():
    B, Hqk, Hv, d = 2, 1, 2, 16
    rng = np.random.default_rng(11)
    state = oracle.round_bf16(rng.standard_normal((B, Hv, d, d)) * 0.1).reshape(B, Hv, d, d)
    q, k, v = (rng.standard_normal((B, n, d)) for n in (Hqk, Hqk, Hv))
    g = np.log(0.9) * np.ones((B, Hv))
    beta = 0.5 * np.ones((B, Hv))
    s64 = state.copy()
    o64, s64 = oracle.decode(q, k, v, g, beta, s64)
    s16 = state.copy()
    o16, s16 = oracle.decode(q, k, v, g, beta, s16, state_bf16=True)
    assert np.array_equal(o16, o64)                           # o from the unrounded state
    assert np.array_equal(s16, oracle.round_bf16(s64).reshape(s64.shape))
    assert np.array_equal(s16, oracle.round_bf16(s16).reshape(s16.shape))   # representable
    assert not np.array_equal(s16, s64)


# planted mistakes in the bf16 storage path: each must fail a bf16 pin

BF16_MUTANTS = {
    "bf16_truncates": ("u += 0x7fffu + ((u >> 16) & 1u);", "u += 0u;"),
    "bf16_ties_away_from_zero": ("u += 0x7fffu + ((u >> 16) & 1u);", "u += 0x8000u;"),
    "bf16_state_not_rounded": ("if (round_state_bf16) {", "if (0 * round_state_bf16) {"),
}


def _bf16_pins_pass(lib, monkeypatch):
    dp = ctypes.POINTER(ctypes.c_double)
    lib.gdn_oracle_decode_ex.restype = ctypes.c_int
    lib.gdn_oracle_decode_ex.argtypes = [dp] * 6 + [ctypes.c_int] * 5 + [ctypes.c_double] * 2 + \
        [ctypes.c_int] * 2 + [dp, ctypes.c_int, ctypes.c_int]
    lib.gdn_oracle_round_bf16.restype = None
    lib.gdn_oracle_round_bf16.argtypes = [dp, dp, ctypes.c_long]
    monkeypatch.setattr(oracle, "_lib", lib)
    try:
        test_round_bf16_is_round_to_nearest_even_through_float()
        test_bf16_state_decode_reads_o_before_rounding_and_stores_bf16()
    except AssertionError:
        return False
    return True


@pytest.mark.parametrize("name", sorted(BF16_MUTANTS))
def test_bf16_pins_catch_planted_mistake(name, tmp_path, monkeypatch):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "gdn_oracle.c")).read()
    old, new = BF16_MUTANTS[name]
    assert src.count(old) == 1, f"mutation site for {name} not found"
    (tmp_path / f"{name}.c").write_text(src.replace(old, new, 1))
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-o", str(tmp_path / f"{name}.so"),
                    str(tmp_path / f"{name}.c"), "-lm"], check=True)
    assert not _bf16_pins_pass(ctypes.CDLL(str(tmp_path / f"{name}.so")), monkeypatch), \
        f"mutant {name} passed the bf16 pins"


def test_unmutated_copy_passes_bf16_pins(tmp_path, monkeypatch):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "gdn_oracle.c")).read()
    (tmp_path / "same.c").write_text(src)
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-o",
                    str(tmp_path / "same.so"), str(tmp_path / "same.c"), "-lm"], check=True)
    assert _bf16_pins_pass(ctypes.CDLL(str(tmp_path / "same.so")), monkeypatch)
