"""Independent fp64 formulations used to pin the oracle (tests only).

``brute_prefill`` forms the d_k x d_k matrix (I - beta k k^T) explicitly and
multiplies full matrices, token by token: a second, differently written
statement of the gated delta rule S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T)
+ beta_t v_t k_t^T, o_t = S_t q_t.

``chunked_prefill`` is the chunk-parallel (WY / UT-transform) form of the same
recurrence, derived by unrolling it inside a chunk of C tokens with S_0 the
state entering the chunk, G_r = sum_{s<=r} g_s and gamma_r = exp(G_r):

    u_r   = beta_r (v_r - alpha_r S_{r-1} k_r)                 (so S_r = alpha_r S_{r-1} + u_r k_r^T)
    A_rs  = beta_r exp(G_r - G_s) (k_r . k_s)   for s < r, else 0
    T     = (I + A)^-1
    W     = T diag(beta * gamma) K,   U~ = T diag(beta) V
    U     = U~ - W S_0^T
    O     = diag(gamma) Q S_0^T + (M o Q K^T) U,   M_rs = exp(G_r - G_s) for s <= r
    S_C   = gamma_C S_0 + U^T diag(exp(G_C - G_s)) K

It checks the algebra the GPU kernels are built on before any of them exists.
"""
from __future__ import annotations

import numpy as np


def _norm(x, eps, scale=1.0):
    return x / np.sqrt(np.dot(x, x) + eps) * scale


def _f64(x):
    if hasattr(x, "detach"):
        import torch
        return x.detach().to(torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def brute_prefill(q, k, v, g, beta, state_in, cu_seqlens, scale=None, eps=1e-6):
    q, k, v, g, beta = map(_f64, (q, k, v, g, beta))
    cu = [int(c) for c in cu_seqlens]
    T, Hqk, dk = q.shape
    _, Hv, dv = v.shape
    N = len(cu) - 1
    G = Hv // Hqk
    scale = dk ** -0.5 if scale is None else scale
    o = np.zeros((T, Hv, dv))
    s_out = np.zeros((N, Hv, dv, dk))
    eye = np.eye(dk)
    for n in range(N):
        for h in range(Hv):
            hq = h // G
            S = np.zeros((dv, dk)) if state_in is None else _f64(state_in)[n, h].copy()
            for t in range(cu[n], cu[n + 1]):
                qh = _norm(q[t, hq], eps, scale)
                kh = _norm(k[t, hq], eps)
                a, b = np.exp(g[t, h]), beta[t, h]
                S = a * S @ (eye - b * np.outer(kh, kh)) + b * np.outer(v[t, h], kh)
                o[t, h] = S @ qh
            s_out[n, h] = S
    return o, s_out


def chunked_prefill(q, k, v, g, beta, state_in, cu_seqlens, C, scale=None, eps=1e-6):
    q, k, v, g, beta = map(_f64, (q, k, v, g, beta))
    cu = [int(c) for c in cu_seqlens]
    T, Hqk, dk = q.shape
    _, Hv, dv = v.shape
    N = len(cu) - 1
    G = Hv // Hqk
    scale = dk ** -0.5 if scale is None else scale
    o = np.zeros((T, Hv, dv))
    s_out = np.zeros((N, Hv, dv, dk))
    for n in range(N):
        for h in range(Hv):
            hq = h // G
            S = np.zeros((dv, dk)) if state_in is None else _f64(state_in)[n, h].copy()
            for c0 in range(cu[n], cu[n + 1], C):
                c1 = min(c0 + C, cu[n + 1])
                L = c1 - c0
                Q = np.stack([_norm(q[t, hq], eps, scale) for t in range(c0, c1)])
                K = np.stack([_norm(k[t, hq], eps) for t in range(c0, c1)])
                V = v[c0:c1, h]
                b = beta[c0:c1, h]
                Gc = np.cumsum(g[c0:c1, h])
                gam = np.exp(Gc)
                D = Gc[:, None] - Gc[None, :]
                lower = np.tril(np.ones((L, L)), -1)
                A = np.where(lower > 0, b[:, None] * np.exp(np.where(lower > 0, D, 0.0)) * (K @ K.T), 0.0)
                Tm = np.linalg.inv(np.eye(L) + A)
                W = Tm @ (b[:, None] * gam[:, None] * K)
                Ut = Tm @ (b[:, None] * V)
                U = Ut - W @ S.T
                incl = np.tril(np.ones((L, L)))
                M = np.where(incl > 0, np.exp(np.where(incl > 0, D, 0.0)), 0.0)
                O = gam[:, None] * (Q @ S.T) + (M * (Q @ K.T)) @ U
                o[c0:c1, h] = O
                Kt = np.exp(Gc[-1] - Gc)[:, None] * K
                S = gam[-1] * S + U.T @ Kt
            s_out[n, h] = S
    return o, s_out
