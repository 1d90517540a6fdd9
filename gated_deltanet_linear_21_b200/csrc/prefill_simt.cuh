// Chunked Gated DeltaNet prefill in fp32 SIMT arithmetic (any supported
// head size, fp32 or bf16 I/O). It serves the workloads whose precision or
// shape the tensor-core kernel does not cover (fp32 inputs checked at 1e-4,
// small heads).
//
// Chunk form of the gated delta rule, derived by unrolling the recurrence
// S_t = alpha_t S_{t-1} + u_t k^_t^T with u_t = beta_t (v_t - alpha_t S_{t-1} k^_t)
// over a chunk of L tokens entering with state S (G_r = sum_{s<=r} g_s,
// gamma_r = exp(G_r)):
//
//   A_rs = beta_r exp(G_r - G_s) (k^_r . k^_s)      s < r   (strictly lower)
//   (I + A) W  = diag(beta gamma) K^                forward substitution
//   (I + A) U~ = diag(beta) V
//   U = U~ - W S^T
//   o_r = gamma_r S q^_r + sum_{s<=r} exp(G_r - G_s) (q^_r . k^_s) u_s
//   S  <- gamma_L S + sum_s exp(G_L - G_s) u_s k^_s^T
//
// The pages prefill "in blocks" ("On descend d'un cran", section "Ce que fait
// le moteur") but give no chunk algorithm; this is the standard WY (UT
// transform) form of the delta rule, and the host tests check it against the
// token-by-token fp64 oracle.
//
// One CTA owns one (sequence, value head, slice of dvp state rows); rows of
// S evolve independently, so slices need no communication.
#pragma once

#include "common.cuh"

namespace gdn {

struct SimtSmem {
  // offsets in floats into dynamic shared memory
  int Q, K, W, U, A, P, S, G, B, total;
  __host__ __device__ SimtSmem(int C, int dk, int dvp) {
    Q = 0;
    K = Q + C * dk;
    W = K + C * dk;
    U = W + C * dk;
    A = U + C * dvp;
    P = A + C * C;
    S = P + C * C;
    G = S + dvp * dk;
    B = G + C;
    total = B + C;
  }
};

// grid: (dv / dvp, Hv, n_seqs); block 256; dynamic smem SimtSmem(C, dk, dvp).total floats
template <typename TIO>
__global__ void __launch_bounds__(256)
prefill_simt_kernel(const TIO* __restrict__ q, const TIO* __restrict__ k,
                    const TIO* __restrict__ v, const float* __restrict__ g,
                    const float* __restrict__ beta, const float* state_in,
                    const int32_t* __restrict__ cu_seqlens, int Hqk, int Hv, int dk,
                    int dv, int dvp, int C, float scale, TIO* __restrict__ o,
                    float* state_out, long long total_T) {
  extern __shared__ float sm[];
  const SimtSmem L_(C, dk, dvp);
  float* Qs = sm + L_.Q;   // [C][dk]  q^ (scaled)
  float* Ks = sm + L_.K;   // [C][dk]  k^
  float* Ws = sm + L_.W;   // [C][dk]  W
  float* Us = sm + L_.U;   // [C][dvp] U~ then U
  float* As = sm + L_.A;   // [C][C]   A (strictly lower)
  float* Ps = sm + L_.P;   // [C][C]   exp(G_r-G_s) q^_r.k^_s, s <= r
  float* Ss = sm + L_.S;   // [dvp][dk] state slice
  float* Gs = sm + L_.G;   // [C] cumulative log-decay
  float* Bs = sm + L_.B;   // [C] beta

  const int part = blockIdx.x, h = blockIdx.y, n = blockIdx.z;
  const int hq = h / (Hv / Hqk);
  const int i0 = part * dvp;
  const int tid = threadIdx.x, nthr = blockDim.x;
  const int lane = tid & 31, warp = tid >> 5, nwarp = nthr >> 5;

  // a cu_seqlens that breaks its rules never makes a token outside [0, total_T) read
  long long t_begin = cu_seqlens[n], t_end = cu_seqlens[n + 1];
  if (t_end > total_T) t_end = total_T;
  if (t_begin < 0) t_begin = 0;
  if (t_begin > t_end) t_begin = t_end;

  const size_t sbase = ((size_t)n * Hv + h) * (size_t)dv * dk + (size_t)i0 * dk;
  for (int e = tid; e < dvp * dk; e += nthr)
    Ss[e] = state_in ? state_in[sbase + e] : 0.f;

  for (long long c0 = t_begin; c0 < t_end; c0 += C) {
    const int L = (int)min((long long)C, t_end - c0);
    __syncthreads();  // previous chunk done with every buffer
    // --- load and L2-normalise q, k rows (one warp per row) ---
    for (int r = warp; r < C; r += nwarp) {
      float ssq = 0.f, ssk = 0.f;
      const TIO* qr = q + ((size_t)(c0 + r) * Hqk + hq) * dk;
      const TIO* kr = k + ((size_t)(c0 + r) * Hqk + hq) * dk;
      for (int j = lane; j < dk; j += 32) {
        float qv = r < L ? to_f32(qr[j]) : 0.f;
        float kv = r < L ? to_f32(kr[j]) : 0.f;
        Qs[r * dk + j] = qv;
        Ks[r * dk + j] = kv;
        ssq += qv * qv;
        ssk += kv * kv;
      }
      ssq = group_sum<32>(ssq);
      ssk = group_sum<32>(ssk);
      const float qinv = scale / sqrtf(ssq + kNormEps);
      const float kinv = 1.0f / sqrtf(ssk + kNormEps);
      for (int j = lane; j < dk; j += 32) {
        Qs[r * dk + j] *= qinv;
        Ks[r * dk + j] *= kinv;
      }
    }
    for (int e = tid; e < C * dvp; e += nthr) {
      const int r = e / dvp, i = e - r * dvp;
      Us[e] = r < L ? to_f32(v[((size_t)(c0 + r) * Hv + h) * dv + i0 + i]) : 0.f;
    }
    for (int r = tid; r < C; r += nthr) {
      Gs[r] = r < L ? g[(size_t)(c0 + r) * Hv + h] : 0.f;
      Bs[r] = r < L ? beta[(size_t)(c0 + r) * Hv + h] : 0.f;
    }
    __syncthreads();
    if (tid == 0) {  // in-chunk cumulative log-decay
      float acc = 0.f;
      for (int r = 0; r < C; ++r) { acc += Gs[r]; Gs[r] = acc; }
    }
    __syncthreads();
    // --- A (strictly lower) and the decayed q.k matrix (lower incl. diagonal) ---
    for (int e = tid; e < C * C; e += nthr) {
      const int r = e / C, s = e - r * C;
      float a = 0.f, p = 0.f;
      if (s <= r) {
        float kk = 0.f, qk = 0.f;
        for (int j = 0; j < dk; ++j) {
          kk += Ks[r * dk + j] * Ks[s * dk + j];
          qk += Qs[r * dk + j] * Ks[s * dk + j];
        }
        const float dec = expf(Gs[r] - Gs[s]);
        p = dec * qk;
        if (s < r) a = Bs[r] * dec * kk;
      }
      As[e] = a;
      Ps[e] = p;
    }
    // right-hand sides: W <- diag(beta gamma) K^, U~ <- diag(beta) V
    for (int e = tid; e < C * dk; e += nthr) {
      const int r = e / dk;
      Ws[e] = Bs[r] * expf(Gs[r]) * Ks[e];
    }
    __syncthreads();
    for (int e = tid; e < C * dvp; e += nthr) Us[e] *= Bs[e / dvp];
    // --- forward substitution (I + A) X = RHS, row by row ---
    for (int r = 1; r < L; ++r) {
      __syncthreads();
      for (int c = tid; c < dk + dvp; c += nthr) {
        float* X = c < dk ? Ws + c : Us + (c - dk);
        const int ld = c < dk ? dk : dvp;
        float acc = X[r * ld];
        for (int s = 0; s < r; ++s) acc -= As[r * C + s] * X[s * ld];
        X[r * ld] = acc;
      }
    }
    __syncthreads();
    // --- U = U~ - W S^T ---
    for (int e = tid; e < C * dvp; e += nthr) {
      const int r = e / dvp, i = e - r * dvp;
      float acc = 0.f;
      for (int j = 0; j < dk; ++j) acc += Ws[r * dk + j] * Ss[i * dk + j];
      Us[e] -= acc;
    }
    __syncthreads();
    // --- o = diag(gamma) Q S^T + P U ---
    for (int e = tid; e < L * dvp; e += nthr) {
      const int r = e / dvp, i = e - r * dvp;
      float inter = 0.f, intra = 0.f;
      for (int j = 0; j < dk; ++j) inter += Qs[r * dk + j] * Ss[i * dk + j];
      for (int s = 0; s <= r; ++s) intra += Ps[r * C + s] * Us[s * dvp + i];
      o[((size_t)(c0 + r) * Hv + h) * dv + i0 + i] = from_f32<TIO>(expf(Gs[r]) * inter + intra);
    }
    __syncthreads();
    // --- S <- gamma_L S + sum_s exp(G_L - G_s) u_s k^_s^T ---
    const float GL = Gs[L - 1];
    for (int s = tid; s < C; s += nthr) Bs[s] = s < L ? expf(GL - Gs[s]) : 0.f;  // beta no longer needed
    __syncthreads();
    const float gL = expf(GL);
    for (int e = tid; e < dvp * dk; e += nthr) {
      const int i = e / dk, j = e - i * dk;
      float acc = 0.f;
      for (int s = 0; s < L; ++s) acc += Us[s * dvp + i] * Bs[s] * Ks[s * dk + j];
      Ss[e] = gL * Ss[e] + acc;
    }
  }
  __syncthreads();
  for (int e = tid; e < dvp * dk; e += nthr) state_out[sbase + e] = Ss[e];
}

}  // namespace gdn
