// Chunked Gated DeltaNet prefill on the sm_100a tensor cores (bf16 inputs,
// d_k = d_v = 128, chunk C = 64, fp32 state).
//
// The Herbert pages prefill the prompt in blocks ("On descend d'un cran",
// section "Ce que fait le moteur") with bf16 data and f32 accumulation ("On
// descend d'un cran : #002 le même compilateur sur un GPU", section "Le
// contrat numérique"), but print no chunk algorithm. This kernel uses the WY
// (UT-transform) form of the gated delta rule. For a chunk of L <= 64 tokens
// entering with state S (rows i0..i0+DVP of the d_v x d_k state), with
// G_r = sum_{s<=r} g_s, gamma_r = exp(G_r), rk_s = 1/|k_s|, rq_r = scale/|q_r|:
//
//   A   = strictly-lower( diag(beta) (exp(G_r - G_s)) o (K^ K^^T) )   64 x 64
//   T   = (I + A)^-1
//   W   = T diag(beta gamma rk) K_raw          U~ = T diag(beta) V_raw
//   U   = U~ - W S^T
//   O   = diag(gamma rq) Q_raw S^T + P U,   P_rs = exp(G_r - G_s) rq_r rk_s q_r.k_s (s <= r)
//   S  <- gamma_L S + U^T diag(exp(G_L - G_s) rk_s) K_raw
//
// The triangular solve is done in blocks of 16: the four diagonal 16 x 16
// unit-lower-triangular blocks are inverted by forward substitution in fp32
// (D = (I + A_d)^-1), and the strictly block-lower rest is folded in with
// N = D A_o, which is nilpotent of order 4, so
//   T = (I + N)^-1 D = E + N^2 E,  E = D - N D,
// three 64 x 64 x 64 tensor-core products.
//
// Every contraction runs on tcgen05 (bf16 operands in 128B-swizzled shared
// memory, fp32 accumulators in TMEM). q, k and v tiles are brought in raw by
// TMA in the swizzled layout the MMA reads: the stacked [k; q] tile serves as
// the K-major operand of [k;q][k;q]^T and of Q_raw S^T, and -- read MN-major --
// as the token-contracted operand of W and of the state update, so k is never
// rewritten; the L2 norms come from the diagonal of [k;q][k;q]^T and are
// folded into scalings of the small 64 x 64 matrices.
//
// One CTA of 128 threads owns one (sequence, value head, slice of DVP state
// rows); rows of S evolve independently, so slices never communicate. The
// fp32 master state lives in registers (thread t holds column t of the
// slice); a bf16 copy in shared memory feeds the MMAs.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace gdn {
namespace tc {

constexpr int kC = 64;     // chunk length
constexpr int kD = 128;    // d_k = d_v
constexpr int kThreads = 128;
constexpr uint32_t kTmemCols = 512;

// TMEM column map (fp32 columns)
constexpr uint32_t kColG = 0;      // [k;q][k;q]^T            M=128, N=128
constexpr uint32_t kColN = 0;      // N, then N D (lanes 0-15) and N^2 (lanes 16-31)  M=64, N=64
constexpr uint32_t kColZ = 64;     // N^2 E                    M=64, N=64
constexpr uint32_t kColW = 128;    // W (lanes 0-15)           M=64, N=128
constexpr uint32_t kColPU = 128;   // P U (lanes 16-31)        M=64, N=DVP
constexpr uint32_t kColU = 256;    // U~ -> U (lanes 0-15), Q_raw S^T (lanes 16-31)   M=64, N=DVP
constexpr uint32_t kColDS = 320;   // dS^T                     M=128, N=DVP

template <int DVP>
struct Smem {
  static constexpr uint32_t kKQ = 0;                       // 2 x 32 KB: [k;q] raw, 2 atom columns of 16 KB
  static constexpr uint32_t kKQBytes = 2 * 16384;
  static constexpr uint32_t kV = 2 * kKQBytes;             // 2 x v raw tile [64][DVP]
  static constexpr uint32_t kVBytes = kC * DVP * 2;
  static constexpr uint32_t kVStride = kVBytes < 1024 ? 1024 : kVBytes;
  static constexpr uint32_t kDm = kV + 2 * kVStride;      // D            [64][64]
  static constexpr uint32_t kAo = kDm + 8192;             // A_o, then N^2
  static constexpr uint32_t kNm = kAo + 8192;             // N, then T_w
  static constexpr uint32_t kEm = kNm + 8192;             // E = D - N D, then T_u
  static constexpr uint32_t kPm = kEm + 8192;             // P
  static constexpr uint32_t kWn = kPm + 8192;             // -W           [64][128]
  static constexpr uint32_t kSb = kWn + 16384;            // S slice bf16 [DVP][128]
  static constexpr uint32_t kSbBytes = DVP * 256;
  static constexpr uint32_t kUb = kSb + (kSbBytes < 1024 ? 1024 : kSbBytes);   // U^T   [DVP][64]
  static constexpr uint32_t kUBytes = DVP * 128 < 1024 ? 1024 : DVP * 128;
  static constexpr uint32_t kUsb = kUb + kUBytes;          // U_s^T [DVP][64]
  static constexpr uint32_t kAd = kUsb + kUBytes;          // 4 diagonal blocks of A, fp32 [4][16][16]
  static constexpr uint32_t kVec = kAd + 4 * 16 * 16 * 4;  // G, beta, rk, rq, scan scratch
  static constexpr uint32_t kBar = kVec + 5 * 64 * 4;      // mbarriers: tma[2], mma
  static constexpr uint32_t kTmemSlot = kBar + 3 * 8;
  static constexpr uint32_t kFlags = kTmemSlot + 8;
  static constexpr uint32_t kTotal = kFlags + 16;
  static constexpr uint32_t kAlloc = kTotal + 1024;        // slack for 1024-byte alignment
};

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}
__device__ __forceinline__ void st_shared_b16(uint32_t addr, __nv_bfloat16 v) {
  asm volatile("st.shared.b16 [%0], %1;" ::"r"(addr), "h"(*reinterpret_cast<unsigned short*>(&v))
               : "memory");
}
__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

using sm100::sw128_off;

// Write 64 fp32 values as one 64-element bf16 row (8 swizzled chunks) of a
// 128B-swizzled [rows][64] tile.
__device__ __forceinline__ void store_row64(uint32_t tile, int row, const float* x) {
#pragma unroll
  for (int c = 0; c < 8; ++c) st_shared_v4(tile + sw128_off(row, c * 8, 0), sm100::pack8_bf16(x + 8 * c));
}

template <int DVP>
__global__ void __launch_bounds__(kThreads, 1)
prefill_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                  const __grid_constant__ CUtensorMap vmap, const float* __restrict__ g,
                  const float* __restrict__ beta, const float* state_in,
                  const int32_t* __restrict__ cu_seqlens, int Hqk, int Hv, float scale,
                  __nv_bfloat16* __restrict__ o, float* state_out, int total_T) {
  using L = Smem<DVP>;
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(sm);
  float* vG = reinterpret_cast<float*>(sm + L::kVec);       // [64] cumulative log-decay
  float* vB = vG + 64;                                      // [64] beta
  float* vRk = vB + 64;                                     // [64] 1/|k|
  float* vRq = vRk + 64;                                    // [64] scale/|q|
  float* vScan = vRq + 64;                                  // scan scratch
  uint64_t* bar_tma = reinterpret_cast<uint64_t*>(sm + L::kBar);
  uint64_t* bar_mma = bar_tma + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::kTmemSlot);
  float* Ad = reinterpret_cast<float*>(sm + L::kAd);

  const int part = blockIdx.x, h = blockIdx.y, n = blockIdx.z;
  const int hq = h / (Hv / Hqk);
  const int i0 = part * DVP;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  int t_begin = cu_seqlens[n], t_end = cu_seqlens[n + 1];
  t_end = min(t_end, total_T);
  t_begin = min(max(t_begin, 0), t_end);
  const int nchunks = (t_end - t_begin + kC - 1) / kC;

  if (tid == 0) {
    mbar_init(&bar_tma[0], 1);
    mbar_init(&bar_tma[1], 1);
    mbar_init(bar_mma, 1);
    fence_mbar_init();
    prefetch_tensormap(&qmap);
    prefetch_tensormap(&kmap);
    prefetch_tensormap(&vmap);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tlane = static_cast<uint32_t>(warp * 32) << 16;   // this warp's TMEM lane quarter

  // fp32 master state: thread t holds S[i0 + i][t], i < DVP
  const size_t s_off = ((size_t)n * Hv + h) * kD * kD + (size_t)i0 * kD;
  float Sreg[DVP];
#pragma unroll
  for (int i = 0; i < DVP; ++i) Sreg[i] = state_in ? state_in[s_off + (size_t)i * kD + tid] : 0.f;
  const uint32_t sSb = sbase + L::kSb;
#pragma unroll
  for (int i = 0; i < DVP; ++i) st_shared_b16(sSb + sw128_off(i, tid, DVP * 128), __float2bfloat16_rn(Sreg[i]));

  auto issue_tma = [&](int ci) {
    const int slot = ci & 1;
    const int c0 = t_begin + ci * kC;
    uint8_t* kq = sm + L::kKQ + slot * L::kKQBytes;
    mbar_arrive_expect_tx(&bar_tma[slot], 4 * 8192 + L::kVBytes);
    tma_load_3d(kq, &kmap, &bar_tma[slot], 0, hq, c0);
    tma_load_3d(kq + 16384, &kmap, &bar_tma[slot], 64, hq, c0);
    tma_load_3d(kq + 8192, &qmap, &bar_tma[slot], 0, hq, c0);
    tma_load_3d(kq + 16384 + 8192, &qmap, &bar_tma[slot], 64, hq, c0);
    tma_load_3d(sm + L::kV + slot * L::kVStride, &vmap, &bar_tma[slot], i0, h, c0);
  };
  if (tid == 0) {
    if (nchunks > 0) issue_tma(0);
    if (nchunks > 1) issue_tma(1);
  }

  uint32_t mma_phase = 0;
  uint32_t tma_phase[2] = {0, 0};
  bool abort = false;

  // Wait for the MMA barrier; a timeout anywhere aborts the whole CTA.
  auto wait_mma = [&]() -> bool {
    bool ok = mbar_wait(bar_mma, mma_phase);
    mma_phase ^= 1;
    ok = __syncthreads_and(ok);
    tc_fence_after();
    return ok;
  };
  // Make this thread's shared-memory and TMEM reads/writes visible before an MMA issue.
  auto publish = [&]() {
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  };

  constexpr uint32_t kIdG = idesc_bf16(128, 128, false, false);
  constexpr uint32_t kId64 = idesc_bf16(64, 64, false, true);      // K-major A, MN-major B
  constexpr uint32_t kIdW = idesc_bf16(64, 128, false, true);
  constexpr uint32_t kIdU = idesc_bf16(64, DVP, false, true);
  constexpr uint32_t kIdChain = idesc_bf16(64, DVP, false, false);
  constexpr uint32_t kIdDS = idesc_bf16(128, DVP, true, false);
  constexpr uint32_t kVRow = DVP * 2;   // bytes per v row (swizzle width)

  for (int ci = 0; ci < nchunks && !abort; ++ci) {
    const int slot = ci & 1;
    const int c0 = t_begin + ci * kC;
    const int Lc = min(kC, t_end - c0);
    const uint32_t sKQ = sbase + L::kKQ + slot * L::kKQBytes;
    const uint32_t sV = sbase + L::kV + slot * L::kVStride;

    // ---- gates: cumulative log-decay and beta (rows >= Lc are padding) ----
    if (tid < 64) {
      const bool valid = tid < Lc;
      float gv = valid ? g[(size_t)(c0 + tid) * Hv + h] : 0.f;
      const float bv = valid ? beta[(size_t)(c0 + tid) * Hv + h] : 0.f;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float up = __shfl_up_sync(0xffffffffu, gv, off);
        if (lane >= off) gv += up;
      }
      if (lane == 31) vScan[warp] = gv;
      vB[tid] = bv;
      vG[tid] = gv;
    }
    {
      bool ok = mbar_wait(&bar_tma[slot], tma_phase[slot]);
      tma_phase[slot] ^= 1;
      if (!__syncthreads_and(ok)) { abort = true; break; }
    }
    if (tid >= 32 && tid < 64) vG[tid] += vScan[0];

    // ---- [k;q][k;q]^T : KK^T (rows 0-63), QK^T (rows 64-127), norms on the diagonal ----
    if (tid == 0) {
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_bf16(tmem + kColG, desc_kmajor(sKQ, kk, 16384), desc_kmajor(sKQ, kk, 16384), kIdG, kk > 0);
      mma_commit(bar_mma);
    }
    if (!wait_mma()) { abort = true; break; }

    float row[64];
    {
      float tmp[32];
      tmem_ld32(tmem + tlane + kColG, tmp);
#pragma unroll
      for (int j = 0; j < 32; ++j) row[j] = tmp[j];
      tmem_ld32(tmem + tlane + kColG + 32, tmp);
#pragma unroll
      for (int j = 0; j < 32; ++j) row[32 + j] = tmp[j];
      // own squared norm: column tid of row tid
      float diag = 0.f;
      if (warp < 2) {
#pragma unroll
        for (int j = 0; j < 64; ++j) diag = (j == tid) ? row[j] : diag;
      } else {
        tmem_ld32(tmem + tlane + kColG + 64 + 32 * (warp - 2), tmp);
#pragma unroll
        for (int j = 0; j < 32; ++j) diag = (j == lane) ? tmp[j] : diag;
      }
      const int r = tid & 63;
      const bool valid = r < Lc;
      if (tid < 64) vRk[r] = valid ? 1.0f / sqrtf(diag + kNormEps) : 0.f;
      else vRq[r] = valid ? scale / sqrtf(diag + kNormEps) : 0.f;
    }
    __syncthreads();

    // ---- A (diagonal blocks fp32, off-diagonal blocks bf16) and P ----
    {
      const int r = tid & 63;
      const float Gr = vG[r];
      if (tid < 64) {
        const float fr = vB[r] * vRk[r];
        const int b = r >> 4;
        float a[64];
#pragma unroll
        for (int s = 0; s < 64; ++s) a[s] = (s < r) ? fr * vRk[s] * expf(Gr - vG[s]) * row[s] : 0.f;
        // diagonal block (fp32, for the forward substitution)
#pragma unroll
        for (int bb = 0; bb < 4; ++bb) {
          if (bb == b) {
#pragma unroll
            for (int s = 0; s < 16; ++s) Ad[(bb * 16 + (r & 15)) * 16 + s] = a[bb * 16 + s];
          }
        }
        // A_o: blocks strictly left of the diagonal block
        float ao[64];
#pragma unroll
        for (int s = 0; s < 64; ++s) ao[s] = (s < 16 * b) ? a[s] : 0.f;
        store_row64(sbase + L::kAo, r, ao);
      } else {
        const float fr = vRq[r];
        float p[64];
#pragma unroll
        for (int s = 0; s < 64; ++s) p[s] = (s <= r) ? fr * vRk[s] * expf(Gr - vG[s]) * row[s] : 0.f;
        store_row64(sbase + L::kPm, r, p);
      }
    }
    __syncthreads();

    // ---- D = (I + A_d)^-1, one column of one diagonal block per thread ----
    if (tid < 64) {
      const int b = tid >> 4, j = tid & 15;
      const float* Ab = Ad + b * 256;
      float x[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        float acc = 0.f;
#pragma unroll
        for (int k2 = 0; k2 < i; ++k2) acc = fmaf(Ab[i * 16 + k2], x[k2], acc);
        x[i] = (i == j) ? 1.f : (i > j ? -acc : 0.f);
      }
#pragma unroll
      for (int i = 0; i < 16; ++i)
        st_shared_b16(sbase + L::kDm + sw128_off(16 * b + i, 16 * b + j, 0), __float2bfloat16_rn(x[i]));
    } else {
      // zero the off-diagonal blocks of D
      const int r = tid - 64, b = r >> 4;
#pragma unroll
      for (int c = 0; c < 8; ++c)
        if ((c >> 1) != b) st_shared_v4(sbase + L::kDm + sw128_off(r, 8 * c, 0), make_uint4(0, 0, 0, 0));
    }
    publish();

    // ---- N = D A_o ----
    if (tid == 0) {
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16(tmem + kColN, desc_kmajor(sbase + L::kDm, kk, 0),
                 desc_mnmajor(sbase + L::kAo, kk, 128, 8192), kId64, kk > 0);
      mma_commit(bar_mma);
    }
    if (!wait_mma()) { abort = true; break; }
    {
      float tmp[32];
      float v[64];
      tmem_ld32(tmem + tlane + kColN, tmp);
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = tmp[j];
      tmem_ld32(tmem + tlane + kColN + 32, tmp);
#pragma unroll
      for (int j = 0; j < 32; ++j) v[32 + j] = tmp[j];
      if (lane < 16) store_row64(sbase + L::kNm, warp * 16 + lane, v);
    }
    publish();

    // ---- N D (lanes 0-15) and N^2 (lanes 16-31) ----
    if (tid == 0) {
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16(tmem + kColN, desc_kmajor(sbase + L::kNm, kk, 0),
                 desc_mnmajor(sbase + L::kDm, kk, 128, 8192), kId64, kk > 0);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16(tmem + (16u << 16) + kColN, desc_kmajor(sbase + L::kNm, kk, 0),
                 desc_mnmajor(sbase + L::kNm, kk, 128, 8192), kId64, kk > 0);
      mma_commit(bar_mma);
    }
    if (!wait_mma()) { abort = true; break; }
    float E[64];   // lanes 0-15: row of E = D - N D (fp32)
    {
      float tmp[32];
      tmem_ld32(tmem + tlane + kColN, tmp);
#pragma unroll
      for (int j = 0; j < 32; ++j) E[j] = tmp[j];
      tmem_ld32(tmem + tlane + kColN + 32, tmp);
#pragma unroll
      for (int j = 0; j < 32; ++j) E[32 + j] = tmp[j];
      const int r = warp * 16 + (lane & 15);
      if (lane < 16) {
        // E = D - N D, with D read back from its bf16 tile
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 dv = ld_shared_v4(sbase + L::kDm + sw128_off(r, 8 * c, 0));
          const __nv_bfloat162* d2 = reinterpret_cast<const __nv_bfloat162*>(&dv);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 df = __bfloat1622float2(d2[e]);
            E[8 * c + 2 * e] = df.x - E[8 * c + 2 * e];
            E[8 * c + 2 * e + 1] = df.y - E[8 * c + 2 * e + 1];
          }
        }
        store_row64(sbase + L::kEm, r, E);
      } else {
        store_row64(sbase + L::kAo, r, E);   // N^2 (A_o no longer needed)
      }
    }
    publish();

    // ---- Z = N^2 E ;  T = E + Z ----
    if (tid == 0) {
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16(tmem + kColZ, desc_kmajor(sbase + L::kAo, kk, 0),
                 desc_mnmajor(sbase + L::kEm, kk, 128, 8192), kId64, kk > 0);
      mma_commit(bar_mma);
    }
    if (!wait_mma()) { abort = true; break; }
    {
      float tmp[32];
      float tw[64], tu[64];
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        tmem_ld32(tmem + tlane + kColZ + 32 * half, tmp);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int s = 32 * half + j;
          const float t = E[s] + tmp[j];
          const float bs = vB[s];
          tu[s] = t * bs;
          tw[s] = t * bs * expf(vG[s]) * vRk[s];
        }
      }
      if (lane < 16) {
        const int r = warp * 16 + lane;
        store_row64(sbase + L::kNm, r, tw);   // T_w (N no longer needed)
        store_row64(sbase + L::kEm, r, tu);   // T_u (E no longer needed)
      }
    }
    publish();

    // ---- W = T_w K_raw  (M=64, N=128) ;  U~ = T_u V_raw (M=64, N=DVP) ----
    if (tid == 0) {
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16(tmem + kColW, desc_kmajor(sbase + L::kNm, kk, 0), desc_mnmajor(sKQ, kk, 128, 16384), kIdW,
                 kk > 0);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16(tmem + kColU, desc_kmajor(sbase + L::kEm, kk, 0), desc_mnmajor(sV, kk, kVRow, L::kVBytes),
                 kIdU, kk > 0);
      mma_commit(bar_mma);
    }
    if (!wait_mma()) { abort = true; break; }
    {
      float tmp[32];
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        tmem_ld32(tmem + tlane + kColW + 32 * q4, tmp);
        if (lane < 16) {
          const int r = warp * 16 + lane;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            float x[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) x[e] = -tmp[8 * c + e];
            st_shared_v4(sbase + L::kWn + sw128_off(r, 32 * q4 + 8 * c, 8192), pack8_bf16(x));
          }
        }
      }
    }
    publish();

    // ---- chain: U = U~ + (-W) S^T (lanes 0-15) ; Q_raw S^T (lanes 16-31) ----
    if (tid == 0) {
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_bf16(tmem + kColU, desc_kmajor(sbase + L::kWn, kk, 8192), desc_kmajor(sSb, kk, DVP * 128),
                 kIdChain, 1);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_bf16(tmem + (16u << 16) + kColU, desc_kmajor(sKQ + 8192, kk, 16384),
                 desc_kmajor(sSb, kk, DVP * 128), kIdChain, kk > 0);
      mma_commit(bar_mma);
    }
    if (!wait_mma()) { abort = true; break; }
    const float GL = vG[Lc - 1];
    float oq[DVP];   // lanes 16-31: gamma_r rq_r (Q_raw S^T)_r
    {
      float uv[DVP];
      if constexpr (DVP == 16) {
        tmem_ld16(tmem + tlane + kColU, uv);
      } else {
#pragma unroll
        for (int q32 = 0; q32 < DVP / 32; ++q32) {
          float tmp[32];
          tmem_ld32(tmem + tlane + kColU + 32 * q32, tmp);
#pragma unroll
          for (int j = 0; j < 32; ++j) uv[32 * q32 + j] = tmp[j];
        }
      }
      const int r = warp * 16 + (lane & 15);
      if (lane < 16) {
        const float us = expf(GL - vG[r]) * vRk[r];
#pragma unroll
        for (int i = 0; i < DVP; ++i) {
          st_shared_b16(sbase + L::kUb + sw128_off(i, r, 0), __float2bfloat16_rn(uv[i]));
          st_shared_b16(sbase + L::kUsb + sw128_off(i, r, 0), __float2bfloat16_rn(uv[i] * us));
        }
      } else {
        const float rho = expf(vG[r]) * vRq[r];
#pragma unroll
        for (int i = 0; i < DVP; ++i) oq[i] = rho * uv[i];
      }
    }
    publish();

    // ---- chain: P U (lanes 16-31) ; dS^T = K_raw^T U_s (M=128) ----
    if (tid == 0) {
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16(tmem + (16u << 16) + kColPU, desc_kmajor(sbase + L::kPm, kk, 0),
                 desc_kmajor(sbase + L::kUb, kk, 0), kIdChain, kk > 0);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16(tmem + kColDS, desc_mnmajor(sKQ, kk, 128, 16384), desc_kmajor(sbase + L::kUsb, kk, 0),
                 kIdDS, kk > 0);
      mma_commit(bar_mma);
    }
    if (!wait_mma()) { abort = true; break; }
    {
      float pu[DVP], ds[DVP];
      if constexpr (DVP == 16) {
        tmem_ld16(tmem + tlane + kColPU, pu);
        tmem_ld16(tmem + tlane + kColDS, ds);
      } else {
#pragma unroll
        for (int q32 = 0; q32 < DVP / 32; ++q32) {
          float tmp[32];
          tmem_ld32(tmem + tlane + kColPU + 32 * q32, tmp);
#pragma unroll
          for (int j = 0; j < 32; ++j) pu[32 * q32 + j] = tmp[j];
          tmem_ld32(tmem + tlane + kColDS + 32 * q32, tmp);
#pragma unroll
          for (int j = 0; j < 32; ++j) ds[32 * q32 + j] = tmp[j];
        }
      }
      if (lane >= 16) {
        const int r = warp * 16 + lane - 16;
        if (r < Lc) {
          __nv_bfloat16* orow = o + ((size_t)(c0 + r) * Hv + h) * kD + i0;
#pragma unroll
          for (int c = 0; c < DVP / 8; ++c) {
            float x[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) x[e] = oq[8 * c + e] + pu[8 * c + e];
            *reinterpret_cast<uint4*>(orow + 8 * c) = pack8_bf16(x);
          }
        }
      }
      const float gL = expf(GL);
#pragma unroll
      for (int i = 0; i < DVP; ++i) {
        Sreg[i] = fmaf(gL, Sreg[i], ds[i]);
        st_shared_b16(sSb + sw128_off(i, tid, DVP * 128), __float2bfloat16_rn(Sreg[i]));
      }
    }
    publish();
    // the raw tiles of this slot are free (every MMA reading them completed)
    if (tid == 0 && ci + 2 < nchunks) issue_tma(ci + 2);
  }

  if (abort) {
    // drain any TMA still landing in shared memory before the CTA exits (bounded)
    if (tid == 0) {
      for (int s = 0; s < 2; ++s) mbar_wait(&bar_tma[s], tma_phase[s], 100000000ll);
    }
    __syncthreads();
  } else {
#pragma unroll
    for (int i = 0; i < DVP; ++i) state_out[s_off + (size_t)i * kD + tid] = Sreg[i];
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace tc
}  // namespace gdn
