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
// One CTA of 256 threads owns one (sequence, value head, slice of DVP state
// rows); rows of S evolve independently, so slices never communicate. Warps
// w and w+4 read the same TMEM lane quarter and split every row epilogue by
// column halves. The fp32 master state lives in registers (thread (q, h)
// holds half h of column 32q+lane of the slice); a bf16 copy in shared memory
// (MN-major, one 16-byte-chunked row per d_k index) feeds the MMAs.
//
// exp(G_r - G_s) is formed as exp(G_r - m) * exp(m - G_s) with m the middle
// of the chunk's decay range, i.e. one exponential per token instead of one
// per matrix entry; chunks whose decay range could leave the fp32 exponent
// range (more than e^160 across the chunk) take an exact per-entry path.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace gdn {
namespace tc {

constexpr int kC = 64;     // chunk length
constexpr int kD = 128;    // d_k = d_v
constexpr int kThreads = 256;
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
  static constexpr uint32_t kVec = kAd + 4 * 16 * 16 * 4;  // G, beta, rk, rq, ck, cw, scan scratch
  static constexpr uint32_t kBar = kVec + 7 * 64 * 4;      // mbarriers: tma[2], mma
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
  constexpr int kHalf = DVP / 2;          // state-slice columns per thread
  constexpr uint32_t kR = DVP * 2;        // bytes per row of the MN-major v / U / S tiles
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(sm);
  float* vG = reinterpret_cast<float*>(sm + L::kVec);       // [64] cumulative log-decay G
  float* vB = vG + 64;                                      // [64] beta
  float* vRk = vB + 64;                                     // [64] 1/|k|
  float* vRq = vRk + 64;                                    // [64] scale/|q|
  float* vCk = vRq + 64;                                    // [64] column factor of A and P
  float* vCw = vCk + 64;                                    // [64] -beta gamma rk (column factor of T_w)
  float* vScan = vCw + 64;                                  // scan scratch / flags
  uint64_t* bar_tma = reinterpret_cast<uint64_t*>(sm + L::kBar);
  uint64_t* bar_mma = bar_tma + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::kTmemSlot);
  float* Ad = reinterpret_cast<float*>(sm + L::kAd);

  const int part = blockIdx.x, h = blockIdx.y, n = blockIdx.z;
  const int hq = h / (Hv / Hqk);
  const int i0 = part * DVP;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qd = warp & 3;                 // TMEM lane quarter
  const int ch = warp >> 2;                // column half
  const int r128 = qd * 32 + lane;         // row of an M=128 accumulator held by this thread
  const int r64 = qd * 16 + (lane & 15);   // row of an M=64 accumulator (lanes 0-15 / 16-31 halves)
  const bool lo16 = lane < 16;

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
  const uint32_t tlane = static_cast<uint32_t>(qd * 32) << 16;

  // fp32 master state: S[i0 + ch*kHalf + j][r128], j < kHalf
  const size_t s_off = ((size_t)n * Hv + h) * kD * kD + (size_t)(i0 + ch * kHalf) * kD + r128;
  float Sreg[kHalf];
#pragma unroll
  for (int j = 0; j < kHalf; ++j) Sreg[j] = state_in ? state_in[s_off + (size_t)j * kD] : 0.f;
  const uint32_t sSb = sbase + L::kSb;
  auto store_state = [&]() {
#pragma unroll
    for (int c = 0; c < kHalf / 8; ++c)
      st_shared_v4(sSb + mn_off<kR>(r128, ch * kHalf + 8 * c), pack8_bf16(Sreg + 8 * c));
  };
  store_state();

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

  // gates of the next chunk are fetched one chunk ahead (threads 0-63)
  float g_next = 0.f, b_next = 0.f;
  auto fetch_gates = [&](int ci) {
    const int c0 = t_begin + ci * kC;
    const bool valid = ci < nchunks && c0 + tid < t_end;
    g_next = valid ? g[(size_t)(c0 + tid) * Hv + h] : 0.f;
    b_next = valid ? beta[(size_t)(c0 + tid) * Hv + h] : 0.f;
  };
  if (tid < 64) fetch_gates(0);

  uint32_t mma_phase = 0;
  uint32_t tma_phase[2] = {0, 0};
  bool abort = false;

  auto wait_mma = [&]() -> bool {
    bool ok = mbar_wait(bar_mma, mma_phase);
    mma_phase ^= 1;
    ok = __syncthreads_and(ok);
    tc_fence_after();
    return ok;
  };
  auto publish = [&]() {
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  };

  constexpr uint32_t kIdG = idesc_bf16(128, 128, false, false);
  constexpr uint32_t kId64 = idesc_bf16(64, 64, false, true);      // K-major A, MN-major B
  constexpr uint32_t kIdW = idesc_bf16(64, 128, false, true);
  constexpr uint32_t kIdSlice = idesc_bf16(64, DVP, false, true);
  constexpr uint32_t kIdDS = idesc_bf16(128, DVP, true, true);

  for (int ci = 0; ci < nchunks && !abort; ++ci) {
    const int slot = ci & 1;
    const int c0 = t_begin + ci * kC;
    const int Lc = min(kC, t_end - c0);
    const uint32_t sKQ = sbase + L::kKQ + slot * L::kKQBytes;
    const uint32_t sV = sbase + L::kV + slot * L::kVStride;

    // ---- gates: inclusive scan of g, beta; next chunk's gates prefetched ----
    if (tid < 64) {
      float gv = g_next;
      const float bv = b_next;
      const unsigned nonpos = __ballot_sync(0xffffffffu, gv <= 0.f);
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float up = __shfl_up_sync(0xffffffffu, gv, off);
        if (lane >= off) gv += up;
      }
      if (lane == 31) vScan[warp] = gv;
      if (lane == 0) vScan[2 + warp] = nonpos == 0xffffffffu ? 1.f : 0.f;
      vB[tid] = bv;
      vG[tid] = gv;
      fetch_gates(ci + 1);
    }
    {
      bool ok = mbar_wait(&bar_tma[slot], tma_phase[slot]);
      tma_phase[slot] ^= 1;
      if (!__syncthreads_and(ok)) { abort = true; break; }
    }
    if (tid >= 32 && tid < 64) vG[tid] += vScan[0];

    // ---- [k;q][k;q]^T : KK^T (rows 0-63), QK^T (rows 64-127), squared norms on the diagonal ----
    if (tid == 0) {
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_bf16(tmem + kColG, desc_kmajor(sKQ, kk, 16384), desc_kmajor(sKQ, kk, 16384), kIdG, kk > 0);
      mma_commit(bar_mma);
    }
    if (!wait_mma()) { abort = true; break; }

    const float G0 = vG[0], GL = vG[Lc - 1];
    const bool fast = vScan[2] > 0.f && vScan[3] > 0.f && (G0 - GL) <= 160.f;
    const float gm = 0.5f * (G0 + GL);   // reference point of the factored decay

    float rowv[32];   // columns 32ch..32ch+31 of row r128
    tmem_ld32(tmem + tlane + kColG + 32 * ch, rowv);
    {
      bool own = false;
      float diag = 0.f;
      if (qd < 2) {
        own = (qd == ch);
#pragma unroll
        for (int j = 0; j < 32; ++j) diag = (j == lane) ? rowv[j] : diag;
      } else if (ch == 0) {
        float tmp[32];
        tmem_ld32(tmem + tlane + kColG + 64 + 32 * (qd - 2), tmp);
#pragma unroll
        for (int j = 0; j < 32; ++j) diag = (j == lane) ? tmp[j] : diag;
        own = true;
      }
      if (own) {
        const int r = r128 & 63;
        const bool valid = r < Lc;
        if (qd < 2) {
          const float rk = valid ? 1.0f / sqrtf(diag + kNormEps) : 0.f;
          const float Gr = vG[r];
          vRk[r] = rk;
          vCk[r] = fast ? expf(gm - Gr) * rk : rk;
          vCw[r] = -vB[r] * expf(Gr) * rk;
        } else {
          vRq[r] = valid ? scale / sqrtf(diag + kNormEps) : 0.f;
        }
      }
    }
    __syncthreads();

    // ---- A (diagonal blocks fp32, off-diagonal blocks bf16) and P, half a row per thread ----
    {
      const int r = r128 & 63;
      const float Gr = vG[r];
      float x[32];
      if (qd < 2) {
        const float fr = vB[r] * vRk[r] * (fast ? expf(Gr - gm) : 1.f);
        if (fast) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int s = 32 * ch + j;
            x[j] = (s < r) ? fr * vCk[s] * rowv[j] : 0.f;
          }
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int s = 32 * ch + j;
            x[j] = (s < r) ? fr * vCk[s] * expf(Gr - vG[s]) * rowv[j] : 0.f;
          }
        }
        const int b = r >> 4;
        if ((b >> 1) == ch) {   // this half holds the diagonal block: keep it in fp32
          float* dst = Ad + (b * 16 + (r & 15)) * 16;
          if (b & 1) {
#pragma unroll
            for (int j = 0; j < 16; ++j) dst[j] = x[16 + j];
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) dst[j] = x[j];
          }
        }
        // A_o: only the blocks strictly left of the diagonal block
#pragma unroll
        for (int j = 0; j < 32; ++j) x[j] = (32 * ch + j < 16 * b) ? x[j] : 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c)
          st_shared_v4(sbase + L::kAo + sw128_off(r, 32 * ch + 8 * c, 0), pack8_bf16(x + 8 * c));
      } else {
        const float fr = vRq[r] * (fast ? expf(Gr - gm) : 1.f);
        if (fast) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int s = 32 * ch + j;
            x[j] = (s <= r) ? fr * vCk[s] * rowv[j] : 0.f;
          }
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int s = 32 * ch + j;
            x[j] = (s <= r) ? fr * vCk[s] * expf(Gr - vG[s]) * rowv[j] : 0.f;
          }
        }
#pragma unroll
        for (int c = 0; c < 4; ++c)
          st_shared_v4(sbase + L::kPm + sw128_off(r, 32 * ch + 8 * c, 0), pack8_bf16(x + 8 * c));
      }
    }
    __syncthreads();

    // ---- D = (I + A_d)^-1: one column of one diagonal block per thread (threads 0-63) ----
    if (tid < 64) {
      const int b = tid >> 4, j = tid & 15;
      const float* Ab = Ad + b * 256;
      float xs[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        float acc = 0.f;
#pragma unroll
        for (int k2 = 0; k2 < i; ++k2) acc = fmaf(Ab[i * 16 + k2], xs[k2], acc);
        xs[i] = (i == j) ? 1.f : (i > j ? -acc : 0.f);
      }
#pragma unroll
      for (int i = 0; i < 16; ++i)
        st_shared_b16(sbase + L::kDm + sw128_off(16 * b + i, 16 * b + j, 0), __float2bfloat16_rn(xs[i]));
    } else {
      // zero the off-diagonal blocks of D: 64 rows x 6 chunks
      for (int e = tid - 64; e < 64 * 6; e += kThreads - 64) {
        const int row = e / 6, idx = e - row * 6, b = row >> 4;
        const int c = idx < 2 * b ? idx : idx + 2;
        st_shared_v4(sbase + L::kDm + sw128_off(row, 8 * c, 0), make_uint4(0, 0, 0, 0));
      }
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
      float v[32];
      tmem_ld32(tmem + tlane + kColN + 32 * ch, v);
      if (lo16) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
          st_shared_v4(sbase + L::kNm + sw128_off(r64, 32 * ch + 8 * c, 0), pack8_bf16(v + 8 * c));
      }
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
    float E[32];   // lanes 0-15: half row of E = D - N D (fp32)
    {
      tmem_ld32(tmem + tlane + kColN + 32 * ch, E);
      if (lo16) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint4 dv = ld_shared_v4(sbase + L::kDm + sw128_off(r64, 32 * ch + 8 * c, 0));
          const __nv_bfloat162* d2 = reinterpret_cast<const __nv_bfloat162*>(&dv);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 df = __bfloat1622float2(d2[e]);
            E[8 * c + 2 * e] = df.x - E[8 * c + 2 * e];
            E[8 * c + 2 * e + 1] = df.y - E[8 * c + 2 * e + 1];
          }
          st_shared_v4(sbase + L::kEm + sw128_off(r64, 32 * ch + 8 * c, 0), pack8_bf16(E + 8 * c));
        }
      } else {
#pragma unroll
        for (int c = 0; c < 4; ++c)   // N^2 (A_o is no longer needed)
          st_shared_v4(sbase + L::kAo + sw128_off(r64, 32 * ch + 8 * c, 0), pack8_bf16(E + 8 * c));
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
      float z[32], tw[32], tu[32];
      tmem_ld32(tmem + tlane + kColZ + 32 * ch, z);
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int s = 32 * ch + j;
        const float t = E[j] + z[j];
        tu[j] = t * vB[s];
        tw[j] = t * vCw[s];   // carries the minus sign: the MMA below yields -W
      }
      if (lo16) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          st_shared_v4(sbase + L::kNm + sw128_off(r64, 32 * ch + 8 * c, 0), pack8_bf16(tw + 8 * c));
          st_shared_v4(sbase + L::kEm + sw128_off(r64, 32 * ch + 8 * c, 0), pack8_bf16(tu + 8 * c));
        }
      }
    }
    publish();

    // ---- -W = -T_w K_raw  (M=64, N=128) ;  U~ = T_u V_raw (M=64, N=DVP) ----
    if (tid == 0) {
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16(tmem + kColW, desc_kmajor(sbase + L::kNm, kk, 0), desc_mnmajor(sKQ, kk, 128, 16384), kIdW,
                 kk > 0);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16(tmem + kColU, desc_kmajor(sbase + L::kEm, kk, 0), desc_mnmajor(sV, kk, kR, L::kVBytes),
                 kIdSlice, kk > 0);
      mma_commit(bar_mma);
    }
    if (!wait_mma()) { abort = true; break; }
    {
      float w[64];
      tmem_ld32(tmem + tlane + kColW + 64 * ch, w);
      tmem_ld32(tmem + tlane + kColW + 64 * ch + 32, w + 32);
      if (lo16) {
#pragma unroll
        for (int c = 0; c < 8; ++c)
          st_shared_v4(sbase + L::kWn + sw128_off(r64, 64 * ch + 8 * c, 8192), pack8_bf16(w + 8 * c));
      }
    }
    publish();

    // ---- chain: U = U~ + (-W) S^T (lanes 0-15) ; Q_raw S^T (lanes 16-31) ----
    if (tid == 0) {
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_bf16(tmem + kColU, desc_kmajor(sbase + L::kWn, kk, 8192), desc_mnmajor(sSb, kk, kR, 128 * kR),
                 kIdSlice, 1);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_bf16(tmem + (16u << 16) + kColU, desc_kmajor(sKQ + 8192, kk, 16384),
                 desc_mnmajor(sSb, kk, kR, 128 * kR), kIdSlice, kk > 0);
      mma_commit(bar_mma);
    }
    if (!wait_mma()) { abort = true; break; }
    float oq[kHalf];   // lanes 16-31: gamma_r rq_r (Q_raw S^T)_r, this thread's column half
    {
      float uv[kHalf];
      tmem_ld<kHalf>(tmem + tlane + kColU + ch * kHalf, uv);
      if (lo16) {
        const float us = expf(GL - vG[r64]) * vRk[r64];
        float usv[kHalf];
#pragma unroll
        for (int j = 0; j < kHalf; ++j) usv[j] = uv[j] * us;
#pragma unroll
        for (int c = 0; c < kHalf / 8; ++c) {
          st_shared_v4(sbase + L::kUb + mn_off<kR>(r64, ch * kHalf + 8 * c), pack8_bf16(uv + 8 * c));
          st_shared_v4(sbase + L::kUsb + mn_off<kR>(r64, ch * kHalf + 8 * c), pack8_bf16(usv + 8 * c));
        }
      } else {
        const float rho = expf(vG[r64]) * vRq[r64];
#pragma unroll
        for (int j = 0; j < kHalf; ++j) oq[j] = rho * uv[j];
      }
    }
    publish();

    // ---- chain: P U (lanes 16-31) ; dS^T = K_raw^T U_s (M=128) ----
    if (tid == 0) {
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16(tmem + (16u << 16) + kColPU, desc_kmajor(sbase + L::kPm, kk, 0),
                 desc_mnmajor(sbase + L::kUb, kk, kR, 64 * kR), kIdSlice, kk > 0);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16(tmem + kColDS, desc_mnmajor(sKQ, kk, 128, 16384), desc_mnmajor(sbase + L::kUsb, kk, kR, 64 * kR),
                 kIdDS, kk > 0);
      mma_commit(bar_mma);
    }
    if (!wait_mma()) { abort = true; break; }
    {
      float pu[kHalf], ds[kHalf];
      tmem_ld<kHalf>(tmem + tlane + kColPU + ch * kHalf, pu);
      tmem_ld<kHalf>(tmem + tlane + kColDS + ch * kHalf, ds);
      if (!lo16 && r64 < Lc) {
        __nv_bfloat16* orow = o + ((size_t)(c0 + r64) * Hv + h) * kD + i0 + ch * kHalf;
#pragma unroll
        for (int c = 0; c < kHalf / 8; ++c) {
          float xo[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) xo[e] = oq[8 * c + e] + pu[8 * c + e];
          *reinterpret_cast<uint4*>(orow + 8 * c) = pack8_bf16(xo);
        }
      }
      const float gL = expf(GL);
#pragma unroll
      for (int j = 0; j < kHalf; ++j) Sreg[j] = fmaf(gL, Sreg[j], ds[j]);
      store_state();
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
    for (int j = 0; j < kHalf; ++j) state_out[s_off + (size_t)j * kD] = Sreg[j];
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
