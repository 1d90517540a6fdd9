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
//   T   = (I + A)^-1,  T_u = T diag(beta),  T_w = T diag(beta gamma rk)
//   U   = T_u V_raw - T_w (K_raw S^T)                     (= U~ - W S^T)
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
// Every contraction runs on tcgen05 (bf16 operands in swizzled shared memory,
// fp32 accumulators in TMEM). q, k and v tiles arrive raw by TMA in the
// layout the MMA reads: the stacked [k; q] tile is the K-major operand of
// [k;q] k^T and of [k;q] S^T, and -- read MN-major -- the token-contracted
// operand of the state update; k is never rewritten. Norms come from the
// Gram diagonal (k) and a short SIMT pass (q) and are folded into scalings
// of the 64 x 64 matrices.
//
// Software pipeline. On this GPU one tcgen05 issue -> commit -> observe round
// trip costs ~450 cycles whatever its size, so the kernel is bound by serial
// round trips, not by tensor throughput. Each loop iteration therefore
// carries three independent pieces of work and pays three round trips:
//   RT-a : X = [k;q](c) S^T           | Gram(c+2) = [k;q](c+2) k(c+2)^T | [ND | N^2](c+1)
//   RT-b : U(c) = [T_u | -T_w][V ; K S^T] | Z = N^2 E (c+1)         | N = D A_o (c+2)
//   RT-c : P U (c) and dS^T = K^T U_s (c)
// i.e. the state chain of chunk c, the second half of the solve of chunk c+1
// and the Gram / A / P / D work of chunk c+2. The D inverse (SIMT) runs while
// the RT-b tensor work is in flight. k and q tiles are loaded twice by TMA
// (once for the Gram, once for the chain; the second load hits L2), so only
// three raw-tile slots are needed.
//
// One CTA of 256 threads owns one (sequence, value head, slice of DVP state
// rows); rows of S evolve independently, so slices never communicate. Warps
// w and w+4 read the same TMEM lane quarter and split row epilogues by column
// halves. The fp32 master state lives in registers (thread (q, h) holds half
// h of column 32q+lane of the slice); a bf16 copy in shared memory (MN-major,
// one row per d_k index) feeds the MMAs.
//
// exp(G_r - G_s) is formed as exp(G_r - m) * exp(m - G_s) with m the middle
// of the chunk's decay range (one exponential per token, not per entry);
// chunks whose decay range could leave the fp32 exponent range (more than
// e^160 across the chunk) take an exact per-entry path.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace gdn {
namespace tc {

constexpr int kC = 64;     // chunk length
constexpr int kD = 128;    // d_k = d_v
constexpr int kThreads = 256;
constexpr uint32_t kTmemCols = 512;

// TMEM column map (fp32 columns); every region is read within its round trip.
constexpr uint32_t kColX = 0;      // [k;q] S^T          M=128, N=DVP
constexpr uint32_t kColG = 64;     // [k;q] k^T          M=128, N=64
constexpr uint32_t kColS2 = 128;   // N [D | N]          M=64 (lanes 0-15), N=128
constexpr uint32_t kColS13 = 256;  // Z = N^2 E (lanes 0-15), N = D A_o (lanes 16-31)   M=64, N=64
constexpr uint32_t kColU = 320;    // U                  M=64 (lanes 0-15), N=DVP
constexpr uint32_t kColPU = 384;   // [* ; P] U          M=128, N=DVP (rows 64-127 used)
constexpr uint32_t kColDS = 448;   // dS^T               M=128, N=DVP

// Per-chunk vectors, a ring of three (chunks c, c+1, c+2 are in flight).
struct ChunkVec {
  float G[64];    // cumulative log-decay
  float B[64];    // beta
  float Rk[64];   // 1/|k| (0 on padding rows)
  float Rq[64];   // scale/|q| (0 on padding rows)
  float Ck[64];   // column factor of A and P
  float Cw[64];   // -beta gamma rk: column factor of -T_w
  float gm;       // reference point of the factored decay
  int fast;       // factored decay usable
  int len;        // tokens in the chunk
  int pad;
};

template <int DVP>
struct Smem {
  static constexpr uint32_t kR = DVP * 2;                   // bytes per row of MN-major slice tiles
  static constexpr uint32_t kKQP = 0;                        // [k;q] raw tile for the Gram (32 KB)
  static constexpr uint32_t kKQC = 32768;                    // 2 x [k;q] raw tiles for the chain
  static constexpr uint32_t kVKS = kKQC + 2 * 32768;         // 2 x [V ; K S^T]   [128][DVP]
  static constexpr uint32_t kVKSBytes = 128 * kR;
  static constexpr uint32_t kAo = kVKS + 2 * kVKSBytes;      // A_o            [64][64]
  static constexpr uint32_t kP0 = kAo + 8192;                // P ring (each preceded by an 8 KB tile)
  static constexpr uint32_t kEm = kP0 + 8192;                // E = D - N D    [64][64]
  static constexpr uint32_t kP1 = kEm + 8192;
  static constexpr uint32_t kN2 = kP1 + 8192;                // N^2            [64][64]
  static constexpr uint32_t kP2 = kN2 + 8192;
  static_assert(kP1 == kP0 + 16384 && kP2 == kP1 + 16384, "P ring stride");
  static constexpr uint32_t kDm = kP2 + 8192;                // D              [64][64]
  static constexpr uint32_t kNm = kDm + 8192;                // N (right after D: [D | N] is one operand)
  static constexpr uint32_t kTT = kNm + 8192;                // [T_u | -T_w]   [64][128]
  static constexpr uint32_t kUb = kTT + 16384;               // U              [64][DVP]
  static constexpr uint32_t kUsb = kUb + 64 * kR;            // U_s            [64][DVP]
  static constexpr uint32_t kSb = kUsb + 64 * kR;            // S^T slice      [128][DVP]
  static constexpr uint32_t kAd = kSb + 128 * kR;            // diagonal blocks of A, fp32 [4][16][16]
  static constexpr uint32_t kVec = kAd + 4096;               // 3 x ChunkVec
  static constexpr uint32_t kBar = kVec + 3 * sizeof(ChunkVec);   // mbarriers: prep, chain[2], mma
  static constexpr uint32_t kTmemSlot = kBar + 4 * 8;
  static constexpr uint32_t kScan = kTmemSlot + 16;           // scan scratch
  static constexpr uint32_t kTotal = kScan + 64;
  static constexpr uint32_t kAlloc = kTotal + 1024;           // slack for 1024-byte alignment
  static_assert(kAlloc <= 227 * 1024, "shared memory budget");
  static_assert((kVKS % 1024) == 0 && (kAo % 1024) == 0 && (kUb % 1024) == 0, "tile alignment");
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

template <int DVP>
__global__ void __launch_bounds__(kThreads, 1)
prefill_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                  const __grid_constant__ CUtensorMap vmap, const float* __restrict__ g,
                  const float* __restrict__ beta, const float* state_in,
                  const int32_t* __restrict__ cu_seqlens, int Hqk, int Hv, float scale,
                  __nv_bfloat16* __restrict__ o, float* state_out, int total_T) {
  using L = Smem<DVP>;
  using namespace sm100;
  static_assert(DVP == 16 || DVP == 32, "slice width");
  constexpr int kHalf = DVP / 2;          // state-slice columns per thread
  constexpr uint32_t kR = L::kR;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(sm);
  ChunkVec* vecs = reinterpret_cast<ChunkVec*>(sm + L::kVec);
  uint64_t* bar_prep = reinterpret_cast<uint64_t*>(sm + L::kBar);
  uint64_t* bar_chain = bar_prep + 1;   // [2]
  uint64_t* bar_mma = bar_prep + 3;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::kTmemSlot);
  float* scan = reinterpret_cast<float*>(sm + L::kScan);
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
    mbar_init(bar_prep, 1);
    mbar_init(&bar_chain[0], 1);
    mbar_init(&bar_chain[1], 1);
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
  const uint32_t tmem = __shfl_sync(0xffffffffu, *tmem_slot, 0);   // provably warp-uniform
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

  // ---- TMA: the Gram slot and the two chain slots ----
  // (warp-collective: called by every lane of warp 0)
  auto load_kq = [&](uint8_t* kq, uint64_t* bar, int c0, uint32_t extra_bytes) {
    mbar_arrive_expect_tx_warp(bar, 4 * 8192 + extra_bytes);
    tma_load_3d_warp(kq, &kmap, bar, 0, hq, c0);
    tma_load_3d_warp(kq + 16384, &kmap, bar, 64, hq, c0);
    tma_load_3d_warp(kq + 8192, &qmap, bar, 0, hq, c0);
    tma_load_3d_warp(kq + 16384 + 8192, &qmap, bar, 64, hq, c0);
  };
  auto issue_prep_tma = [&](int j) {   // raw [k;q] of chunk j for its Gram
    load_kq(sm + L::kKQP, bar_prep, t_begin + j * kC, 0);
  };
  auto issue_chain_tma = [&](int j) {  // raw [k;q] and v slice of chunk j for its state chain
    const int s = j & 1;
    uint8_t* kq = sm + L::kKQC + s * 32768;
    load_kq(kq, &bar_chain[s], t_begin + j * kC, 64 * kR);
    tma_load_3d_warp(sm + L::kVKS + s * L::kVKSBytes, &vmap, &bar_chain[s], i0, h, t_begin + j * kC);
  };
  if (warp == 0) {
    if (nchunks > 0) { issue_prep_tma(0); issue_chain_tma(0); }
    if (nchunks > 1) issue_chain_tma(1);
  }

  // gates of chunk j are fetched one iteration before their scan (threads 0-63)
  float g_next = 0.f, b_next = 0.f;
  auto fetch_gates = [&](int j) {
    const int c0 = t_begin + j * kC;
    const bool valid = j >= 0 && j < nchunks && c0 + tid < t_end;
    g_next = valid ? g[(size_t)(c0 + tid) * Hv + h] : 0.f;
    b_next = valid ? beta[(size_t)(c0 + tid) * Hv + h] : 0.f;
  };
  if (tid < 64) fetch_gates(0);

  uint32_t mma_phase = 0, prep_phase = 0;
  uint32_t chain_phase[2] = {0, 0};
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

  constexpr uint32_t kIdX = idesc_bf16(128, DVP, false, true);
  constexpr uint32_t kIdG = idesc_bf16(128, 64, false, false);
  constexpr uint32_t kIdS2 = idesc_bf16(64, 128, false, true);
  constexpr uint32_t kId64 = idesc_bf16(64, 64, false, true);
  constexpr uint32_t kIdU = idesc_bf16(64, DVP, false, true);
  constexpr uint32_t kIdPU = idesc_bf16(128, DVP, false, true);
  constexpr uint32_t kIdDS = idesc_bf16(128, DVP, true, true);

  float E[64];        // lanes 0-15 of warps 0-3: row of E(c+1) = D - N D, fp32
  float oreg[kHalf];  // warps with qd >= 2: gamma_r rq_r (Q S^T)_r of chunk c, this column half

  for (int it = -2; it < nchunks && !abort; ++it) {
    const int c = it;                        // state chain
    const int cp2 = it + 1;                  // second half of the solve
    const int cp1 = it + 2;                  // Gram, A, P, D
    const bool do_chain = c >= 0;
    const bool do_p2 = cp2 >= 0 && cp2 < nchunks;
    const bool do_p1 = cp1 < nchunks;
    ChunkVec& vc = vecs[(c + 3) % 3];
    ChunkVec& v2 = vecs[(cp2 + 3) % 3];
    ChunkVec& v1 = vecs[(cp1 + 3) % 3];
    const uint32_t sKQC = sbase + L::kKQC + (c & 1) * 32768;
    const uint32_t sVKS = sbase + L::kVKS + (c & 1) * L::kVKSBytes;
    const uint32_t sKQP = sbase + L::kKQP;

    // ---- gates of chunk c+2: inclusive scan of g, beta ----
    if (do_p1 && tid < 64) {
      float gv = g_next;
      const float bv = b_next;
      const unsigned nonpos = __ballot_sync(0xffffffffu, gv <= 0.f);
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float up = __shfl_up_sync(0xffffffffu, gv, off);
        if (lane >= off) gv += up;
      }
      if (lane == 31) scan[warp] = gv;
      if (lane == 0) scan[2 + warp] = nonpos == 0xffffffffu ? 1.f : 0.f;
      v1.B[tid] = bv;
      v1.G[tid] = gv;
    }
    if (tid < 64) fetch_gates(cp1 + 1);
    // ---- operands for RT-a have landed ----
    {
      bool ok = true;
      if (do_p1) { ok = mbar_wait(bar_prep, prep_phase); prep_phase ^= 1; }
      if (do_chain && ok) { ok = mbar_wait(&bar_chain[c & 1], chain_phase[c & 1]); chain_phase[c & 1] ^= 1; }
      if (!__syncthreads_and(ok)) { abort = true; break; }
    }
    if (do_p1) {
      if (tid >= 32 && tid < 64) v1.G[tid] += scan[0];
      if (tid == 0) {
        v1.len = min(kC, t_end - (t_begin + cp1 * kC));
        v1.fast = (scan[2] > 0.f && scan[3] > 0.f) ? 1 : 0;
      }
    }

    // ================= RT-a: X(c) | Gram(c+2) | [ND | N^2](c+1) =================
    if (!(do_chain || do_p1 || do_p2)) continue;   // nothing in flight (empty sequence)
    if (warp == 0) {
      if (do_chain) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_warp(tmem + kColX, desc_kmajor(sKQC, kk, 16384), desc_mnmajor(sSb, kk, kR, 128 * kR), kIdX,
                   kk > 0);
      }
      if (do_p1) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_warp(tmem + kColG, desc_kmajor(sKQP, kk, 16384), desc_kmajor(sKQP, kk, 16384), kIdG, kk > 0);
      }
      if (do_p2) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16_warp(tmem + kColS2, desc_kmajor(sbase + L::kNm, kk, 0),
                   desc_mnmajor(sbase + L::kDm, kk, 128, 8192), kIdS2, kk > 0);
      }
      mma_commit_warp(bar_mma);
    }
    if (!wait_mma()) { abort = true; break; }

    // chain: K S^T rows -> second half of the U operand; rho Q S^T rows kept for the output
    if (do_chain) {
      float xv[kHalf];
      tmem_ld<kHalf>(tmem + tlane + kColX + ch * kHalf, xv);
      if (qd < 2) {
#pragma unroll
        for (int cc = 0; cc < kHalf / 8; ++cc)
          st_shared_v4(sVKS + mn_off<kR>(64 + r128, ch * kHalf + 8 * cc), pack8_bf16(xv + 8 * cc));
      } else {
        const int r = r128 - 64;
        const float rho = expf(vc.G[r]) * vc.Rq[r];
#pragma unroll
        for (int j = 0; j < kHalf; ++j) oreg[j] = rho * xv[j];
      }
    }
    // second half of the solve of c+1: E = D - N D (warps 0-3), N^2 (warps 4-7)
    if (do_p2) {
      float v[64];
      tmem_ld32(tmem + tlane + kColS2 + 64 * ch, v);
      tmem_ld32(tmem + tlane + kColS2 + 64 * ch + 32, v + 32);
      if (lo16) {
        if (ch == 0) {
#pragma unroll
          for (int cc = 0; cc < 8; ++cc) {
            const uint4 dv = ld_shared_v4(sbase + L::kDm + sw128_off(r64, 8 * cc, 0));
            const __nv_bfloat162* d2 = reinterpret_cast<const __nv_bfloat162*>(&dv);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 df = __bfloat1622float2(d2[e]);
              E[8 * cc + 2 * e] = df.x - v[8 * cc + 2 * e];
              E[8 * cc + 2 * e + 1] = df.y - v[8 * cc + 2 * e + 1];
            }
            st_shared_v4(sbase + L::kEm + sw128_off(r64, 8 * cc, 0), pack8_bf16(E + 8 * cc));
          }
        } else {
#pragma unroll
          for (int cc = 0; cc < 8; ++cc)
            st_shared_v4(sbase + L::kN2 + sw128_off(r64, 8 * cc, 0), pack8_bf16(v + 8 * cc));
        }
      }
    }
    // Gram of c+2: k norms from the diagonal, q norms by a short SIMT pass
    float gram[32];
    if (do_p1) {
      tmem_ld32(tmem + tlane + kColG + 32 * ch, gram);
      const int len = v1.len;
      if (qd < 2 && qd == ch) {
        float diag = 0.f;
#pragma unroll
        for (int j = 0; j < 32; ++j) diag = (j == lane) ? gram[j] : diag;
        const int r = r128;
        const float rk = r < len ? 1.0f / sqrtf(diag + kNormEps) : 0.f;
        const float Gr = v1.G[r];
        const float G0 = v1.G[0], GL = v1.G[len - 1];
        const bool fast = v1.fast && (G0 - GL) <= 160.f;
        const float gm = 0.5f * (G0 + GL);
        v1.Rk[r] = rk;
        v1.Ck[r] = fast ? expf(gm - Gr) * rk : rk;
        v1.Cw[r] = -v1.B[r] * expf(Gr) * rk;
        if (r == 0) { v1.gm = gm; v1.fast = fast ? 1 : 0; }
      }
      {
        const int r = tid >> 2, quarter = tid & 3;   // 4 threads per q row
        float ss = 0.f;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const int col = 32 * quarter + 8 * cc;
          const uint4 raw = ld_shared_v4(sKQP + sw128_off(64 + r, col, 16384));
          const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(p2[e]);
            ss = fmaf(f.x, f.x, fmaf(f.y, f.y, ss));
          }
        }
        ss += __shfl_xor_sync(0xffffffffu, ss, 1);
        ss += __shfl_xor_sync(0xffffffffu, ss, 2);
        if (quarter == 0) v1.Rq[r] = r < len ? scale / sqrtf(ss + kNormEps) : 0.f;
      }
    }
    __syncthreads();
    // the Gram slot is consumed: fetch the next chunk's raw tiles for its Gram
    if (warp == 0 && cp1 + 1 < nchunks) issue_prep_tma(cp1 + 1);

    // ---- A (diagonal blocks fp32, off-diagonal blocks bf16) and P of c+2 ----
    if (do_p1) {
      const int r = r128 & 63;
      const float Gr = v1.G[r];
      const bool fast = v1.fast != 0;
      const float gm = v1.gm;
      float x[32];
      if (qd < 2) {
        const float fr = v1.B[r] * v1.Rk[r] * (fast ? expf(Gr - gm) : 1.f);
        if (fast) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int s = 32 * ch + j;
            x[j] = (s < r) ? fr * v1.Ck[s] * gram[j] : 0.f;
          }
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int s = 32 * ch + j;
            x[j] = (s < r) ? fr * v1.Ck[s] * expf(Gr - v1.G[s]) * gram[j] : 0.f;
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
#pragma unroll
        for (int j = 0; j < 32; ++j) x[j] = (32 * ch + j < 16 * b) ? x[j] : 0.f;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
          st_shared_v4(sbase + L::kAo + sw128_off(r, 32 * ch + 8 * cc, 0), pack8_bf16(x + 8 * cc));
      } else {
        const float fr = v1.Rq[r] * (fast ? expf(Gr - gm) : 1.f);
        if (fast) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int s = 32 * ch + j;
            x[j] = (s <= r) ? fr * v1.Ck[s] * gram[j] : 0.f;
          }
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int s = 32 * ch + j;
            x[j] = (s <= r) ? fr * v1.Ck[s] * expf(Gr - v1.G[s]) * gram[j] : 0.f;
          }
        }
        const uint32_t sP = sbase + L::kP0 + ((cp1 + 3) % 3) * 16384;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
          st_shared_v4(sP + sw128_off(r, 32 * ch + 8 * cc, 0), pack8_bf16(x + 8 * cc));
      }
    }
    publish();

    // ================= RT-b: U(c) | Z(c+1) | N(c+2) =================
    if (warp == 0) {
      if (do_chain) {
        const uint32_t sTT = sbase + L::kTT;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_warp(tmem + kColU, desc_kmajor(sTT, kk, 8192), desc_mnmajor(sVKS, kk, kR, 128 * kR), kIdU,
                   kk > 0);
      }
      if (do_p2) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16_warp(tmem + kColS13, desc_kmajor(sbase + L::kN2, kk, 0),
                   desc_mnmajor(sbase + L::kEm, kk, 128, 8192), kId64, kk > 0);
      }
    }
    // D = (I + A_d)^-1 of c+2 while that tensor work is in flight
    if (do_p1) {
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
        for (int e = tid - 64; e < 64 * 6; e += kThreads - 64) {
          const int row = e / 6, idx = e - row * 6, b = row >> 4;
          const int cc = idx < 2 * b ? idx : idx + 2;
          st_shared_v4(sbase + L::kDm + sw128_off(row, 8 * cc, 0), make_uint4(0, 0, 0, 0));
        }
      }
    }
    publish();
    const bool rtb = do_chain || do_p2 || do_p1;
    if (warp == 0) {
      if (do_p1) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16_warp(tmem + (16u << 16) + kColS13, desc_kmajor(sbase + L::kDm, kk, 0),
                   desc_mnmajor(sbase + L::kAo, kk, 128, 8192), kId64, kk > 0);
      }
      if (rtb) mma_commit_warp(bar_mma);
    }
    if (rtb && !wait_mma()) { abort = true; break; }

    // chain: U and U_s of chunk c (bf16, MN-major) for P U and the state update
    if (do_chain) {
      float uv[kHalf];
      tmem_ld<kHalf>(tmem + tlane + kColU + ch * kHalf, uv);
      if (lo16) {
        const float us = expf(vc.G[vc.len - 1] - vc.G[r64]) * vc.Rk[r64];
        float usv[kHalf];
#pragma unroll
        for (int j = 0; j < kHalf; ++j) usv[j] = uv[j] * us;
#pragma unroll
        for (int cc = 0; cc < kHalf / 8; ++cc) {
          st_shared_v4(sbase + L::kUb + mn_off<kR>(r64, ch * kHalf + 8 * cc), pack8_bf16(uv + 8 * cc));
          st_shared_v4(sbase + L::kUsb + mn_off<kR>(r64, ch * kHalf + 8 * cc), pack8_bf16(usv + 8 * cc));
        }
      }
    }
    // T(c+1) = E + Z -> [T_u | -T_w] (warps 0-3) ; N(c+2) -> bf16 (warps 4-7)
    if (do_p2 || do_p1) {
      float v[64];
      tmem_ld32(tmem + tlane + kColS13, v);
      tmem_ld32(tmem + tlane + kColS13 + 32, v + 32);
      if (ch == 0 && lo16 && do_p2) {
        float tu[64];
#pragma unroll
        for (int s = 0; s < 64; ++s) {
          const float t = E[s] + v[s];
          tu[s] = t * v2.B[s];
          v[s] = t * v2.Cw[s];
        }
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) {
          st_shared_v4(sbase + L::kTT + sw128_off(r64, 8 * cc, 8192), pack8_bf16(tu + 8 * cc));
          st_shared_v4(sbase + L::kTT + sw128_off(r64, 64 + 8 * cc, 8192), pack8_bf16(v + 8 * cc));
        }
      }
      if (ch == 1 && !lo16 && do_p1) {
#pragma unroll
        for (int cc = 0; cc < 8; ++cc)
          st_shared_v4(sbase + L::kNm + sw128_off(r64, 8 * cc, 0), pack8_bf16(v + 8 * cc));
      }
    }
    publish();

    // ================= RT-c: P U (c) and dS^T (c) =================
    if (do_chain) {
      if (warp == 0) {
        const uint32_t sPa = sbase + L::kP0 + ((c + 3) % 3) * 16384 - 8192;   // rows 64-127 of this M=128 operand are P(c)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16_warp(tmem + kColPU, desc_kmajor(sPa, kk, 0), desc_mnmajor(sbase + L::kUb, kk, kR, 64 * kR), kIdPU,
                   kk > 0);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16_warp(tmem + kColDS, desc_mnmajor(sKQC, kk, 128, 16384),
                   desc_mnmajor(sbase + L::kUsb, kk, kR, 64 * kR), kIdDS, kk > 0);
        mma_commit_warp(bar_mma);
      }
      if (!wait_mma()) { abort = true; break; }
      float pu[kHalf], ds[kHalf];
      tmem_ld<kHalf>(tmem + tlane + kColPU + ch * kHalf, pu);
      tmem_ld<kHalf>(tmem + tlane + kColDS + ch * kHalf, ds);
      const int len = vc.len;
      if (qd >= 2 && r128 - 64 < len) {
        const int r = r128 - 64;
        const int c0 = t_begin + c * kC;
        __nv_bfloat16* orow = o + ((size_t)(c0 + r) * Hv + h) * kD + i0 + ch * kHalf;
#pragma unroll
        for (int cc = 0; cc < kHalf / 8; ++cc) {
          float xo[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) xo[e] = oreg[8 * cc + e] + pu[8 * cc + e];
          *reinterpret_cast<uint4*>(orow + 8 * cc) = pack8_bf16(xo);
        }
      }
      const float gL = expf(vc.G[len - 1]);
#pragma unroll
      for (int j = 0; j < kHalf; ++j) Sreg[j] = fmaf(gL, Sreg[j], ds[j]);
      store_state();
      publish();
      // this chain slot is free: bring in chunk c+2 for its state chain
      if (warp == 0 && c + 2 < nchunks) issue_chain_tma(c + 2);
    }
  }

  if (abort) {
    // drain any TMA still landing in shared memory before the CTA exits (bounded)
    if (tid == 0) {
      mbar_wait(bar_prep, prep_phase, 100000000ll);
      for (int s = 0; s < 2; ++s) mbar_wait(&bar_chain[s], chain_phase[s], 100000000ll);
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
