// Chunked Gated DeltaNet prefill on the sm_100a tensor cores, as one
// persistent kernel with two kinds of CTA (bf16 inputs, d_k = d_v = 128,
// chunk C = 64, fp32 state).
//
// Algorithm: the WY (UT-transform) form of the gated delta rule. For a chunk
// of L <= 64 tokens entering with state S, with G_r = sum_{s<=r} g_s,
// gamma_r = exp(G_r), rk_s = 1/|k_s|, rq_r = scale/|q_r|:
//
//   A   = strictly-lower( diag(beta) (exp(G_r - G_s)) o (K^ K^^T) )   64 x 64
//   T   = (I + A)^-1,  T_u = T diag(beta),  T_w = T diag(beta gamma rk)
//   U   = T_u V_raw - T_w (K_raw S^T)
//   O   = diag(gamma rq) Q_raw S^T + P U,   P_rs = exp(G_r - G_s) rq_r rk_s q_r.k_s (s <= r)
//   S  <- gamma_L S + U^T diag(exp(G_L - G_s) rk_s) K_raw
//
// The pages prefill "in blocks" ("On descend d'un cran", section "Ce que fait
// le moteur") with bf16 data and f32 accumulation ("On descend d'un cran :
// #002 le même compilateur sur un GPU", section "Le contrat numérique"), but
// print no chunk algorithm; this is the standard chunked form of the delta rule.
//
// Division of labour. Everything in the list above that does not involve S --
// the Gram matrix, A, P, the triangular solve and the scaled T_u | -T_w -- is
// independent across chunks and heads, and is the bulk of the work. The
// sequential part is the state chain: per chunk three dependent tcgen05 round
// trips (X = [k;q] S^T, U, then P U and dS). So the grid (one CTA per SM, all
// co-resident: cooperative launch) is split:
//
//   prep CTAs  take (head, chunk) items from a global counter in the order the
//              chains will need them, compute T and P once per item and publish
//              a ~25 KB package (T_u | -T_w, P, row scales) into a ring in the
//              workspace, which stays in L2;
//   chain CTAs each own one (sequence, value head, slice of DVP state rows) at a
//              time, bring in k, q, v by TMA and the chunk's package by a bulk
//              copy, and run only the state chain.
//
// Ring protocol, per (sequence, head) chain j and slot s = c mod R: a prep CTA
// waits until consumed[j][s] >= slices * (c / R) (every slice read the
// previous occupant), writes the package, fences and publishes
// ready[j][s] = c / R + 1 with release semantics; a chain CTA waits for that
// value with acquire semantics, copies the package, and adds 1 to
// consumed[j][s]. Items are ordered by (round, chunk, chain) where a round is
// the set of slice-chains the chain CTAs work on together, so a prep CTA never
// waits on a chain that is not running. Every wait is bounded (~2 s): past it
// the CTA records an error word and stops.
//
// Triangular solve: the four diagonal 16 x 16 unit-lower-triangular blocks of
// I + A are inverted by forward substitution in fp32 (D), then N = D A_o is
// nilpotent of order 4 and T = E + N^2 E with E = D - N D (three 64^3 MMAs).
// exp(G_r - G_s) is formed as exp(G_r - m) exp(m - G_s) around the middle m of
// the chunk's decay range; chunks whose range could leave the fp32 exponent
// range take an exact per-entry path.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace gdn {
namespace pc {

constexpr int kC = 64;
constexpr int kD = 128;
constexpr int kThreads = 256;
constexpr uint32_t kTmemCols = 512;
constexpr int kRing = 8;            // packages in flight per chain
constexpr int kMaxRounds = 1024;

// ---- package: everything a chain CTA needs from the preparation of one chunk ----
constexpr uint32_t kPkgTT = 0;        // [T_u | -T_w]  bf16 [64][128], K-major 128B-swizzled image
constexpr uint32_t kPkgP = 16384;     // P             bf16 [64][64],  same layout
constexpr uint32_t kPkgRho = 24576;   // gamma_r rq_r  fp32 [64]
constexpr uint32_t kPkgUs = 24832;    // exp(G_L - G_r) rk_r  fp32 [64]
constexpr uint32_t kPkgGL = 25088;    // gamma_L fp32, tokens int
constexpr uint32_t kPkgCopy = 25104;  // bytes copied per package (multiple of 16)
constexpr uint32_t kPkgStride = 25600;

// ---- workspace layout ----
struct Workspace {
  static constexpr size_t kCounter = 0;      // uint32 item counter
  static constexpr size_t kFlags = 256;      // ready[chains][R], then consumed[chains][R]
  __host__ __device__ static size_t flags_bytes(long chains) { return (size_t)chains * kRing * 2 * sizeof(uint32_t); }
  __host__ __device__ static size_t pkg_offset(long chains) {
    return (kFlags + flags_bytes(chains) + 1023) & ~size_t(1023);
  }
  __host__ __device__ static size_t bytes(long chains) { return pkg_offset(chains) + (size_t)chains * kRing * kPkgStride; }
  __host__ __device__ static size_t zeroed_bytes(long chains) { return kFlags + flags_bytes(chains); }
};

// ---- TMEM column map ----
constexpr uint32_t kColG = 0;      // prep: [k;q] k^T       M=128, N=64
constexpr uint32_t kColN = 64;     // prep: N = D A_o       M=64 (lanes 0-15)
constexpr uint32_t kColS2 = 128;   // prep: N D (lanes 0-15), N^2 (lanes 16-31)
constexpr uint32_t kColZ = 192;    // prep: N^2 E           M=64 (lanes 0-15)
constexpr uint32_t kColX = 256;    // chain: [k;q] S^T      M=128, N=DVP
constexpr uint32_t kColU = 320;    // chain: U              M=64 (lanes 0-15), N=DVP
constexpr uint32_t kColPU = 384;   // chain: [* ; P] U      M=128, N=DVP (rows 64-127)
constexpr uint32_t kColDS = 448;   // chain: dS^T           M=128, N=DVP

template <int DVP>
struct Smem {
  static constexpr uint32_t kR = DVP * 2;
  // chain role
  static constexpr uint32_t kKQC = 0;                         // 2 x [k;q] raw (32 KB each)
  static constexpr uint32_t kVKS = 65536;                     // 2 x [V ; K S^T] [128][DVP]
  static constexpr uint32_t kVKSBytes = 128 * kR;
  static constexpr uint32_t kPkg = kVKS + 2 * kVKSBytes;      // 2 x package
  static constexpr uint32_t kUb = kPkg + 2 * kPkgStride;      // U   [64][DVP]
  static constexpr uint32_t kUsb = kUb + 64 * kR;             // U_s [64][DVP]
  static constexpr uint32_t kSb = kUsb + 64 * kR;             // S^T [128][DVP]
  static constexpr uint32_t kChainEnd = kSb + 128 * kR;
  // prep role (aliases the chain region; a CTA has one role)
  static constexpr uint32_t kKQP = 0;                         // 2 x [k;q] raw (32 KB each)
  static constexpr uint32_t kAo = 65536;                      // A_o [64][64]
  static constexpr uint32_t kDm = kAo + 8192;                 // D
  static constexpr uint32_t kNm = kDm + 8192;                 // N
  static constexpr uint32_t kEm = kNm + 8192;                 // E = D - N D
  static constexpr uint32_t kN2 = kEm + 8192;                 // N^2
  static constexpr uint32_t kAd = kN2 + 8192;                 // diagonal blocks of A, fp32 [4][16][16]
  static constexpr uint32_t kVec = kAd + 4096;                // G, B, Rk, Rq, Ck, Cw [64] each
  static constexpr uint32_t kPrepEnd = kVec + 6 * 256 + 64;
  // common
  static constexpr uint32_t kCommon = ((kChainEnd > kPrepEnd ? kChainEnd : kPrepEnd) + 1023) & ~1023u;
  static constexpr uint32_t kRounds = kCommon;                // round_start[kMaxRounds + 1]
  static constexpr uint32_t kBar = kRounds + 4 * (kMaxRounds + 1) + 12;   // 8-byte aligned below
  static constexpr uint32_t kBarA = (kBar + 7) & ~7u;         // kq[2], pkg[2], mma, prep[2]
  static constexpr uint32_t kMisc = kBarA + 7 * 8;            // tmem slot, item, scan[4], next item (4)
  static constexpr uint32_t kTotal = kMisc + 64;
  static constexpr uint32_t kAlloc = kTotal + 1024;
  static_assert(kAlloc <= 227 * 1024, "shared memory budget");
  static_assert((kVKS % 1024) == 0 && (kPkg % 1024) == 0 && (kUb % 1024) == 0 && (kSb % 1024) == 0,
                "tile alignment");
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
__device__ __forceinline__ void st_global_v4(void* p, uint4 v) {
  *reinterpret_cast<uint4*>(p) = v;
}

using sm100::sw128_off;

struct Params {
  const float* g;
  const float* beta;
  const float* state_in;
  const int32_t* cu_seqlens;
  __nv_bfloat16* o;
  float* state_out;
  uint8_t* ws;          // workspace (counter and flags zeroed before the launch)
  int n_seqs, Hqk, Hv, total_T;
  float scale;
  int n_chain_ctas;     // CTAs [0, n_chain_ctas) run state chains, the rest prepare
};

template <int DVP>
__global__ void __launch_bounds__(kThreads, 1)
prefill_pc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                  const __grid_constant__ CUtensorMap vmap, const Params p) {
  using L = Smem<DVP>;
  using namespace sm100;
  static_assert(DVP == 32 || DVP == 64, "slice width");
  constexpr int kSlices = kD / DVP;
  constexpr int kHalf = DVP / 2;
  constexpr uint32_t kR = L::kR;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(sm);
  int* round_start = reinterpret_cast<int*>(sm + L::kRounds);
  uint64_t* bar_kq = reinterpret_cast<uint64_t*>(sm + L::kBarA);   // [2]
  uint64_t* bar_pkg = bar_kq + 2;                                   // [2]
  uint64_t* bar_mma = bar_kq + 4;
  uint64_t* bar_prep = bar_kq + 5;                                  // [2]
  uint32_t* misc = reinterpret_cast<uint32_t*>(sm + L::kMisc);     // [0] tmem, [2..5] scan, [8..11] next item

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qd = warp & 3, ch = warp >> 2;
  const int r128 = qd * 32 + lane;
  const int r64 = qd * 16 + (lane & 15);
  const bool lo16 = lane < 16;
  const int Hv = p.Hv, Hqk = p.Hqk;
  const long n_chains = (long)p.n_seqs * Hv;
  const long n_slice_chains = n_chains * kSlices;
  const int NC = p.n_chain_ctas;
  const int chains_per_round = NC / kSlices;
  const bool is_chain = (int)blockIdx.x < NC;

  uint32_t* counter = reinterpret_cast<uint32_t*>(p.ws + Workspace::kCounter);
  uint32_t* ready = reinterpret_cast<uint32_t*>(p.ws + Workspace::kFlags);
  uint32_t* consumed = ready + n_chains * kRing;
  uint8_t* pkgs = p.ws + Workspace::pkg_offset(n_chains);

  auto seq_bounds = [&](int n, int& tb, int& te) {
    te = min(p.cu_seqlens[n + 1], p.total_T);
    tb = min(max(p.cu_seqlens[n], 0), te);
  };
  auto n_chunks_of = [&](long j) {
    int tb, te;
    seq_bounds((int)(j / Hv), tb, te);
    return (te - tb + kC - 1) / kC;
  };

  if (tid == 0) {
    for (int i = 0; i < 7; ++i) mbar_init(&bar_kq[i], 1);
    fence_mbar_init();
    prefetch_tensormap(&qmap);
    prefetch_tensormap(&kmap);
    if (is_chain) prefetch_tensormap(&vmap);
  }
  if (warp == 0) {
    tmem_alloc(&misc[0], kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = __shfl_sync(0xffffffffu, misc[0], 0);
  const uint32_t tlane = static_cast<uint32_t>(qd * 32) << 16;

  uint32_t mma_phase = 0;
  bool abort = false;
  auto wait_mma = [&](bool also_ok = true) -> bool {
    bool ok = mbar_wait(bar_mma, mma_phase) && also_ok;
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

  if (is_chain) {
    // ============================== chain role ==============================
    constexpr uint32_t kIdX = idesc_bf16(128, DVP, false, true);
    constexpr uint32_t kIdU = idesc_bf16(64, DVP, false, true);
    constexpr uint32_t kIdPU = idesc_bf16(128, DVP, false, true);
    constexpr uint32_t kIdDS = idesc_bf16(128, DVP, true, true);
    const uint32_t sSb = sbase + L::kSb;
    uint32_t kq_phase[2] = {0, 0}, pkg_phase[2] = {0, 0};
    bool kq_pending[2] = {false, false}, pkg_pending[2] = {false, false};

    for (long sc = blockIdx.x; sc < n_slice_chains && !abort; sc += NC) {
      const long j = sc / kSlices;
      const int part = (int)(sc % kSlices);
      const int n = (int)(j / Hv), h = (int)(j % Hv);
      const int hq = h / (Hv / Hqk);
      const int i0 = part * DVP;
      int t_begin, t_end;
      seq_bounds(n, t_begin, t_end);
      const int nch = (t_end - t_begin + kC - 1) / kC;

      const size_t s_off = ((size_t)n * Hv + h) * kD * kD + (size_t)(i0 + ch * kHalf) * kD + r128;
      float Sreg[kHalf];
#pragma unroll
      for (int q2 = 0; q2 < kHalf; ++q2) Sreg[q2] = p.state_in ? p.state_in[s_off + (size_t)q2 * kD] : 0.f;
      auto store_state = [&]() {
#pragma unroll
        for (int c8 = 0; c8 < kHalf / 8; ++c8)
          st_shared_v4(sSb + mn_off<kR>(r128, ch * kHalf + 8 * c8), pack8_bf16(Sreg + 8 * c8));
      };
      store_state();

      auto issue_kq = [&](int c) {   // warp-collective (one warp)
        const int s = c & 1;
        const int c0 = t_begin + c * kC;
        uint8_t* kq = sm + L::kKQC + s * 32768;
        mbar_arrive_expect_tx_warp(&bar_kq[s], 4 * 8192 + 64 * kR);
        tma_load_3d_warp(kq, &kmap, &bar_kq[s], 0, hq, c0);
        tma_load_3d_warp(kq + 16384, &kmap, &bar_kq[s], 64, hq, c0);
        tma_load_3d_warp(kq + 8192, &qmap, &bar_kq[s], 0, hq, c0);
        tma_load_3d_warp(kq + 16384 + 8192, &qmap, &bar_kq[s], 64, hq, c0);
        tma_load_3d_warp(sm + L::kVKS + s * L::kVKSBytes, &vmap, &bar_kq[s], i0, h, c0);
      };
      auto request_pkg = [&](int c) -> bool {   // warp-collective (one warp)
        const int slot = c % kRing;
        bool ok = true;
        if (lane == 0) ok = wait_flag_geq(&ready[j * kRing + slot], (uint32_t)(c / kRing + 1));
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) return false;
        fence_async_global();
        const int s = c & 1;
        mbar_arrive_expect_tx_warp(&bar_pkg[s], kPkgCopy);
        bulk_load_warp(sm + L::kPkg + s * kPkgStride, pkgs + ((size_t)j * kRing + slot) * kPkgStride, kPkgCopy,
                       &bar_pkg[s]);
        return true;
      };

      bool ok = true;
      if (nch > 0) { kq_pending[0] = pkg_pending[0] = true; }
      if (nch > 1) kq_pending[1] = true;
      if (warp == 0 && nch > 0) {
        issue_kq(0);
        if (nch > 1) issue_kq(1);
        ok = request_pkg(0);
      }
      fence_async_smem();   // the bf16 state copy is read by the tensor core
      if (!__syncthreads_and(ok)) { abort = true; break; }

      float oreg[kHalf];
      for (int c = 0; c < nch; ++c) {
        const int s = c & 1;
        const uint32_t sKQC = sbase + L::kKQC + s * 32768;
        const uint32_t sVKS = sbase + L::kVKS + s * L::kVKSBytes;
        const uint32_t sPkg = sbase + L::kPkg + s * kPkgStride;
        const float* pkg_rho = reinterpret_cast<const float*>(sm + L::kPkg + s * kPkgStride + kPkgRho);
        const float* pkg_us = reinterpret_cast<const float*>(sm + L::kPkg + s * kPkgStride + kPkgUs);
        {
          bool w = mbar_wait(&bar_kq[s], kq_phase[s]);
          kq_phase[s] ^= 1;
          kq_pending[s] = false;
          if (w) { w = mbar_wait(&bar_pkg[s], pkg_phase[s]); pkg_phase[s] ^= 1; pkg_pending[s] = false; }
          if (!__syncthreads_and(w)) { abort = true; break; }
        }
        const int len = min(kC, t_end - (t_begin + c * kC));

        // ---- RT-a: X = [k;q] S^T ; meanwhile warp 1 hands back this chunk's ring slot
        //      (its package is in shared memory) and requests the next package ----
        ok = true;
        if (c + 1 < nch) pkg_pending[(c + 1) & 1] = true;
        if (warp == 0) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16_warp(tmem + kColX, desc_kmajor(sKQC, kk, 16384), desc_mnmajor(sSb, kk, kR, 128 * kR), kIdX,
                          kk > 0);
          mma_commit_warp(bar_mma);
        } else if (warp == 1) {
          if (lane == 0) red_add_release_gpu(&consumed[j * kRing + (c % kRing)], 1u);
          if (c + 1 < nch) ok = request_pkg(c + 1);
        }
        if (!wait_mma(ok)) { abort = true; break; }
        {
          float xv[kHalf];
          tmem_ld<kHalf>(tmem + tlane + kColX + ch * kHalf, xv);
          if (qd < 2) {
#pragma unroll
            for (int c8 = 0; c8 < kHalf / 8; ++c8)
              st_shared_v4(sVKS + mn_off<kR>(64 + r128, ch * kHalf + 8 * c8), pack8_bf16(xv + 8 * c8));
          } else {
            const float rho = pkg_rho[r128 - 64];
#pragma unroll
            for (int q2 = 0; q2 < kHalf; ++q2) oreg[q2] = rho * xv[q2];
          }
        }
        publish();

        // ---- RT-b: U = [T_u | -T_w] [V ; K S^T] ----
        if (warp == 0) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16_warp(tmem + kColU, desc_kmajor(sPkg + kPkgTT, kk, 8192), desc_mnmajor(sVKS, kk, kR, 128 * kR),
                          kIdU, kk > 0);
          mma_commit_warp(bar_mma);
        }
        if (!wait_mma()) { abort = true; break; }
        {
          float uv[kHalf];
          tmem_ld<kHalf>(tmem + tlane + kColU + ch * kHalf, uv);
          if (lo16) {
            const float us = pkg_us[r64];
            float usv[kHalf];
#pragma unroll
            for (int q2 = 0; q2 < kHalf; ++q2) usv[q2] = uv[q2] * us;
#pragma unroll
            for (int c8 = 0; c8 < kHalf / 8; ++c8) {
              st_shared_v4(sbase + L::kUb + mn_off<kR>(r64, ch * kHalf + 8 * c8), pack8_bf16(uv + 8 * c8));
              st_shared_v4(sbase + L::kUsb + mn_off<kR>(r64, ch * kHalf + 8 * c8), pack8_bf16(usv + 8 * c8));
            }
          }
        }
        publish();

        // ---- RT-c: P U and dS^T = K^T U_s ----
        if (warp == 0) {
          const uint32_t sPa = sPkg + kPkgP - 8192;   // rows 64-127 of this M=128 operand are P
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_warp(tmem + kColPU, desc_kmajor(sPa, kk, 0), desc_mnmajor(sbase + L::kUb, kk, kR, 64 * kR),
                          kIdPU, kk > 0);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_warp(tmem + kColDS, desc_mnmajor(sKQC, kk, 128, 16384),
                          desc_mnmajor(sbase + L::kUsb, kk, kR, 64 * kR), kIdDS, kk > 0);
          mma_commit_warp(bar_mma);
        }
        if (!wait_mma()) { abort = true; break; }
        {
          float pu[kHalf], ds[kHalf];
          tmem_ld<kHalf>(tmem + tlane + kColPU + ch * kHalf, pu);
          tmem_ld<kHalf>(tmem + tlane + kColDS + ch * kHalf, ds);
          if (qd >= 2 && r128 - 64 < len) {
            const int r = r128 - 64;
            __nv_bfloat16* orow = p.o + ((size_t)(t_begin + c * kC + r) * Hv + h) * kD + i0 + ch * kHalf;
#pragma unroll
            for (int c8 = 0; c8 < kHalf / 8; ++c8) {
              float xo[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) xo[e] = oreg[8 * c8 + e] + pu[8 * c8 + e];
              *reinterpret_cast<uint4*>(orow + 8 * c8) = pack8_bf16(xo);
            }
          }
          const float pkg_gL = *reinterpret_cast<const float*>(sm + L::kPkg + s * kPkgStride + kPkgGL);
#pragma unroll
          for (int q2 = 0; q2 < kHalf; ++q2) Sreg[q2] = fmaf(pkg_gL, Sreg[q2], ds[q2]);
          store_state();
          // this chunk's raw slot is free (every MMA reading it completed): bring in chunk c+2
          if (c + 2 < nch) {
            kq_pending[s] = true;
            if (warp == 1) issue_kq(c + 2);
          }
        }
        publish();
      }
      if (abort) break;
#pragma unroll
      for (int q2 = 0; q2 < kHalf; ++q2) p.state_out[s_off + (size_t)q2 * kD] = Sreg[q2];
    }
    if (abort && tid == 0) {   // let copies still in flight land before the CTA exits (bounded)
      for (int s = 0; s < 2; ++s) {
        if (kq_pending[s]) mbar_wait(&bar_kq[s], kq_phase[s], 100000000ll);
        if (pkg_pending[s]) mbar_wait(&bar_pkg[s], pkg_phase[s], 100000000ll);
      }
    }
  } else {
    // ============================== prep role ===============================
    // round table: items of round r are [round_start[r], round_start[r+1])
    const long n_rounds = (n_slice_chains + NC - 1) / NC;
    if (tid == 0) {
      int acc = 0;
      for (long r = 0; r < n_rounds && r < kMaxRounds; ++r) {
        const long j0 = r * chains_per_round;
        const long j1 = min(j0 + chains_per_round, n_chains);
        int maxc = 0;
        for (long jj = j0; jj < j1; ++jj) maxc = max(maxc, n_chunks_of(jj));
        round_start[r] = acc;
        acc += (int)(j1 - j0) * maxc;
      }
      round_start[min(n_rounds, (long)kMaxRounds)] = acc;
    }
    __syncthreads();
    const int total_items = round_start[min(n_rounds, (long)kMaxRounds)];

    constexpr uint32_t kIdG = idesc_bf16(128, 64, false, false);
    constexpr uint32_t kId64 = idesc_bf16(64, 64, false, true);
    float* vG = reinterpret_cast<float*>(sm + L::kVec);
    float* vB = vG + 64;
    float* vRk = vB + 64;
    float* vRq = vRk + 64;
    float* vCk = vRq + 64;
    float* vCw = vCk + 64;
    float* Ad = reinterpret_cast<float*>(sm + L::kAd);
    float* scan = reinterpret_cast<float*>(&misc[2]);
    uint32_t prep_phase[2] = {0, 0};
    bool prep_pending[2] = {false, false};

    // Next non-empty item: thread 0 claims items until one has tokens (or none are left).
    auto fetch_item = [&](int& valid, int& cc, long& jj) {
      if (tid == 0) {
        uint32_t v = 0, c_ = 0;
        long j_ = 0;
        while (true) {
          const int item = (int)atomicAdd(counter, 1u);
          if (item >= total_items) break;
          int r = 0;
          while (round_start[r + 1] <= item) ++r;
          const long j0 = (long)r * chains_per_round;
          const int cpr = (int)(min(j0 + chains_per_round, n_chains) - j0);
          const int local = item - round_start[r];
          c_ = (uint32_t)(local / cpr);
          j_ = j0 + local % cpr;
          if ((int)c_ < n_chunks_of(j_)) { v = 1; break; }
        }
        misc[8] = v;
        misc[9] = c_;
        misc[10] = (uint32_t)(j_ & 0xffffffffl);
        misc[11] = (uint32_t)(j_ >> 32);
      }
      __syncthreads();
      valid = (int)misc[8];
      cc = (int)misc[9];
      jj = (long)misc[10] | ((long)misc[11] << 32);
      __syncthreads();   // misc is rewritten by the next fetch
    };
    // Raw k, q tiles of an item into buffer b (warp-collective, warp 0), gates into registers (threads 0-63).
    float g_pf = 0.f, b_pf = 0.f;
    auto prefetch_item = [&](int cc, long jj, int b) {
      const int n_ = (int)(jj / Hv), h_ = (int)(jj % Hv);
      int tb, te;
      seq_bounds(n_, tb, te);
      const int c0_ = tb + cc * kC;
      const int len_ = min(kC, te - c0_);
      if (warp == 0) {
        const int hq_ = h_ / (Hv / Hqk);
        uint8_t* kq = sm + L::kKQP + b * 32768;
        prep_pending[b] = true;
        mbar_arrive_expect_tx_warp(&bar_prep[b], 4 * 8192);
        tma_load_3d_warp(kq, &kmap, &bar_prep[b], 0, hq_, c0_);
        tma_load_3d_warp(kq + 16384, &kmap, &bar_prep[b], 64, hq_, c0_);
        tma_load_3d_warp(kq + 8192, &qmap, &bar_prep[b], 0, hq_, c0_);
        tma_load_3d_warp(kq + 16384 + 8192, &qmap, &bar_prep[b], 64, hq_, c0_);
      }
      if (tid < 64) {
        const bool valid_ = tid < len_;
        g_pf = valid_ ? p.g[(size_t)(c0_ + tid) * Hv + h_] : 0.f;
        b_pf = valid_ ? p.beta[(size_t)(c0_ + tid) * Hv + h_] : 0.f;
      }
    };

    int cur_valid, cur_c;
    long cur_j;
    fetch_item(cur_valid, cur_c, cur_j);
    if (cur_valid) prefetch_item(cur_c, cur_j, 0);
    int buf = 0;

    while (!abort && cur_valid) {
      const int c = cur_c;
      const long j = cur_j;
      const int n = (int)(j / Hv);
      int t_begin, t_end;
      seq_bounds(n, t_begin, t_end);
      const int c0 = t_begin + c * kC;
      const int len = min(kC, t_end - c0);
      const int slot = c % kRing;
      uint8_t* pkg = pkgs + ((size_t)j * kRing + slot) * kPkgStride;
      const uint32_t sKQ = sbase + L::kKQP + buf * 32768;
      const float g_cur = g_pf, b_cur = b_pf;

      // claim and prefetch the next item while this one is processed
      int nxt_valid, nxt_c;
      long nxt_j;
      fetch_item(nxt_valid, nxt_c, nxt_j);
      if (nxt_valid) prefetch_item(nxt_c, nxt_j, buf ^ 1);

      // ---- wait until every slice has read the previous occupant of the ring slot ----
      bool ok = true;
      if (tid == 0) ok = wait_flag_geq(&consumed[j * kRing + slot], (uint32_t)(kSlices * (c / kRing)));
      if (!__syncthreads_and(ok)) { abort = true; break; }

      // ---- gates: inclusive scan of g, beta ----
      if (tid < 64) {
        float gv = g_cur;
        const float bv = b_cur;
        const unsigned nonpos = __ballot_sync(0xffffffffu, gv <= 0.f);
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const float up = __shfl_up_sync(0xffffffffu, gv, off);
          if (lane >= off) gv += up;
        }
        if (lane == 31) scan[warp] = gv;
        if (lane == 0) scan[2 + warp] = nonpos == 0xffffffffu ? 1.f : 0.f;
        vB[tid] = bv;
        vG[tid] = gv;
      }
      {
        bool w = mbar_wait(&bar_prep[buf], prep_phase[buf]);
        prep_phase[buf] ^= 1;
        prep_pending[buf] = false;
        if (!__syncthreads_and(w)) { abort = true; break; }
      }
      if (tid >= 32 && tid < 64) vG[tid] += scan[0];

      // ---- Gram [k;q] k^T on the tensor core; norms by SIMT meanwhile ----
      if (warp == 0) {
#pragma unroll 1
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_warp(tmem + kColG, desc_kmajor(sKQ, kk, 16384), desc_kmajor(sKQ, kk, 16384), kIdG, kk > 0);
        mma_commit_warp(bar_mma);
      }
      {
        const int row = tid >> 1, half = tid & 1;   // rows 0-63: k, rows 64-127: q
        float ss = 0.f;
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
          const uint4 raw = ld_shared_v4(sKQ + sw128_off(row, 64 * half + 8 * c8, 16384));
          const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(p2[e]);
            ss = fmaf(f.x, f.x, fmaf(f.y, f.y, ss));
          }
        }
        ss += __shfl_xor_sync(0xffffffffu, ss, 1);
        if (half == 0) {
          const int rr = row & 63;
          if (row < 64) vRk[rr] = rr < len ? 1.0f / sqrtf(ss + kNormEps) : 0.f;
          else vRq[rr] = rr < len ? p.scale / sqrtf(ss + kNormEps) : 0.f;
        }
      }
      __syncthreads();
      const float G0 = vG[0], GL = vG[len - 1];
      const bool fast = scan[2] > 0.f && scan[3] > 0.f && (G0 - GL) <= 160.f;
      const float gm = 0.5f * (G0 + GL);
      if (tid < 64) {
        const float Gr = vG[tid], rk = vRk[tid];
        vCk[tid] = fast ? expf(gm - Gr) * rk : rk;
        vCw[tid] = -vB[tid] * expf(Gr) * rk;
        // row scales the chain needs
        reinterpret_cast<float*>(pkg + kPkgRho)[tid] = expf(Gr) * vRq[tid];
        reinterpret_cast<float*>(pkg + kPkgUs)[tid] = expf(GL - Gr) * rk;
        if (tid == 0) {
          reinterpret_cast<float*>(pkg + kPkgGL)[0] = expf(GL);
          reinterpret_cast<int*>(pkg + kPkgGL)[1] = len;
        }
      }
      if (!wait_mma()) { abort = true; break; }   // (its barrier also publishes vCk, vCw)

      // ---- A (diagonal blocks fp32, off-diagonal blocks bf16) and P ----
      {
        float gram[32];
        tmem_ld32(tmem + tlane + kColG + 32 * ch, gram);
        const int rr = r128 & 63;
        const float Gr = vG[rr];
        float x[32];
        if (qd < 2) {
          const float fr = vB[rr] * vRk[rr] * (fast ? expf(Gr - gm) : 1.f);
          if (fast) {
#pragma unroll
            for (int q2 = 0; q2 < 32; ++q2) {
              const int sidx = 32 * ch + q2;
              x[q2] = (sidx < rr) ? fr * vCk[sidx] * gram[q2] : 0.f;
            }
          } else {
#pragma unroll
            for (int q2 = 0; q2 < 32; ++q2) {
              const int sidx = 32 * ch + q2;
              x[q2] = (sidx < rr) ? fr * vCk[sidx] * expf(Gr - vG[sidx]) * gram[q2] : 0.f;
            }
          }
          const int b = rr >> 4;
          if ((b >> 1) == ch) {
            float* dst = Ad + (b * 16 + (rr & 15)) * 16;
            if (b & 1) {
#pragma unroll
              for (int q2 = 0; q2 < 16; ++q2) dst[q2] = x[16 + q2];
            } else {
#pragma unroll
              for (int q2 = 0; q2 < 16; ++q2) dst[q2] = x[q2];
            }
          }
#pragma unroll
          for (int q2 = 0; q2 < 32; ++q2) x[q2] = (32 * ch + q2 < 16 * b) ? x[q2] : 0.f;
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8)
            st_shared_v4(sbase + L::kAo + sw128_off(rr, 32 * ch + 8 * c8, 0), pack8_bf16(x + 8 * c8));
        } else {
          const float fr = vRq[rr] * (fast ? expf(Gr - gm) : 1.f);
          if (fast) {
#pragma unroll
            for (int q2 = 0; q2 < 32; ++q2) {
              const int sidx = 32 * ch + q2;
              x[q2] = (sidx <= rr) ? fr * vCk[sidx] * gram[q2] : 0.f;
            }
          } else {
#pragma unroll
            for (int q2 = 0; q2 < 32; ++q2) {
              const int sidx = 32 * ch + q2;
              x[q2] = (sidx <= rr) ? fr * vCk[sidx] * expf(Gr - vG[sidx]) * gram[q2] : 0.f;
            }
          }
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8)   // P goes straight into the package image
            st_global_v4(pkg + kPkgP + sw128_off(rr, 32 * ch + 8 * c8, 0), pack8_bf16(x + 8 * c8));
        }
      }
      __syncthreads();

      // ---- D = (I + A_d)^-1 ----
      if (tid < 64) {
        const int b = tid >> 4, jj = tid & 15;
        const float* Ab = Ad + b * 256;
        float xs[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float acc = 0.f;
#pragma unroll
          for (int k2 = 0; k2 < i; ++k2) acc = fmaf(Ab[i * 16 + k2], xs[k2], acc);
          xs[i] = (i == jj) ? 1.f : (i > jj ? -acc : 0.f);
        }
#pragma unroll
        for (int i = 0; i < 16; ++i)
          st_shared_b16(sbase + L::kDm + sw128_off(16 * b + i, 16 * b + jj, 0), __float2bfloat16_rn(xs[i]));
      } else {
        for (int e = tid - 64; e < 64 * 6; e += kThreads - 64) {
          const int row = e / 6, idx = e - row * 6, b = row >> 4;
          const int cc = idx < 2 * b ? idx : idx + 2;
          st_shared_v4(sbase + L::kDm + sw128_off(row, 8 * cc, 0), make_uint4(0, 0, 0, 0));
        }
      }
      publish();

      // ---- N = D A_o ----
      if (warp == 0) {
#pragma unroll 1
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16_warp(tmem + kColN, desc_kmajor(sbase + L::kDm, kk, 0), desc_mnmajor(sbase + L::kAo, kk, 128, 8192),
                        kId64, kk > 0);
        mma_commit_warp(bar_mma);
      }
      if (!wait_mma()) { abort = true; break; }
      {
        float v[32];
        tmem_ld32(tmem + tlane + kColN + 32 * ch, v);
        if (lo16) {
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8)
            st_shared_v4(sbase + L::kNm + sw128_off(r64, 32 * ch + 8 * c8, 0), pack8_bf16(v + 8 * c8));
        }
      }
      publish();

      // ---- N D (lanes 0-15) and N^2 (lanes 16-31) ----
      if (warp == 0) {
#pragma unroll 1
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16_warp(tmem + kColS2, desc_kmajor(sbase + L::kNm, kk, 0), desc_mnmajor(sbase + L::kDm, kk, 128, 8192),
                        kId64, kk > 0);
#pragma unroll 1
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16_warp(tmem + (16u << 16) + kColS2, desc_kmajor(sbase + L::kNm, kk, 0),
                        desc_mnmajor(sbase + L::kNm, kk, 128, 8192), kId64, kk > 0);
        mma_commit_warp(bar_mma);
      }
      if (!wait_mma()) { abort = true; break; }
      float E[32];   // lanes 0-15: columns 32ch..32ch+31 of row r64 of E = D - N D (fp32)
      {
        float v[32];
        tmem_ld32(tmem + tlane + kColS2 + 32 * ch, v);
        if (lo16) {
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8) {
            const uint4 dv = ld_shared_v4(sbase + L::kDm + sw128_off(r64, 32 * ch + 8 * c8, 0));
            const __nv_bfloat162* d2 = reinterpret_cast<const __nv_bfloat162*>(&dv);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 df = __bfloat1622float2(d2[e]);
              E[8 * c8 + 2 * e] = df.x - v[8 * c8 + 2 * e];
              E[8 * c8 + 2 * e + 1] = df.y - v[8 * c8 + 2 * e + 1];
            }
            st_shared_v4(sbase + L::kEm + sw128_off(r64, 32 * ch + 8 * c8, 0), pack8_bf16(E + 8 * c8));
          }
        } else {
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8)
            st_shared_v4(sbase + L::kN2 + sw128_off(r64, 32 * ch + 8 * c8, 0), pack8_bf16(v + 8 * c8));
        }
      }
      publish();

      // ---- Z = N^2 E ; T = E + Z -> [T_u | -T_w] into the package ----
      if (warp == 0) {
#pragma unroll 1
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16_warp(tmem + kColZ, desc_kmajor(sbase + L::kN2, kk, 0), desc_mnmajor(sbase + L::kEm, kk, 128, 8192),
                        kId64, kk > 0);
        mma_commit_warp(bar_mma);
      }
      if (!wait_mma()) { abort = true; break; }
      {
        float z[32];
        tmem_ld32(tmem + tlane + kColZ + 32 * ch, z);
        if (lo16) {
          float tu[32], tw[32];
#pragma unroll
          for (int q2 = 0; q2 < 32; ++q2) {
            const int sidx = 32 * ch + q2;
            const float t = E[q2] + z[q2];
            tu[q2] = t * vB[sidx];
            tw[q2] = t * vCw[sidx];
          }
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8) {
            st_global_v4(pkg + kPkgTT + sw128_off(r64, 32 * ch + 8 * c8, 8192), pack8_bf16(tu + 8 * c8));
            st_global_v4(pkg + kPkgTT + sw128_off(r64, 64 + 32 * ch + 8 * c8, 8192), pack8_bf16(tw + 8 * c8));
          }
        }
      }
      // ---- publish the package ----
      __threadfence();
      tc_fence_before();
      __syncthreads();
      tc_fence_after();
      if (tid == 0) st_release_gpu(&ready[j * kRing + slot], (uint32_t)(c / kRing + 1));
      cur_valid = nxt_valid;
      cur_c = nxt_c;
      cur_j = nxt_j;
      buf ^= 1;
    }
    if (abort && tid == 0) {   // let prefetches still in flight land before the CTA exits (bounded)
      for (int b = 0; b < 2; ++b)
        if (prep_pending[b]) mbar_wait(&bar_prep[b], prep_phase[b], 100000000ll);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace pc
}  // namespace gdn
