// Chunked Gated DeltaNet prefill on the sm_100a tensor cores, as one
// persistent kernel with two kinds of CTA (bf16 or f16 inputs, d_k = d_v =
// 128, chunk C = 64, fp32 state). T is the 16-bit input type; every
// tensor-core operand the kernel forms is rounded to T as well, so that no
// product mixes the two formats, and accumulation is fp32 throughout.
//
// Algorithm: the WY (UT-transform) form of the gated delta rule. For a chunk
// of L <= 64 tokens entering with state S, with G_r = sum_{s<=r} g_s,
// gamma_r = exp(G_r), rk_s = 1/|k_s|, rq_r = scale/|q_r|:
//
//   A   = strictly-lower( diag(beta) (exp(G_r - G_s)) o (K^ K^^T) )   64 x 64
//   T   = (I + A)^-1,  T_u = T diag(beta),  T_w = T diag(beta gamma rk)
//   W   = T_w K_raw,   P_rs = exp(G_r - G_s) rq_r rk_s q_r.k_s  (s <= r)
//   U   = T_u V_raw - W S^T
//   O   = diag(gamma rq) Q_raw S^T + P U
//       = [P T_u] V_raw + [diag(gamma rq) Q_raw - P W] S^T
//   S  <- gamma_L S + U^T diag(exp(G_L - G_s) rk_s) K_raw
//
// so that, with the state-independent operands
//
//   A1 = [ -W ; diag(gamma rq) Q_raw - P W ]   128 x d_k
//   A2 = [ T_u ; P T_u ]                       128 x 64
//
// one product Y = A2 V_raw + A1 S^T yields U (rows 0-63) and O (rows 64-127)
// of the chunk, and a second, dS^T = K_raw^T diag(us) U, moves the state.
//
// The pages prefill "in blocks" ("On descend d'un cran", section "Ce que fait
// le moteur") with bf16 data and f32 accumulation ("On descend d'un cran :
// #002 le même compilateur sur un GPU", section "Le contrat numérique"), but
// print no chunk algorithm; this is the standard chunked form of the delta rule.
//
// Division of labour. Everything that does not involve S -- the Gram matrix,
// A, P, the triangular solve, W and the products in A1, A2 -- is independent
// across chunks and heads and is the bulk of the work. The sequential part is
// the state chain: per chunk two dependent tcgen05 round trips (Y, then dS).
// So the grid (one CTA per SM, all co-resident: cooperative launch) is split:
//
//   prep CTAs  take (head, chunk) items from a global counter in the order the
//              chains will need them and publish a ~48 KB package (A1 and A2
//              as tensor-core operand images, two row-scale values) into a
//              ring in the workspace, which stays in L2;
//   chain CTAs each own one (sequence, value head, slice of DVP state rows) at a
//              time and run only the state chain on the packages, k and v.
//
// Every CTA has eight compute warps (0-7) and three with jobs of their own.
// In a chain CTA warp 8 acquires ready flags and issues the copies of package,
// k and v, warp 9 hands ring slots back once a copy has landed, and warp 10
// issues every tensor-core product, so the compute warps only run the
// epilogues (U_s on warps 0, 1, 4, 5, O on 2, 3, 6, 7, which also store O;
// then the state). Y and dS commit to barriers of their own and every compute
// warp waits for them on its own. In a prep CTA warp 8 claims items, fetches
// their gates and tiles and waits for ring slots, warp 10 copies each staged
// package out to its ring slot and publishes it once the copies are complete,
// and warp 0 of the compute warps issues the MMAs (warp 9 has no job there). Handovers use
// mbarriers with bounded waits; the prep compute warps synchronise among
// themselves with named barrier 1. (The register file is allocated per 128
// threads, so eleven warps cost no registers over nine.)
//
// Ring protocol. The chain CTAs work on the slice-chains in rounds; in round r
// chain j = r P + q runs at position q < P (P chains per round). Each position
// has a ring of R package slots and numbers its packages s = base_r + c, with
// base_r the sum over earlier rounds of the longest chain's chunk count; slot
// s mod R holds package s. The prep hand-over warp waits until consumed[q][s mod R]
// >= slices * (s / R) (every slice read the previous occupant) before it hands
// the item over; the compute warps stage the package in shared memory, the
// writing warp copies it out with bulk copies and, once those are complete (and
// fenced), sets ready[q][s mod R] = s / R + 1 with release semantics. A
// chain's issuing warp waits for that value with acquire semantics and copies
// the package into shared memory; its releasing warp then adds 1 to
// consumed[q][s mod R] (and arrives on the input buffer's free barrier, so that
// its waits, which go by mbarrier parity, never fall a phase behind). Numbers a shorter chain leaves unused are counted as
// consumed by its chain CTAs at the end of the round. Items are ordered by (round, chunk, chain), so a prep CTA never waits
// on a chain that is not running, and the workspace holds P R packages however
// many sequences there are. Every wait is bounded (~2 s): past it the CTA
// records an error word and stops.
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
constexpr int kCompute = 256;        // compute threads (warps 0-7)
constexpr int kThreads = 352;        // and three warps with their own jobs:
constexpr int kCtlWarp = 8;          // chain: issues the copies; prep: claims and hands over items
constexpr int kRelWarp = 9;          // chain: hands ring slots back; prep: publishes packages
constexpr int kMmaWarp = 10;         // chain: issues the tensor-core work
constexpr uint32_t kTmemCols = 512;
constexpr int kRing = 12;            // package slots per ring position
constexpr int kFlagStride = 32;      // flag words per ring position: each position's flags on a 128-byte line
constexpr int kMaxRounds = 1024;
constexpr int kMaxPositions = 74;    // chains per round at most

// ---- package: what a chain CTA needs from the preparation of one chunk ----
constexpr uint32_t kPkgA1 = 0;        // A1 T [128][128]: two K-major 128B-swizzled atoms, 16 KB apart
constexpr uint32_t kPkgA2 = 32768;    // A2 T [128][64]:  one K-major 128B-swizzled atom
constexpr uint32_t kPkgUs = 49152;    // us_r = exp(G_L - G_r) rk_r, fp32 [64]
constexpr uint32_t kPkgGL = 49408;    // gamma_L fp32, tokens int
constexpr uint32_t kPkgCopy = 49424;  // bytes copied per package (multiple of 16)
constexpr uint32_t kPkgStride = 50176;

// ---- workspace layout ----
struct Workspace {
  static constexpr size_t kCounter = 0;      // uint32 counter of the items after the first one per prep CTA
  static constexpr size_t kFlags = 256;      // ready[positions][32], then consumed[positions][32] (R used)
  __host__ __device__ static constexpr size_t flags_bytes(long positions) {
    return (size_t)positions * kFlagStride * 2 * sizeof(uint32_t);
  }
  __host__ __device__ static constexpr size_t pkg_offset(long positions) {
    return (kFlags + flags_bytes(positions) + 1023) & ~size_t(1023);
  }
  __host__ __device__ static constexpr size_t bytes(long positions) {
    return pkg_offset(positions) + (size_t)positions * kRing * kPkgStride;
  }
  __host__ __device__ static constexpr size_t zeroed_bytes(long positions) { return kFlags + flags_bytes(positions); }
};

// ---- TMEM column map ----
// prep: a stage's accumulator is read out before the next stage's MMA is
// issued, so later stages reuse the columns of earlier ones
constexpr uint32_t kColG = 0;      // [k;q] k^T             M=128, N=64
constexpr uint32_t kColN = 64;     // N = D A_o             M=64 (lanes 0-15)
constexpr uint32_t kColS2 = 128;   // N D (lanes 0-15), N^2 (lanes 16-31)
constexpr uint32_t kColZ = 0;      // N^2 E                 M=64 (the Gram columns, read in stage 1)
constexpr uint32_t kColW = 64;     // -W, d_k 0-63 in lanes 0-15, 64-127 in lanes 16-31 (N's columns)
constexpr uint32_t kColPW = 128;   // -P W, the same split (N D, N^2's columns)
constexpr uint32_t kColPT = 192;   // P T_u                 M=64, N=64 (lanes 0-15)
// chain:
constexpr uint32_t kColY = 0;      // Y = [U ; O]           M=128, N=DVP, two buffers 128 columns apart
constexpr uint32_t kColDS = 256;   // dS^T                  M=128, N=DVP
constexpr uint32_t kColA1 = 384;   // A1 staged as the A operand of A1 S^T: two buffers of 64 columns

template <int DVP>
struct Smem {
  // A slice of DVP state rows is stored as blocks of kBlk columns, each an
  // MN-major tile with rows of kRB bytes and the matching swizzle.
  static constexpr int kBlk = DVP < 64 ? DVP : 64;
  static constexpr int kBlocks = DVP / kBlk;
  static constexpr uint32_t kRB = kBlk * 2;
  static constexpr uint32_t kR = DVP * 2;
  // chain role: kNB input buffers {package image, k tile, v slice} (three, where
  // they fit at 32-row slices, measured no faster than two)
  static constexpr int kNB = 2;
  static constexpr uint32_t kIn = 0;
  static constexpr uint32_t kInK = kPkgStride;                // k [64][128] as two 64-column halves, 8 KB apart
  static constexpr uint32_t kInV = kInK + 16384;              // v [64][DVP]
  static constexpr uint32_t kInBytes = (kInV + 64 * kR + 1023) & ~1023u;
  static constexpr uint32_t kUsb = kNB * kInBytes;            // U_s [64][DVP]
  static constexpr uint32_t kSb = kUsb + ((64 * kR + 1023) & ~1023u);   // S^T [128][DVP]
  static constexpr uint32_t kChainEnd = kSb + 128 * kR;
  // prep role (aliases the chain region; a CTA has one role)
  static constexpr uint32_t kKQP = 0;                         // 2 x [k;q] raw (32 KB each)
  static constexpr uint32_t kAo = 65536;                      // A_o [64][64]
  static constexpr uint32_t kDm = kAo + 8192;                 // D
  static constexpr uint32_t kNm = kDm + 8192;                 // N
  static constexpr uint32_t kEm = kNm + 8192;                 // E = D - N D
  static constexpr uint32_t kN2 = kEm + 8192;                 // N^2
  static constexpr uint32_t kPm = kN2 + 8192;                 // P
  static constexpr uint32_t kTw = kPm + 8192;                 // -T_w
  static constexpr uint32_t kTu = kTw + 8192;                 // T_u
  static constexpr uint32_t kWm = kTu + 8192;                 // -W [64][128], two halves 8 KB apart
  static constexpr uint32_t kA1b = kWm + 16384;               // rho Q - P W [64][128], two halves 8 KB apart
  static constexpr uint32_t kA2b = kA1b + 16384;              // P T_u [64][64]
  static constexpr uint32_t kPv = kA2b + 8192;                // package vectors: us[64], gamma_L, tokens (2 x 512 B)
  static constexpr uint32_t kAd = kPv + 1024;                 // diagonal blocks of A, fp32 [4][16][kAdRow]
  static constexpr int kAdRow = 20;                           // (80-byte rows: eight rows, eight bank groups)
  static constexpr uint32_t kVec = kAd + 4 * 16 * kAdRow * 4; // 8 vectors of 64 fp32
  static constexpr uint32_t kQueue = kVec + 8 * 256;          // 2 items handed over by the control warp:
  static constexpr uint32_t kQueueBytes = 640;                //   {valid, s, q, len}, g[64] @64, beta[64] @320
  static constexpr uint32_t kRounds = kQueue + 2 * kQueueBytes;      // round_start[kMaxRounds + 1]
  static constexpr uint32_t kRBase = kRounds + 4 * (kMaxRounds + 1);   // base_r [kMaxRounds + 1]
  static constexpr uint32_t kPrepEnd = kRBase + 4 * (kMaxRounds + 1);
  // common
  static constexpr uint32_t kCommon = ((kChainEnd > kPrepEnd ? kChainEnd : kPrepEnd) + 7) & ~7u;
  static constexpr uint32_t kBarA = kCommon;                  // mbarriers (chain 9, prep 16)
  static constexpr uint32_t kMisc = kBarA + 16 * 8;           // tmem slot
  static constexpr uint32_t kTotal = kMisc + 64;
  static constexpr uint32_t kAlloc = kTotal + 1024;
  static_assert(kAlloc <= 227 * 1024, "shared memory budget");
  static_assert((kInBytes % 1024) == 0 && (kInK % 1024) == 0 && (kInV % 1024) == 0 && (kUsb % 1024) == 0 &&
                    (kSb % 1024) == 0 && (kWm % 1024) == 0 && (kA1b % 1024) == 0 && (kA2b % 1024) == 0,
                "tile alignment");
  // byte offset of element (row, col) of a slice tile with `rows` rows
  __device__ static __forceinline__ uint32_t tile_off(int row, int col, int rows) {
    return (uint32_t)(col / kBlk) * (uint32_t)rows * kRB + sm100::mn_off<kRB>(row, col % kBlk);
  }
};

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}
__device__ __forceinline__ void st_shared_u16(uint32_t addr, unsigned short v) {
  asm volatile("st.shared.b16 [%0], %1;" ::"r"(addr), "h"(v) : "memory");
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
  void* o;              // T [total_T][Hv][128]
  float* state_out;
  uint8_t* ws;          // workspace (counter and flags zeroed before the launch)
  int n_seqs, Hqk, Hv, total_T;
  float scale;
  int n_chain_ctas;     // CTAs [0, n_chain_ctas) run state chains, the rest prepare
};

template <int DVP, typename T>
__global__ void __launch_bounds__(kThreads, 1)
prefill_pc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                  const __grid_constant__ CUtensorMap vmap, const __grid_constant__ CUtensorMap omap,
                  const Params p) {
  using L = Smem<DVP>;
  using namespace sm100;
  static_assert(DVP == 32 || DVP == 64 || DVP == 128, "slice width");
  constexpr uint32_t kFmt = Op16<T>::kFmt;   // every MMA operand is T: raw tiles and formed operands alike
  T* const out = static_cast<T*>(p.o);
  constexpr int kSlices = kD / DVP;
  constexpr int kHalf = DVP / 2;
  constexpr uint32_t kR = L::kR, kRB = L::kRB;
  constexpr int kPart = kHalf;   // epilogue columns per TMEM load
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(sm);
  int* round_start = reinterpret_cast<int*>(sm + L::kRounds);
  int* rbase = reinterpret_cast<int*>(sm + L::kRBase);
  // chain-role mbarriers (the prep role's sixteen are named where it starts)
  constexpr int NB = L::kNB;
  uint64_t* bar_full = reinterpret_cast<uint64_t*>(sm + L::kBarA);  // [NB] input buffer landed
  uint64_t* bar_free = bar_full + NB;                                // [NB] input buffer free again
  uint64_t* bar_mma = bar_full + 2 * NB;   // the Y product's commits
  uint64_t* bar_u = bar_mma + 1;           // U_s staged (the 4 U warps)
  uint64_t* bar_ds = bar_mma + 2;          // the dS product's commits
  uint64_t* bar_s = bar_mma + 3;           // the 16-bit state copy is written (the 8 compute warps)
  uint64_t* bar_o = bar_mma + 4;           // O staged for the TMA store (the 4 O warps)
  uint32_t* misc = reinterpret_cast<uint32_t*>(sm + L::kMisc);     // [0] tmem

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qd = warp & 3, ch = (warp >> 2) & 1;
  const int r128 = qd * 32 + lane;
  const int r64 = qd * 16 + (lane & 15);
  const bool lo16 = lane < 16;
  const int Hv = p.Hv, Hqk = p.Hqk;
  const long n_chains = (long)p.n_seqs * Hv;
  const long n_slice_chains = n_chains * kSlices;
  const int NC = p.n_chain_ctas;
  const int chains_per_round = NC / kSlices;
  const bool is_chain = (int)blockIdx.x < NC;
  const bool is_ctl = warp == kCtlWarp, is_rel = warp == kRelWarp;

  uint32_t* counter = reinterpret_cast<uint32_t*>(p.ws + Workspace::kCounter);
  uint32_t* ready = reinterpret_cast<uint32_t*>(p.ws + Workspace::kFlags);   // [position][slot]
  uint32_t* consumed = ready + (long)chains_per_round * kFlagStride;
  uint8_t* pkgs = p.ws + Workspace::pkg_offset(chains_per_round);

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
    // chain: a buffer is free once the compute warps and the MMA warp are done with
    // it and the releasing warp has seen its copy land (so that the releasing warp,
    // which waits by parity, never falls a phase behind); U_s and O are staged by
    // four warps each
    if (is_chain) {
      for (int i = 0; i < NB; ++i) {
        mbar_init(&bar_full[i], 1);
        mbar_init(&bar_free[i], 9);   // the 8 compute warps + the releasing warp
      }
      mbar_init(bar_mma, 1);
      mbar_init(bar_u, 4);            // the 4 U warps
      mbar_init(bar_ds, 1);
      mbar_init(bar_s, 8);            // the 8 compute warps
      mbar_init(bar_o, 4);            // the 4 O warps
    } else {
      for (int i = 0; i < 16; ++i) mbar_init(&bar_full[i], 1);
    }
    fence_mbar_init();
    prefetch_tensormap(&qmap);
    prefetch_tensormap(&kmap);
    if (is_chain) {
      prefetch_tensormap(&vmap);
      prefetch_tensormap(&omap);
    }
  }
  if (warp == 0) {
    tmem_alloc(&misc[0], kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];
  const uint32_t tlane = static_cast<uint32_t>(qd * 32) << 16;

  bool abort = false;

  if (is_chain) {
    // ============================== chain role ==============================
    // The CTA runs slice-chains sc = blockIdx.x + r NC in turn; input buffer
    // gc % NB holds the gc-th chunk it runs (package, k tile, v slice).
    auto decode_sc = [&](long sc, long& j, int& h, int& i0, int& t_begin, int& t_end) {
      j = sc / kSlices;
      h = (int)(j % Hv);
      i0 = (int)(sc % kSlices) * DVP;
      seq_bounds((int)(j / Hv), t_begin, t_end);
    };
    // the longest chain of the round that chain j belongs to (warp-collective)
    auto round_maxc = [&](long j, int q) {
      const long j0 = j - q;
      int m = 0;
      for (long jj = j0 + lane; jj < min(j0 + chains_per_round, n_chains); jj += 32) m = max(m, n_chunks_of(jj));
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, off));
      return m;
    };
    const int q = (int)blockIdx.x / kSlices;   // ring position (the same in every round)
    if (is_ctl) {
      // ---- issuing warp: per chunk, wait for the package's ready flag and a free input
      //      buffer, then copy package, k and v in ----
      const uint32_t* rdy = ready + q * kFlagStride;
      const uint8_t* ring = pkgs + (size_t)q * kRing * kPkgStride;
      long gc = 0;
      int base = 0;
      for (long sc = blockIdx.x; sc < n_slice_chains && !abort; sc += NC) {
        long j;
        int h, i0, t_begin, t_end;
        decode_sc(sc, j, h, i0, t_begin, t_end);
        const int hq = h / (Hv / Hqk);
        const int nch = (t_end - t_begin + kC - 1) / kC;
        const int maxc = round_maxc(j, q);
        if (!GDN_CHECK(j < n_chains && h < Hv && hq < Hqk && i0 + DVP <= kD && q < chains_per_round &&
                       0 <= t_begin && t_begin <= t_end && t_end <= p.total_T)) {
          abort = true;
          break;
        }
        for (int c = 0; c < nch; ++c, ++gc) {
          const int b = (int)(gc % NB);
          const int s = base + c, slot = s % kRing;
          if (!GDN_CHECK(s >= 0 && t_begin + c * kC < t_end)) { abort = true; break; }
          bool ok = true;
          if (lane == 0) ok = wait_flag_geq(&rdy[slot], (uint32_t)(s / kRing + 1));
          if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) { abort = true; break; }
          if (gc >= NB && !mbar_wait(&bar_free[b], (uint32_t)((gc - NB) / NB) & 1u)) { abort = true; break; }
          __syncwarp();
          fence_async_global();
          uint8_t* dst = sm + L::kIn + b * L::kInBytes;
          const int c0 = t_begin + c * kC;
          mbar_arrive_expect_tx_warp(&bar_full[b], kPkgCopy + 16384 + 64 * kR);
          bulk_load_warp(dst, ring + (size_t)slot * kPkgStride, kPkgCopy, &bar_full[b]);
          // (the chains' k reads are its last: the prep CTAs read it before the package exists)
          tma_load_3d_warp_hint(dst + L::kInK, &kmap, &bar_full[b], 0, hq, c0, l2_evict_first_policy());
          tma_load_3d_warp_hint(dst + L::kInK + 8192, &kmap, &bar_full[b], 64, hq, c0, l2_evict_first_policy());
#pragma unroll
          for (int vb = 0; vb < L::kBlocks; ++vb)
            tma_load_3d_warp_hint(dst + L::kInV + vb * 64 * L::kRB, &vmap, &bar_full[b], i0 + vb * L::kBlk, h, c0,
                                  l2_evict_first_policy());   // (its only reader)
        }
        base += maxc;
      }
    } else if (is_rel) {
      // ---- releasing warp: hands each ring slot back once its copy has landed, and
      //      counts the numbers a shorter chain leaves unused as read ----
      uint32_t* cns = consumed + q * kFlagStride;
      long gc = 0;
      int base = 0;
      for (long sc = blockIdx.x; sc < n_slice_chains && !abort; sc += NC) {
        long j;
        int h, i0, t_begin, t_end;
        decode_sc(sc, j, h, i0, t_begin, t_end);
        const int nch = (t_end - t_begin + kC - 1) / kC;
        const int maxc = round_maxc(j, q);
        if (!GDN_CHECK(q < chains_per_round && base >= 0 && maxc >= nch)) { abort = true; break; }
        for (int c = 0; c < nch; ++c, ++gc) {
          if (!mbar_wait(&bar_full[gc % NB], (uint32_t)(gc / NB) & 1u)) { abort = true; break; }
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&bar_free[gc % NB]);   // (the buffer is not refilled before this)
            red_add_release_gpu(&cns[(base + c) % kRing], 1u);
          }
        }
        if (abort) break;
        if (lane == 0)
          for (int c = nch; c < maxc; ++c) red_add_release_gpu(&cns[(base + c) % kRing], 1u);
        base += maxc;
      }
    } else if (warp == kMmaWarp || warp < 8) {
      constexpr uint32_t kIdY = idesc_f16kind(128, DVP, false, true, kFmt);
      // Each group of the chain's K-steps from one asm block (mma_run_warp) at 32-row slices,
      // one block a step at wider ones: measured side by side on the B200, either way round
      // costs 0.5-1 % of the call.
      constexpr bool kBatchedIssue = DVP == 32;
      constexpr uint32_t kIdDS = idesc_f16kind(128, DVP, true, true, kFmt);
      const uint32_t sSb = sbase + L::kSb;
      const uint32_t sUsb = sbase + L::kUsb;
      if (warp == kMmaWarp) {
        // ---- MMA warp: per chunk Y = A2 V + A1 S^T (rows 0-63 U, rows 64-127 O; A1 staged
        //      in TMEM by tcgen05.cp, so that only S^T streams from shared memory) into
        //      TMEM buffer gc & 1, then dS^T = K_raw^T U_s and, when the next chunk's
        //      data is in, its A2 V into the other Y buffer; it waits on the compute
        //      warps through mbarriers (bounded) ----
        auto issue_a2v = [&](int b, uint32_t ycol) {   // A2 V_raw of input buffer b, the first term of Y
          const uint32_t in = sbase + L::kIn + b * L::kInBytes;
          const uint64_t a2 = desc_kmajor(in + kPkgA2, 0, 0), v0 = desc_mnmajor(in + L::kInV, 0, kRB, 64 * kRB);
          if constexpr (kBatchedIssue)
            mma_run_warp<4, 2, kRB>(tmem + ycol, a2, v0, kIdY, 0u);
          else
            mma_k<4, true, 0, false, kRB>(tmem + ycol, a2, v0, kIdY, false);
        };
        // the package's A1 (input buffer b) into TMEM buffer ab, so that A1 S^T reads
        // only S^T from shared memory on the chain (the copy is ordered before it)
        auto stage_a1 = [&](int b, uint32_t ab) {
          const uint64_t a0 = desc_kmajor(sbase + L::kIn + b * L::kInBytes + kPkgA1, 0, 16384);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            tmem_cp_128x256b_warp(tmem + kColA1 + 64u * ab + 8u * kk, desc_advance(a0, kmajor_step(kk, 16384)));
        };
        const uint64_t s0 = desc_mnmajor(sSb, 0, kRB, 128 * kRB);   // S^T, the B operand of A1 S^T
        const uint64_t u0 = desc_mnmajor(sUsb, 0, kRB, 64 * kRB);   // U_s, the B operand of dS
        long gc = 0;
        bool early = false;
        uint32_t ph_u = 0, ph_s = 0;
        for (long sc = blockIdx.x; sc < n_slice_chains && !abort; sc += NC) {
          long j;
          int h, i0, t_begin, t_end;
          decode_sc(sc, j, h, i0, t_begin, t_end);
          const int nch = (t_end - t_begin + kC - 1) / kC;
          for (int c = 0; c < nch; ++c, ++gc) {
            const int b = (int)(gc % NB);
            const uint32_t in = sbase + L::kIn + b * L::kInBytes;
            const uint32_t ycol = kColY + 128u * (uint32_t)(gc & 1);   // two Y buffers in TMEM
            const uint32_t ab = (uint32_t)(gc & 1);                     // the A1 buffer in TMEM
            // (a first chunk from a zero state has no A1 S^T; its package carries no A1)
            const bool a1s = c > 0 || p.state_in != nullptr;
            if (!mbar_wait(&bar_full[b], (uint32_t)(gc / NB) & 1u) || !mbar_wait(bar_s, ph_s)) { abort = true; break; }
            ph_s ^= 1;
            __syncwarp();
            tc_fence_after();
            if (!early) issue_a2v(b, ycol);
            if (a1s) {
              if (early) {   // A1 was staged in TMEM while the previous chunk ran
                if constexpr (kBatchedIssue) {
                  mma8_tmem_a_run_warp<kRB>(tmem + ycol, tmem + kColA1 + 64u * ab, s0, kIdY);
                } else {
#pragma unroll
                  for (int kk = 0; kk < 8; ++kk)
                    mma_f16_tmem_a_warp(tmem + ycol, tmem + kColA1 + 64u * ab + 8u * kk,
                                        desc_advance(s0, mnmajor_step(kk, kRB)), kIdY, 1u);
                }
              } else {       // staging it now would only add a pass: read it from shared memory
                mma_k<8, true, 16384, false, kRB>(tmem + ycol, desc_kmajor(in + kPkgA1, 0, 16384), s0, kIdY, true);
              }
            }
            mma_commit_warp(bar_mma);
            const uint64_t kd = desc_mnmajor(in + L::kInK, 0, 128, 8192);   // K_raw^T, the A operand of dS
            if (!mbar_wait(bar_u, ph_u)) { abort = true; break; }
            ph_u ^= 1;
            __syncwarp();
            tc_fence_after();
            if constexpr (kBatchedIssue)
              mma_run_warp<4, 128, kRB>(tmem + kColDS, kd, u0, kIdDS, 0u);
            else
              mma_k<4, false, 128, false, kRB>(tmem + kColDS, kd, u0, kIdDS, false);
            mma_commit_warp(bar_ds);
            // the other Y buffer was last read in chunk gc - 1, whose epilogues all ended
            // before the compute warps' state update of that chunk (and so before bar_u);
            // the other A1 buffer was last read by chunk gc - 1's Y product, complete
            // before its U_s epilogue
            early = false;
            if (c + 1 < nch) {
              const int bn = (int)((gc + 1) % NB);
              const bool nxt = mbar_test_wait(&bar_full[bn], (uint32_t)((gc + 1) / NB) & 1u);
              if (__shfl_sync(0xffffffffu, nxt ? 1 : 0, 0)) {
                issue_a2v(bn, kColY + 128u * (uint32_t)((gc + 1) & 1));
                stage_a1(bn, (uint32_t)((gc + 1) & 1));   // (a later chunk of a chain always has A1)
                early = true;
              }
            }
          }
        }
      } else {
        // ---- compute warps: the Y and dS epilogues and the fp32 state ----
        // Every warp waits for the products on its own: Y and dS commit to separate
        // barriers, and neither product of the next chunk can complete before every
        // warp has arrived after reading this one (bar_s), so no warp can miss a
        // phase. The O warps meet on an mbarrier before the TMA store. No wait here
        // is unbounded: a warp whose wait runs out stops, and the others' waits
        // then run out in turn.
        long gc = 0;
        uint32_t ph_y = 0, ph_ds = 0, ph_o = 0;
        auto warp_arrive = [&](uint64_t* bar) {
          __syncwarp();
          if (lane == 0) mbar_arrive(bar);
        };
        for (long sc = blockIdx.x; sc < n_slice_chains && !abort; sc += NC) {
          long j;
          int h, i0, t_begin, t_end;
          decode_sc(sc, j, h, i0, t_begin, t_end);
          const int n = (int)(j / Hv);
          const int nch = (t_end - t_begin + kC - 1) / kC;

          const size_t s_off = ((size_t)n * Hv + h) * kD * kD + (size_t)(i0 + ch * kHalf) * kD + r128;
          if (!GDN_CHECK(n < p.n_seqs && h < Hv && i0 + DVP <= kD &&
                         s_off + (size_t)(kHalf - 1) * kD < (size_t)p.n_seqs * Hv * kD * kD)) {
            abort = true;
            break;
          }
          float Sreg[kHalf];
#pragma unroll
          for (int q2 = 0; q2 < kHalf; ++q2) Sreg[q2] = p.state_in ? __ldcs(p.state_in + s_off + (size_t)q2 * kD) : 0.f;
          auto store_state = [&]() {
#pragma unroll
            for (int c8 = 0; c8 < kHalf / 8; ++c8)
              st_shared_v4(sSb + L::tile_off(r128, ch * kHalf + 8 * c8, 128), pack8<T>(Sreg + 8 * c8));
          };
          if (nch > 0) {
            store_state();
            fence_async_smem();
            warp_arrive(bar_s);
          }

          for (int c = 0; c < nch; ++c, ++gc) {
            const int b = (int)(gc % NB);
            const uint32_t yb = (uint32_t)(gc & 1);   // the Y buffer in TMEM
            const uint32_t in = sbase + L::kIn + b * L::kInBytes;
            const uint8_t* in_g = sm + L::kIn + b * L::kInBytes;
            const int len = min(kC, t_end - (t_begin + c * kC));
            const bool o_tma = len == kC;
            if (!GDN_CHECK(len > 0 && t_begin + c * kC + len <= p.total_T)) { abort = true; break; }
            if (!mbar_wait(&bar_full[b], (uint32_t)(gc / NB) & 1u) || !mbar_wait(bar_mma, ph_y)) {   // Y
              abort = true;
              break;
            }
            ph_y ^= 1;
            tc_fence_after();
            {
              const float us = qd < 2 ? reinterpret_cast<const float*>(in_g + kPkgUs)[r128] : 0.f;
              T* orow = out + ((size_t)(t_begin + c * kC + (r128 & 63)) * Hv + h) * kD + i0 + ch * kHalf;
#pragma unroll
              for (int pp = 0; pp < kHalf / kPart; ++pp) {
                float yv[kPart];
                tmem_ld<kPart>(tmem + tlane + kColY + 128u * yb + ch * kHalf + pp * kPart, yv);
                if (qd < 2) {   // U_s = diag(us) U -> shared memory (T) for dS
#pragma unroll
                  for (int q2 = 0; q2 < kPart; ++q2) yv[q2] *= us;
#pragma unroll
                  for (int c8 = 0; c8 < kPart / 8; ++c8)
                    st_shared_v4(sUsb + L::tile_off(r128, ch * kHalf + pp * kPart + 8 * c8, 64), pack8<T>(yv + 8 * c8));
                } else if (o_tma) {   // O staged in the consumed v tile for the TMA store
#pragma unroll
                  for (int c8 = 0; c8 < kPart / 8; ++c8)
                    st_shared_v4(in + L::kInV + L::tile_off(r128 - 64, ch * kHalf + pp * kPart + 8 * c8, 64),
                                 pack8<T>(yv + 8 * c8));
                } else if (r128 - 64 < len) {   // a sequence's last, partial chunk: row by row
#pragma unroll
                  for (int c8 = 0; c8 < kPart / 8; ++c8)
                    *reinterpret_cast<uint4*>(orow + pp * kPart + 8 * c8) = pack8<T>(yv + 8 * c8);
                }
              }
            }
            fence_async_smem();
            tc_fence_before();
            if (qd < 2) {
              warp_arrive(bar_u);
            } else if (o_tma) {   // the O warps' staging is complete, then thread 64 stores the O tile
              warp_arrive(bar_o);
              if (tid == 64) {
                if (!mbar_wait(bar_o, ph_o)) {
                  abort = true;
                } else {
#pragma unroll
                  for (int vb = 0; vb < L::kBlocks; ++vb)
                    tma_store_3d_hint(&omap, in_g + L::kInV + vb * 64 * kRB, i0 + vb * L::kBlk, h, t_begin + c * kC,
                                      l2_evict_first_policy());
                  bulk_commit_group();
                }
              }
              ph_o ^= 1;
              abort = __shfl_sync(0xffffffffu, abort ? 1 : 0, 0) != 0;   // (warp-uniform)
              if (abort) break;
            }
            if (!mbar_wait(bar_ds, ph_ds)) { abort = true; break; }   // dS
            ph_ds ^= 1;
            tc_fence_after();
            {
              const float gL = *reinterpret_cast<const float*>(in_g + kPkgGL);
#pragma unroll
              for (int pp = 0; pp < kHalf / kPart; ++pp) {
                float ds[kPart];
                tmem_ld<kPart>(tmem + tlane + kColDS + ch * kHalf + pp * kPart, ds);
#pragma unroll
                for (int q2 = 0; q2 < kPart; ++q2) Sreg[pp * kPart + q2] = fmaf(gL, Sreg[pp * kPart + q2], ds[q2]);
              }
              store_state();
            }
            // each warp tells the MMA warp its state rows are written and it is done with
            // the buffer (no CTA-wide barrier here)
            fence_async_smem();
            tc_fence_before();
            // At 64-row slices and wider the state-written arrival does not wait for the O
            // tile's read (measured side by side on the B200: 0.6-0.8 % faster at 128-row
            // slices, 0.5 % slower at 32).
            if constexpr (DVP >= 64) {
              __syncwarp();
              if (lane == 0 && c + 1 < nch) mbar_arrive(bar_s);
              if (tid == 64) bulk_wait_read_all();   // the O tile has left the buffer
              __syncwarp();
              if (lane == 0) mbar_arrive(&bar_free[b]);
            } else {
              if (tid == 64) bulk_wait_read_all();   // the O tile has left the buffer
              __syncwarp();
              if (lane == 0) {
                if (c + 1 < nch) mbar_arrive(bar_s);
                mbar_arrive(&bar_free[b]);
              }
            }
          }
          if (abort) break;
#pragma unroll
          for (int q2 = 0; q2 < kHalf; ++q2) __stcs(p.state_out + s_off + (size_t)q2 * kD, Sreg[q2]);
        }
      }
    }
  } else {
    // ============================== prep role ===============================
    // The hand-over warp first prefetches into L2 the raw tiles and gates of the CTA's
    // first item (fixed: items [0, prep CTAs) go one to each) as it lies in round 0,
    // where it is chunk c of chain q with item = c P0 + q (P0 the round's chains), so
    // that the hand-over's loads find them there; a guess outside the chain's
    // chunks prefetches nothing.
    if (is_ctl) {
      const long p0 = min((long)chains_per_round, n_chains);
      const long item = (long)blockIdx.x - NC;
      if (p0 > 0 && item >= 0) {
        const long j = item % p0;
        int tb, te;
        seq_bounds((int)(j / Hv), tb, te);
        const int c0 = tb + (int)(item / p0) * kC;
        if (c0 < te) {
          const int h = (int)(j % Hv), hq = h / (Hv / Hqk);
          if (lane == 0) {
            tma_prefetch_3d(&kmap, 0, hq, c0);
            tma_prefetch_3d(&kmap, 64, hq, c0);
            tma_prefetch_3d(&qmap, 0, hq, c0);
            tma_prefetch_3d(&qmap, 64, hq, c0);
          }
          for (int e = lane; e < kC && c0 + e < te; e += 32) {
            prefetch_l2(p.g + (size_t)(c0 + e) * Hv + h);
            prefetch_l2(p.beta + (size_t)(c0 + e) * Hv + h);
          }
        }
      }
    }
    // round table: items of round r are [round_start[r], round_start[r+1])
    const int n_rounds = (int)min((n_slice_chains + NC - 1) / NC, (long)kMaxRounds);
    // the longest chain of each round (warps over rounds, lanes over its chains) ...
    for (int r = warp; r < n_rounds; r += kThreads / 32) {
      const long j0 = (long)r * chains_per_round;
      const long j1 = min(j0 + chains_per_round, n_chains);
      int maxc = 0;
      for (long jj = j0 + lane; jj < j1; jj += 32) maxc = max(maxc, n_chunks_of(jj));
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) maxc = max(maxc, __shfl_xor_sync(0xffffffffu, maxc, off));
      if (lane == 0) rbase[r + 1] = maxc;
    }
    __syncthreads();
    // ... then the prefix sums: items before round r, numbers before round r
    if (tid == 0) {
      int acc = 0, nb = 0;
      for (int r = 0; r < n_rounds; ++r) {
        const int maxc = rbase[r + 1];
        const long j0 = (long)r * chains_per_round;
        round_start[r] = acc;
        rbase[r] = nb;
        acc += (int)(min(j0 + chains_per_round, n_chains) - j0) * maxc;
        nb += maxc;
      }
      round_start[n_rounds] = acc;
    }
    __syncthreads();
    const int total_items = round_start[n_rounds];

    // prep-role mbarriers: a two-entry queue between the hand-over warp and the
    // compute warps, the compute warps' MMA commits, and the hand-offs of a
    // package from the compute warps to the writing warp, and back
    uint64_t* bar_pfull = bar_full;        // [2] hand-over -> compute: entry k & 1 (its tiles counted in bytes)
    uint64_t* bar_pmma = bar_full + 4;     // the compute warps' MMA commits
    uint64_t* bar_ppub = bar_full + 5;     // [2] writer -> hand-over: published, the entry may be reused
    uint64_t* bar_pstage = bar_full + 7;   // [2] compute -> writer: the package images are staged
    uint64_t* bar_psread = bar_full + 9;   // [2] writer -> compute: the staged images have been read
    // compute-warp barriers (named barrier 1 over warps 0-7)
    auto cbar = [&]() { named_bar_sync(1, kCompute); };
    auto cbar_and = [&](bool ok) { return named_bar_and(1, kCompute, ok); };
    uint32_t mma_phase = 0;
    // wait for an MMA commit with the compute warps' barrier (which also makes
    // the result consistent across them), or without it when the next barrier,
    // publish(ok), takes the decision: every MMA of the next stage is issued
    // after that barrier, so no thread can miss a phase of bar_pmma
    auto wait_mma = [&](bool also_ok = true) -> bool {
      bool ok = mbar_wait(bar_pmma, mma_phase) && also_ok;
      mma_phase ^= 1;
      ok = cbar_and(ok);
      tc_fence_after();
      return ok;
    };
    auto wait_mma_local = [&]() -> bool {
      const bool ok = mbar_wait(bar_pmma, mma_phase);
      mma_phase ^= 1;
      tc_fence_after();
      return ok;
    };
    // shared-memory writes -> visible to the tensor core; TMEM reads done; returns
    // whether `ok` holds on every compute thread
    auto publish = [&](bool ok) -> bool {
      fence_async_smem();
      tc_fence_before();
      ok = cbar_and(ok);
      tc_fence_after();
      return ok;
    };

    if (is_ctl) {
      // ---- hand-over warp: claim items, fetch gates and raw k, q tiles, wait for the
      //      ring slot and hand the item over; queue entry k & 1 is reused once the
      //      writing warp has published item k - 2 ----
      auto hand_over = [&](int k) -> bool {   // false once none is left (or a wait ran out)
        const int b = k & 1;
        uint32_t* qe = reinterpret_cast<uint32_t*>(sm + L::kQueue + b * L::kQueueBytes);
        int v = 0, c = 0, q = 0, s = 0;
        long j = 0;
        if (lane == 0) {
          // a CTA's first item is fixed (items [0, prep CTAs), one each: no contended
          // atomic on the way to the first packages); the counter numbers the rest
          bool first = k == 0;
          while (true) {
            const int item = first ? (int)blockIdx.x - NC : ((int)gridDim.x - NC) + (int)atomicAdd(counter, 1u);
            first = false;
            if (item >= total_items) break;
            int r = 0, hi = n_rounds - 1;   // the round holding the item
            while (r < hi) {
              const int mid = (r + hi + 1) >> 1;
              if (round_start[mid] <= item) r = mid;
              else hi = mid - 1;
            }
            const long j0 = (long)r * chains_per_round;
            const int cpr = (int)(min(j0 + chains_per_round, n_chains) - j0);
            const int local = item - round_start[r];
            c = local / cpr;
            q = local % cpr;
            j = j0 + q;
            s = rbase[r] + c;
            if (!GDN_CHECK(r >= 0 && r < n_rounds && cpr > 0 && local >= 0 && q < chains_per_round &&
                           j < n_chains && s >= 0))
              break;
            if (c < n_chunks_of(j)) { v = 1; break; }
          }
        }
        v = __shfl_sync(0xffffffffu, v, 0);
        c = __shfl_sync(0xffffffffu, c, 0);
        q = __shfl_sync(0xffffffffu, q, 0);
        s = __shfl_sync(0xffffffffu, s, 0);
        j = __shfl_sync(0xffffffffu, j, 0);
        bool ok = true;
        int len = 0, c0 = 0, h = 0;
        if (v) {
          h = (int)(j % Hv);
          int tb, te;
          seq_bounds((int)(j / Hv), tb, te);
          c0 = tb + c * kC;
          len = min(kC, te - c0);
          // the raw k, q tiles first: their latency covers the gates and the slot wait
          const int hq = h / (Hv / Hqk);
          if (!GDN_CHECK(0 <= c0 && len > 0 && c0 + len <= p.total_T && h < Hv && hq < Hqk)) {
            len = 0;   // (no gate is read; the tile loads below stay inside their tensor maps)
            v = 0;
          }
          uint8_t* kq = sm + L::kKQP + b * 32768;
          mbar_expect_tx_warp(&bar_pfull[b], 4 * 8192);
          tma_load_3d_warp(kq, &kmap, &bar_pfull[b], 0, hq, c0);
          tma_load_3d_warp(kq + 16384, &kmap, &bar_pfull[b], 64, hq, c0);
          // (q's only readers are the prep items of the group's v heads, handed out together)
          tma_load_3d_warp_hint(kq + 8192, &qmap, &bar_pfull[b], 0, hq, c0, l2_evict_first_policy());
          tma_load_3d_warp_hint(kq + 16384 + 8192, &qmap, &bar_pfull[b], 64, hq, c0, l2_evict_first_policy());
          float* qg = reinterpret_cast<float*>(qe + 16);
          float* qb = reinterpret_cast<float*>(qe + 80);
#pragma unroll
          for (int e = lane; e < kC; e += 32) {
            qg[e] = e < len ? p.g[(size_t)(c0 + e) * Hv + h] : 0.f;
            qb[e] = e < len ? p.beta[(size_t)(c0 + e) * Hv + h] : 0.f;
          }
          // (numbers below kRing have no previous occupant to wait for)
          if (lane == 0 && s >= kRing)
            ok = wait_flag_geq(&consumed[q * kFlagStride + s % kRing], (uint32_t)(kSlices * (s / kRing)));
          ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        }
        const bool go = v && ok && len > 0;
        if (lane == 0) {
          qe[0] = go ? 1u : 0u;
          qe[1] = (uint32_t)s;
          qe[2] = (uint32_t)q;
          qe[3] = (uint32_t)len;
          qe[4] = (uint32_t)c;
        }
        __syncwarp();
        // the arrival publishes the entry; the phase completes once the tiles are in too
        // (an item that gave up after starting its tiles still lets them land first)
        if (lane == 0) mbar_arrive(&bar_pfull[b]);
        return go;
      };
      for (int k = 0;; ++k) {
        if (k >= 2 && !mbar_wait(&bar_ppub[k & 1], (uint32_t)((k - 2) >> 1) & 1u)) break;
        __syncwarp();
        if (!hand_over(k)) break;
      }
    } else if (warp == kMmaWarp) {
      // ---- writing warp: copies each package the compute warps have staged out to its
      //      ring slot in bulk, tells them once the images have been read (they are
      //      overwritten from the next item's T stage on), and once the copies are
      //      complete (and ordered before it) releases the package's ready flag and
      //      hands the queue entry back ----
      for (int it = 0;; ++it) {
        const int b = it & 1;
        const uint32_t par = (uint32_t)(it >> 1) & 1u;
        if (!mbar_wait(&bar_pfull[b], par)) break;   // handed over (or the end marker)
        const uint32_t* qe = reinterpret_cast<const uint32_t*>(sm + L::kQueue + b * L::kQueueBytes);
        if (qe[0] == 0) break;
        if (!GDN_CHECK(qe[2] < (uint32_t)chains_per_round)) break;
        if (!mbar_wait(&bar_pstage[b], par)) break;
        // (a chain's first chunk from a zero state carries no A1)
        const bool need_a1 = qe[4] != 0 || p.state_in != nullptr;
        uint8_t* pkg = pkgs + ((size_t)qe[2] * kRing + qe[1] % kRing) * kPkgStride;
        if (lane == 0) {
          if (need_a1) {
            bulk_store(pkg + kPkgA1, sm + L::kWm, 8192);
            bulk_store(pkg + kPkgA1 + 16384, sm + L::kWm + 8192, 8192);
            bulk_store(pkg + kPkgA1 + 8192, sm + L::kA1b, 8192);
            bulk_store(pkg + kPkgA1 + 16384 + 8192, sm + L::kA1b + 8192, 8192);
          }
          bulk_store(pkg + kPkgA2, sm + L::kTu, 8192);
          bulk_store(pkg + kPkgA2 + 8192, sm + L::kA2b, 8192);
          bulk_store(pkg + kPkgUs, sm + L::kPv + 512 * b, kPkgCopy - kPkgUs);
          bulk_commit_group();
          bulk_wait_read_all();
          mbar_arrive(&bar_psread[b]);
          bulk_wait_all();
          fence_async_global();
          st_release_gpu(&ready[qe[2] * kFlagStride + qe[1] % kRing], qe[1] / kRing + 1);
          mbar_arrive(&bar_ppub[b]);
        }
        __syncwarp();
      }
    } else if (warp < 8) {
      // ---- compute warps ----
      constexpr uint32_t kIdG = idesc_f16kind(128, 64, false, false, kFmt);
      constexpr uint32_t kId64 = idesc_f16kind(64, 64, false, true, kFmt);
      float* vB = reinterpret_cast<float*>(sm + L::kVec) + 64;   // beta (after 64 spare floats)
      float* vRk = vB + 64;
      float* vRq = vRk + 64;
      float* vCk = vRq + 64;
      float* vCw = vCk + 64;
      float* vRho = vCw + 64;
      float* vGf = vRho + 64;                               // G_r
      float* Ad = reinterpret_cast<float*>(sm + L::kAd);

      // D's blocks off the diagonal are zero for every item (no other stage writes D)
      for (int e = tid; e < 64 * 6; e += kCompute) {
        const int row = e / 6, idx = e - row * 6, blk = row >> 4;
        const int cc = idx < 2 * blk ? idx : idx + 2;
        st_shared_v4(sbase + L::kDm + sw128_off(row, 8 * cc, 0), make_uint4(0, 0, 0, 0));
      }
      for (int it = 0; !abort; ++it) {
        const int b = it & 1;
        const uint32_t* qe = reinterpret_cast<const uint32_t*>(sm + L::kQueue + b * L::kQueueBytes);
        {
          const bool w = mbar_wait(&bar_pfull[b], (uint32_t)(it >> 1) & 1u);
          if (!cbar_and(w)) { abort = true; break; }
        }
        if (qe[0] == 0) break;
        const int len = (int)qe[3];
#ifdef GDN_DEBUG
        if (!cbar_and(GDN_CHECK(qe[2] < (uint32_t)chains_per_round && len > 0 && len <= kC))) {
          abort = true;
          break;
        }
#endif
        // a chain's first chunk from a zero state never multiplies A1 (S = 0): skip -W, P W
        const bool need_a1 = qe[4] != 0 || p.state_in != nullptr;
        float* pv = reinterpret_cast<float*>(sm + L::kPv + 512 * b);   // the package's vectors
        const uint32_t sKQ = sbase + L::kKQP + b * 32768;

        // ---- Gram [k;q] k^T on the tensor core; meanwhile the gates' scan, the norms and the row scales ----
        if (warp == 0) {
          const uint64_t g0 = desc_kmajor(sKQ, 0, 16384);   // (K 64-127 in the tile's second 16 KB)
          mma_run_warp<4, 2, 2>(tmem + kColG, g0, g0, kIdG, 0u);
          mma_run_warp<4, 2, 2>(tmem + kColG, desc_advance(g0, 16384), desc_advance(g0, 16384), kIdG, 1u);
          mma_commit_warp(bar_pmma);
        }
        // every warp scans the chunk's gates itself (two values a lane): G_r for rows lane, 32 + lane
        const float* qg = reinterpret_cast<const float*>(qe + 16);
        float g0 = qg[lane], g1 = qg[32 + lane];
        const bool nonpos = __all_sync(0xffffffffu, g0 <= 0.f && g1 <= 0.f);
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const float u0 = __shfl_up_sync(0xffffffffu, g0, off);
          const float u1 = __shfl_up_sync(0xffffffffu, g1, off);
          if (lane >= off) {
            g0 += u0;
            g1 += u1;
          }
        }
        const float s0 = __shfl_sync(0xffffffffu, g0, 31);
        g1 += s0;
        const float G0 = __shfl_sync(0xffffffffu, g0, 0);
        const float GL = __shfl_sync(0xffffffffu, len - 1 < 32 ? g0 : g1, (len - 1) & 31);
        const bool fast = nonpos && (G0 - GL) <= 160.f;
        const float gm = 0.5f * (G0 + GL);
        {   // squared norm of row 16 warp + lane / 2 of [k;q] (warps 0-3 k rows, 4-7 q rows) in two
            // halves on adjacent lanes, four accumulators a lane; then that row's scales
          const int nrow = 16 * warp + (lane >> 1), nhalf = lane & 1;
          float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
          for (int c8 = 0; c8 < 8; ++c8) {
            float f[8];
            unpack8<T>(ld_shared_v4(sKQ + sw128_off(nrow, 64 * nhalf + 8 * c8, 16384)), f);
            a0 = fmaf(f[0], f[0], a0);
            a1 = fmaf(f[1], f[1], a1);
            a2 = fmaf(f[2], f[2], a2);
            a3 = fmaf(f[3], f[3], a3);
            a0 = fmaf(f[4], f[4], a0);
            a1 = fmaf(f[5], f[5], a1);
            a2 = fmaf(f[6], f[6], a2);
            a3 = fmaf(f[7], f[7], a3);
          }
          const float part = (a0 + a1) + (a2 + a3);
          const float other = __shfl_xor_sync(0xffffffffu, part, 1);
          const float ss = nhalf ? other + part : part + other;   // (the first half's sum first)
          const int r = nrow & 63;
          const float Ga = __shfl_sync(0xffffffffu, g0, r & 31), Gb = __shfl_sync(0xffffffffu, g1, r & 31);
          const float Gr = r < 32 ? Ga : Gb;
          const float eg = expf(Gr);
          if (warp < 4) {
            const float rk = r < len ? 1.0f / sqrtf(ss + kNormEps) : 0.f;
            if (nhalf == 0) {
              vRk[r] = rk;
              vCk[r] = fast ? expf(gm - Gr) * rk : rk;
              pv[r] = expf(GL - Gr) * rk;
            } else {
              const float bt = reinterpret_cast<const float*>(qe + 80)[r];
              vB[r] = bt;
              vGf[r] = Gr;
              vCw[r] = -bt * eg * rk;
            }
          } else if (nhalf == 0) {
            const float rq = r < len ? p.scale / sqrtf(ss + kNormEps) : 0.f;
            vRq[r] = rq;
            vRho[r] = eg * rq;
          }
          if (tid == 0) {
            pv[64] = expf(GL);
            reinterpret_cast<int*>(pv)[65] = len;
          }
        }
        if (!wait_mma()) { abort = true; break; }   // (its barrier also publishes the vectors)

        // ---- A (diagonal blocks fp32, off-diagonal blocks T) and P ----
        {
          const int rr = r128 & 63;
          const float Gr = vGf[rr];
          float ck[32];   // this thread's 32 columns of vCk, in 16-byte loads (before the TMEM load)
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 t4 = reinterpret_cast<const float4*>(vCk + 32 * ch)[i];
            ck[4 * i] = t4.x;
            ck[4 * i + 1] = t4.y;
            ck[4 * i + 2] = t4.z;
            ck[4 * i + 3] = t4.w;
          }
          float gram[32];
          tmem_ld32(tmem + tlane + kColG + 32 * ch, gram);
          float x[32];
          if (qd < 2) {
            const float fr = vB[rr] * vRk[rr] * (fast ? expf(Gr - gm) : 1.f);
            if (fast) {
#pragma unroll
              for (int q2 = 0; q2 < 32; ++q2) {
                const int sidx = 32 * ch + q2;
                x[q2] = (sidx < rr) ? fr * ck[q2] * gram[q2] : 0.f;
              }
            } else {
#pragma unroll
              for (int q2 = 0; q2 < 32; ++q2) {
                const int sidx = 32 * ch + q2;
                x[q2] = (sidx < rr) ? fr * ck[q2] * expf(Gr - vGf[sidx]) * gram[q2] : 0.f;
              }
            }
            // the row's diagonal block (columns 16 blk .. 16 blk + 15) goes to A_d in fp32 and
            // is zeroed in A_o; it lies in this thread's 32 columns when blk / 2 == ch (the
            // columns left of it are kept, those right of it are already zero)
            const int blk = rr >> 4;
            if ((blk >> 1) == ch) {
              float4* dst = reinterpret_cast<float4*>(Ad + (blk * 16 + (rr & 15)) * L::kAdRow);
              if (blk & 1) {   // (constant indices keep x in registers)
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4)
                  dst[q4] = make_float4(x[16 + 4 * q4], x[17 + 4 * q4], x[18 + 4 * q4], x[19 + 4 * q4]);
#pragma unroll
                for (int q2 = 16; q2 < 32; ++q2) x[q2] = 0.f;
              } else {
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4)
                  dst[q4] = make_float4(x[4 * q4], x[1 + 4 * q4], x[2 + 4 * q4], x[3 + 4 * q4]);
#pragma unroll
                for (int q2 = 0; q2 < 16; ++q2) x[q2] = 0.f;
              }
            }
#pragma unroll
            for (int c8 = 0; c8 < 4; ++c8)
              st_shared_v4(sbase + L::kAo + sw128_off(rr, 32 * ch + 8 * c8, 0), pack8<T>(x + 8 * c8));
          } else {
            const float fr = vRq[rr] * (fast ? expf(Gr - gm) : 1.f);
            if (fast) {
#pragma unroll
              for (int q2 = 0; q2 < 32; ++q2) {
                const int sidx = 32 * ch + q2;
                x[q2] = (sidx <= rr) ? fr * ck[q2] * gram[q2] : 0.f;
              }
            } else {
#pragma unroll
              for (int q2 = 0; q2 < 32; ++q2) {
                const int sidx = 32 * ch + q2;
                x[q2] = (sidx <= rr) ? fr * ck[q2] * expf(Gr - vGf[sidx]) * gram[q2] : 0.f;
              }
            }
#pragma unroll
            for (int c8 = 0; c8 < 4; ++c8)
              st_shared_v4(sbase + L::kPm + sw128_off(rr, 32 * ch + 8 * c8, 0), pack8<T>(x + 8 * c8));
          }
        }

        // ---- D = (I + A_d)^-1, by the two warps that wrote A_d's blocks (warp 0 blocks 0-1,
        //      warp 5 blocks 2-3: row 16 blk + i of block blk is lane 16 (blk & 1) + i's);
        //      D's other blocks are zero from before the first item ----
        if (warp == 0 || warp == 5) {
          __syncwarp();
          const int blk = (warp == 5 ? 2 : 0) + (lane >> 4), jj = lane & 15;
          const float* Ab = Ad + blk * 16 * L::kAdRow;
          float xs[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float acc0 = 0.f, acc1 = 0.f;   // two chains halve the dependent FMA latency
#pragma unroll
            for (int k2 = 0; k2 + 1 < i; k2 += 2) {
              acc0 = fmaf(Ab[i * L::kAdRow + k2], xs[k2], acc0);
              acc1 = fmaf(Ab[i * L::kAdRow + k2 + 1], xs[k2 + 1], acc1);
            }
            if (i & 1) acc0 = fmaf(Ab[i * L::kAdRow + i - 1], xs[i - 1], acc0);
            xs[i] = (i == jj) ? 1.f : (i > jj ? -(acc0 + acc1) : 0.f);
          }
#pragma unroll
          for (int i = 0; i < 16; ++i)
            st_shared_u16(sbase + L::kDm + sw128_off(16 * blk + i, 16 * blk + jj, 0), Op16<T>::one(xs[i]));
        }
        publish(true);

        // ---- N = D A_o ----
        if (warp == 0) {
          mma_run_warp<4, 2, 128>(tmem + kColN, desc_kmajor(sbase + L::kDm, 0, 0),
                                        desc_mnmajor(sbase + L::kAo, 0, 128, 8192), kId64, 0u);
          mma_commit_warp(bar_pmma);
        }
        const bool ok_n = wait_mma_local();
        {
          float v[32];
          tmem_ld32(tmem + tlane + kColN + 32 * ch, v);
          if (lo16) {
#pragma unroll
            for (int c8 = 0; c8 < 4; ++c8)
              st_shared_v4(sbase + L::kNm + sw128_off(r64, 32 * ch + 8 * c8, 0), pack8<T>(v + 8 * c8));
          }
        }
        if (!publish(ok_n)) { abort = true; break; }

        // ---- N D (lanes 0-15) and N^2 (lanes 16-31) ----
        if (warp == 0) {
          const uint64_t nm = desc_kmajor(sbase + L::kNm, 0, 0);
          mma_run_warp<4, 2, 128>(tmem + kColS2, nm, desc_mnmajor(sbase + L::kDm, 0, 128, 8192), kId64, 0u);
          mma_run_warp<4, 2, 128>(tmem + (16u << 16) + kColS2, nm, desc_mnmajor(sbase + L::kNm, 0, 128, 8192),
                                        kId64, 0u);
          mma_commit_warp(bar_pmma);
        }
        uint4 dq[4];   // (D is final since its stage: read before the wait)
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8) dq[c8] = ld_shared_v4(sbase + L::kDm + sw128_off(r64, 32 * ch + 8 * c8, 0));
        const bool ok_s2 = wait_mma_local();
        float E[32];   // lanes 0-15: columns 32ch..32ch+31 of row r64 of E = D - N D (fp32)
        {
          float v[32];
          tmem_ld32(tmem + tlane + kColS2 + 32 * ch, v);
          if (lo16) {
#pragma unroll
            for (int c8 = 0; c8 < 4; ++c8) {
              float df[8];
              unpack8<T>(dq[c8], df);
#pragma unroll
              for (int e = 0; e < 8; ++e) E[8 * c8 + e] = df[e] - v[8 * c8 + e];
              st_shared_v4(sbase + L::kEm + sw128_off(r64, 32 * ch + 8 * c8, 0), pack8<T>(E + 8 * c8));
            }
          } else {
#pragma unroll
            for (int c8 = 0; c8 < 4; ++c8)
              st_shared_v4(sbase + L::kN2 + sw128_off(r64, 32 * ch + 8 * c8, 0), pack8<T>(v + 8 * c8));
          }
        }
        // (the T stage starts overwriting the previous package's images: wait until they are read)
        const bool ok_rd = tid != 0 || it == 0 || mbar_wait(&bar_psread[(it - 1) & 1], (uint32_t)((it - 1) >> 1) & 1u);
        if (!publish(ok_s2 && ok_rd)) { abort = true; break; }

        // ---- Z = N^2 E ; T = E + Z -> T_u (shared and package), -T_w (shared) ----
        if (warp == 0) {
          mma_run_warp<4, 2, 128>(tmem + kColZ, desc_kmajor(sbase + L::kN2, 0, 0),
                                        desc_mnmajor(sbase + L::kEm, 0, 128, 8192), kId64, 0u);
          mma_commit_warp(bar_pmma);
        }
        const bool ok_z = wait_mma_local();
        {
          float z[32];
          tmem_ld32(tmem + tlane + kColZ + 32 * ch, z);
          if (lo16) {
#pragma unroll
            for (int c8 = 0; c8 < 4; ++c8) {
              float tu[8], tw[8], bb[8], ww[8];
              {
                const float4* b4 = reinterpret_cast<const float4*>(vB + 32 * ch + 8 * c8);
                const float4* w4 = reinterpret_cast<const float4*>(vCw + 32 * ch + 8 * c8);
                const float4 b0 = b4[0], b1 = b4[1], w0 = w4[0], w1 = w4[1];
                bb[0] = b0.x; bb[1] = b0.y; bb[2] = b0.z; bb[3] = b0.w;
                bb[4] = b1.x; bb[5] = b1.y; bb[6] = b1.z; bb[7] = b1.w;
                ww[0] = w0.x; ww[1] = w0.y; ww[2] = w0.z; ww[3] = w0.w;
                ww[4] = w1.x; ww[5] = w1.y; ww[6] = w1.z; ww[7] = w1.w;
              }
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const float t = E[8 * c8 + e] + z[8 * c8 + e];
                tu[e] = t * bb[e];
                tw[e] = t * ww[e];
              }
              const uint32_t off = sw128_off(r64, 32 * ch + 8 * c8, 0);
              st_shared_v4(sbase + L::kTu + off, pack8<T>(tu));
              st_shared_v4(sbase + L::kTw + off, pack8<T>(tw));
            }
          }
        }
        if (!publish(ok_z)) { abort = true; break; }

        // ---- -W = (-T_w) K_raw -> shared (operand of P W and A1 rows 0-63); the two
        //      column halves go to the two lane halves so that every thread has work ----
        const int dhalf = 64 * (lane >> 4) + 32 * ch;   // this thread's 32 columns of a d_k-wide row
        if (need_a1) {
          if (warp == 0) {
            const uint64_t tw = desc_kmajor(sbase + L::kTw, 0, 0);
            mma_run_warp<4, 2, 128>(tmem + kColW, tw, desc_mnmajor(sKQ, 0, 128, 16384), kId64, 0u);
            mma_run_warp<4, 2, 128>(tmem + (16u << 16) + kColW, tw, desc_mnmajor(sKQ + 16384, 0, 128, 16384),
                                          kId64, 0u);
            mma_commit_warp(bar_pmma);
          }
          const bool ok_w = wait_mma_local();
          {
            float w[32];
            tmem_ld32(tmem + tlane + kColW + 32 * ch, w);
#pragma unroll
            for (int c8 = 0; c8 < 4; ++c8)
              st_shared_v4(sbase + L::kWm + sw128_off(r64, dhalf + 8 * c8, 8192), pack8<T>(w + 8 * c8));
          }
          if (!publish(ok_w)) { abort = true; break; }
        }

        // ---- -P W and P T_u -> A1 rows 64-127 = rho Q_raw - P W, A2 rows 64-127 = P T_u ----
        if (warp == 0) {
          if (need_a1) {
            mma_run_warp<4, 2, 128>(tmem + kColPW, desc_kmajor(sbase + L::kPm, 0, 0),
                                          desc_mnmajor(sbase + L::kWm, 0, 128, 8192), kId64, 0u);
            mma_run_warp<4, 2, 128>(tmem + (16u << 16) + kColPW, desc_kmajor(sbase + L::kPm, 0, 0),
                                          desc_mnmajor(sbase + L::kWm + 8192, 0, 128, 8192), kId64, 0u);
          }
          mma_run_warp<4, 2, 128>(tmem + kColPT, desc_kmajor(sbase + L::kPm, 0, 0),
                                        desc_mnmajor(sbase + L::kTu, 0, 128, 8192), kId64, 0u);
          mma_commit_warp(bar_pmma);
        }
        uint4 qq[4];   // (the raw q tile and rho are final: read before the wait)
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8) qq[c8] = ld_shared_v4(sKQ + sw128_off(64 + r64, dhalf + 8 * c8, 16384));
        const float rho = vRho[r64];
        const bool ok_pw = wait_mma_local();
        {
          if (need_a1) {
            float pw[32];
            tmem_ld32(tmem + tlane + kColPW + 32 * ch, pw);
#pragma unroll
            for (int c8 = 0; c8 < 4; ++c8) {
              const int d = dhalf + 8 * c8;
              float qf[8], a[8];
              unpack8<T>(qq[c8], qf);
#pragma unroll
              for (int e = 0; e < 8; ++e) a[e] = fmaf(rho, qf[e], pw[8 * c8 + e]);
              st_shared_v4(sbase + L::kA1b + sw128_off(r64, d, 8192), pack8<T>(a));
            }
          }
          float pt[32];
          tmem_ld32(tmem + tlane + kColPT + 32 * ch, pt);
          if (lo16) {
#pragma unroll
            for (int c8 = 0; c8 < 4; ++c8)
              st_shared_v4(sbase + L::kA2b + sw128_off(r64, 32 * ch + 8 * c8, 0), pack8<T>(pt + 8 * c8));
          }
        }
        // ---- the package images are complete: the writing warp copies them out ----
        if (!publish(ok_pw)) { abort = true; break; }
        if (tid == 0) mbar_arrive(&bar_pstage[b]);
      }
    }
  }

  if (tid == 0) bulk_wait_all();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace pc
}  // namespace gdn
