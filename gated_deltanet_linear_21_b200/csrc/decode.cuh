// Fused single-token decode step of the Gated DeltaNet mixer.
//
// The Herbert Metal article fuses "the whole DeltaNet recurrence step" into
// one launch ("One level down: #004 the same compiler on Apple's chips",
// section "Decode"), and the series treats decode as bound by the bytes it
// must move ("On descend d'un cran : #001 un compilateur pour moteur de LLM",
// section "Ce que coûte un token"; "#002", section "Le décodage : la mémoire
// décide"). Here the step is one kernel that streams every fp32 state row
// exactly once from HBM and back:
//
//   per (sequence b, value head h), with q^, k^ L2-normalised (q^ scaled):
//     a_i = S_i . k^,  b_i = S_i . q^                     (one pass over row i)
//     delta_i = beta (v_i - alpha a_i)
//     S'_i = alpha S_i + delta_i k^                        (written in place)
//     o_i  = alpha b_i + delta_i (k^ . q^)                  (= S'_i . q^)
//
// which is the gated delta rule S' = alpha S (I - beta k^ k^^T) + beta v k^^T,
// o = S' q^ with the product distributed so the row is read once.
//
// Layout: a row of DK state values is spread over DK/4 (fp32) or DK/8 (bf16)
// lanes as 16-byte chunks (fully coalesced accesses); a warp holds several
// row-slots in registers at once so each lane keeps several independent
// 16-byte loads in flight. Dot products are reduced with butterfly shuffles
// inside the row's lane group. The state may be stored in fp32 or in bf16
// (rounded to nearest even after each step); the arithmetic is fp32 either
// way.
#pragma once

#include "common.cuh"

namespace gdn {

// 16 bytes of a state row: 4 fp32 or 8 bf16 values, moved with streaming
// (evict-first) accesses since every state element is touched once per step.
template <typename TS> struct StateChunk;
template <> struct StateChunk<float> {
  static constexpr int kElems = 4;
  static __device__ __forceinline__ void load(const float* p, float* x) {
    const float4 v = ld_stream(reinterpret_cast<const float4*>(p));
    x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
  }
  static __device__ __forceinline__ void store(float* p, const float* x) {
    st_stream(reinterpret_cast<float4*>(p), make_float4(x[0], x[1], x[2], x[3]));
  }
};
template <> struct StateChunk<__nv_bfloat16> {   // stored rounded to nearest even
  static constexpr int kElems = 8;
  static __device__ __forceinline__ void load(const __nv_bfloat16* p, float* x) {
    const uint4 v = __ldcs(reinterpret_cast<const uint4*>(p));
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(h[i]);
      x[2 * i] = f.x;
      x[2 * i + 1] = f.y;
    }
  }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, const float* x) {
    uint4 v;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
    __stcs(reinterpret_cast<uint4*>(p), v);
  }
};

// E consecutive q/k elements as fp32 (E = 4 or 8)
template <int E, typename T>
__device__ __forceinline__ void load_vec(const T* p, float* x) {
#pragma unroll
  for (int i = 0; i < E; i += 4) {
    const float4 v = load4(p + i);
    x[i] = v.x; x[i + 1] = v.y; x[i + 2] = v.z; x[i + 3] = v.w;
  }
}

template <int DK, typename TS>
struct DecodeShape {
  static constexpr int kElems = StateChunk<TS>::kElems;      // state elements per lane access
  static constexpr int kLanesPerRow = DK / kElems;
  static constexpr int kRowsPerSlot = 32 / kLanesPerRow;
  // 4 fp32 rows or 16 bf16 rows per warp: at d_k = 128 every lane keeps 4 (fp32) or 8
  // (bf16) independent 16-byte loads in flight (measured on B200 at 64 sequences x 32
  // heads: 4 fp32 rows 47.2 us a step against 49.1 with 8 and 70 with 2, and 47.4 against
  // 49.4 with 3, 47.9 with 5 and 47.6 with 6; 16 bf16 rows 30.1 against 31.7 with 8)
  static constexpr int kRowsTarget = sizeof(TS) == 4 ? 4 : 16;
  static constexpr int kSlots = kRowsTarget / kRowsPerSlot > 0 ? kRowsTarget / kRowsPerSlot : 1;
  static constexpr int kRowsPerWarp = kRowsPerSlot * kSlots;
  static constexpr int kWarps = 1;   // one-warp CTAs: the most independent loads in flight per SM
  static constexpr int kRowsPerCta = kRowsPerWarp * kWarps;
};

// grid: (B * Hv, ceil(dv / kRowsPerCta)); block: kWarps * 32
template <typename TIO, int DK, typename TS>
__global__ void __launch_bounds__(DecodeShape<DK, TS>::kWarps * 32)
decode_step_kernel(const TIO* __restrict__ q, const TIO* __restrict__ k,
                   const TIO* __restrict__ v, const float* __restrict__ g,
                   const float* __restrict__ beta, TS* __restrict__ state,
                   int Hqk, int Hv, int dv, float scale, TIO* __restrict__ o) {
  using Sh = DecodeShape<DK, TS>;
  constexpr int E = Sh::kElems;
  constexpr int LPR = Sh::kLanesPerRow;
  const int bh = blockIdx.x;                 // b * Hv + h
  const int b = bh / Hv, h = bh - b * Hv;
  const int hq = h / (Hv / Hqk);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int sub = lane % LPR;                // 16-byte chunk within the row
  const int slot_row = lane / LPR;           // row within a slot

  // --- the state rows and v first: their latency covers the q, k normalisation ---
  const int row0 = blockIdx.y * Sh::kRowsPerCta + warp * Sh::kRowsPerWarp + slot_row;
  TS* S = state + (size_t)bh * dv * DK;
  float s[Sh::kSlots][E];
#pragma unroll
  for (int j = 0; j < Sh::kSlots; ++j) {
    const int r = row0 + j * Sh::kRowsPerSlot;
    if (r < dv) {
      StateChunk<TS>::load(S + (size_t)r * DK + E * sub, s[j]);
    } else {
#pragma unroll
      for (int e = 0; e < E; ++e) s[j][e] = 0.f;
    }
  }
  float vv[Sh::kSlots];
#pragma unroll
  for (int j = 0; j < Sh::kSlots; ++j) {
    const int r = row0 + j * Sh::kRowsPerSlot;
    vv[j] = r < dv ? to_f32(v[(size_t)bh * dv + r]) : 0.f;
  }
  const float alpha = expf(g[bh]);
  const float bt = beta[bh];

  // --- normalise q and k (every row group computes the same values) ---
  const size_t qk_off = ((size_t)b * Hqk + hq) * DK + E * sub;
  float kh[E], qh[E];
  load_vec<E>(k + qk_off, kh);
  load_vec<E>(q + qk_off, qh);
  float kk = 0.f, qq = 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    kk = fmaf(kh[e], kh[e], kk);
    qq = fmaf(qh[e], qh[e], qq);
  }
  const float kinv = 1.0f / sqrtf(group_sum<LPR>(kk) + kNormEps);
  const float qinv = scale / sqrtf(group_sum<LPR>(qq) + kNormEps);
  float kq = 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    kh[e] *= kinv;
    qh[e] *= qinv;
    kq = fmaf(kh[e], qh[e], kq);
  }
  kq = group_sum<LPR>(kq);

#pragma unroll
  for (int j = 0; j < Sh::kSlots; ++j) {
    float a = 0.f, bq = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      a = fmaf(s[j][e], kh[e], a);
      bq = fmaf(s[j][e], qh[e], bq);
    }
    a = group_sum<LPR>(a);
    bq = group_sum<LPR>(bq);
    const int r = row0 + j * Sh::kRowsPerSlot;
    const float delta = bt * (vv[j] - alpha * a);
    if (r < dv) {
      float ns[E];
#pragma unroll
      for (int e = 0; e < E; ++e) ns[e] = alpha * s[j][e] + delta * kh[e];
      StateChunk<TS>::store(S + (size_t)r * DK + E * sub, ns);
      if (sub == 0) o[(size_t)bh * dv + r] = from_f32<TIO>(alpha * bq + delta * kq);
    }
  }
}

}  // namespace gdn
