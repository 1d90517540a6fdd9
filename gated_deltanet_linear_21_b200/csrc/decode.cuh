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
// Layout: a row of DK fp32 is spread over DK/4 lanes as float4 (16-byte,
// fully coalesced accesses); a warp holds NB row-slots in registers at once
// so each lane keeps NB independent 16-byte loads in flight. Dot products
// are reduced with butterfly shuffles inside the row's lane group.
#pragma once

#include "common.cuh"

namespace gdn {

template <int DK>
struct DecodeShape {
  static constexpr int kLanesPerRow = DK / 4;
  static constexpr int kRowsPerSlot = 32 / kLanesPerRow;
  static constexpr int kSlots = 8 / kRowsPerSlot > 0 ? 8 / kRowsPerSlot : 1;  // 8 rows per warp
  static constexpr int kRowsPerWarp = kRowsPerSlot * kSlots;
  static constexpr int kWarps = 1;   // one-warp CTAs: the most independent loads in flight per SM
  static constexpr int kRowsPerCta = kRowsPerWarp * kWarps;
};

__device__ __forceinline__ float dot4(float4 a, float4 b) {
  return a.x * b.x + a.y * b.y + a.z * b.z + a.w * b.w;
}

// grid: (B * Hv, ceil(dv / kRowsPerCta)); block: kWarps * 32
template <typename TIO, int DK>
__global__ void __launch_bounds__(DecodeShape<DK>::kWarps * 32)
decode_step_kernel(const TIO* __restrict__ q, const TIO* __restrict__ k,
                   const TIO* __restrict__ v, const float* __restrict__ g,
                   const float* __restrict__ beta, float* __restrict__ state,
                   int Hqk, int Hv, int dv, float scale, TIO* __restrict__ o) {
  using Sh = DecodeShape<DK>;
  constexpr int LPR = Sh::kLanesPerRow;
  const int bh = blockIdx.x;                 // b * Hv + h
  const int b = bh / Hv, h = bh - b * Hv;
  const int hq = h / (Hv / Hqk);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int sub = lane % LPR;                // float4 index within the row
  const int slot_row = lane / LPR;           // row within a slot

  // --- the state rows and v first: their latency covers the q, k normalisation ---
  const int row0 = blockIdx.y * Sh::kRowsPerCta + warp * Sh::kRowsPerWarp + slot_row;
  float4* S = reinterpret_cast<float4*>(state + (size_t)bh * dv * DK);
  float4 s[Sh::kSlots];
#pragma unroll
  for (int j = 0; j < Sh::kSlots; ++j) {
    const int r = row0 + j * Sh::kRowsPerSlot;
    s[j] = r < dv ? ld_stream(S + (size_t)r * LPR + sub) : make_float4(0.f, 0.f, 0.f, 0.f);
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
  const size_t qk_off = ((size_t)b * Hqk + hq) * DK + 4 * sub;
  float4 kr = load4(k + qk_off);
  float4 qr = load4(q + qk_off);
  const float kinv = 1.0f / sqrtf(group_sum<LPR>(dot4(kr, kr)) + kNormEps);
  const float qinv = scale / sqrtf(group_sum<LPR>(dot4(qr, qr)) + kNormEps);
  const float4 kh = make_float4(kr.x * kinv, kr.y * kinv, kr.z * kinv, kr.w * kinv);
  const float4 qh = make_float4(qr.x * qinv, qr.y * qinv, qr.z * qinv, qr.w * qinv);
  const float kq = group_sum<LPR>(dot4(kh, qh));

#pragma unroll
  for (int j = 0; j < Sh::kSlots; ++j) {
    const float a = group_sum<LPR>(dot4(s[j], kh));
    const float bq = group_sum<LPR>(dot4(s[j], qh));
    const int r = row0 + j * Sh::kRowsPerSlot;
    const float delta = bt * (vv[j] - alpha * a);
    if (r < dv) {
      float4 ns;
      ns.x = alpha * s[j].x + delta * kh.x;
      ns.y = alpha * s[j].y + delta * kh.y;
      ns.z = alpha * s[j].z + delta * kh.z;
      ns.w = alpha * s[j].w + delta * kh.w;
      st_stream(S + (size_t)r * LPR + sub, ns);
      if (sub == 0) o[(size_t)bh * dv + r] = from_f32<TIO>(alpha * bq + delta * kq);
    }
  }
}

}  // namespace gdn
