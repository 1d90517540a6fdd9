// C ABI of libgdn.so: argument checks, kernel selection and launches.
// Declared and documented in include/gdn.h.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <set>
#include <string>
#include <algorithm>
#include <utility>

#include "gdn.h"
#include "common.cuh"
#include "decode.cuh"
#include "prefill_simt.cuh"
#include "prefill_pc.cuh"

#include <cudaTypedefs.h>

namespace {

thread_local std::string t_last_error;

gdn_status fail(gdn_status s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
gdn_status fail(gdn_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  t_last_error = buf;
  return s;
}

gdn_status ok() {
  t_last_error.clear();
  return GDN_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
bool head_dim_ok(int d) { return d == 16 || d == 32 || d == 64 || d == 128; }
bool dtype_ok(gdn_dtype dtype) { return dtype == GDN_BF16 || dtype == GDN_F32 || dtype == GDN_F16; }

// Allow a kernel the full opt-in shared memory, once per (kernel, device), so
// that later calls (including ones inside CUDA-graph capture) only launch.
constexpr size_t kSmemOptIn = 227 * 1024;
template <typename F>
gdn_status allow_smem(F* kern, const char* what) {
  static std::mutex mu;
  static std::set<std::pair<const void*, int>> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  std::lock_guard<std::mutex> lock(mu);
  const auto key = std::make_pair(reinterpret_cast<const void*>(kern), dev);
  if (done.count(key)) return GDN_OK;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemOptIn);
  if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  done.insert(key);
  return GDN_OK;
}

gdn_status launch_status(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "%s: launch failed: %s", what, cudaGetErrorString(e));
  return ok();
}

// ---------------------------------------------------------------- decode ---
template <typename TIO, int DK, typename TS>
gdn_status launch_decode(const void* q, const void* k, const void* v, const float* g,
                         const float* beta, TS* state, int B, int Hqk, int Hv, int dv,
                         float scale, void* o, cudaStream_t st) {
  using Sh = gdn::DecodeShape<DK, TS>;
  dim3 grid((unsigned)(B * Hv), (unsigned)((dv + Sh::kRowsPerCta - 1) / Sh::kRowsPerCta));
  gdn::decode_step_kernel<TIO, DK, TS><<<grid, Sh::kWarps * 32, 0, st>>>(
      static_cast<const TIO*>(q), static_cast<const TIO*>(k), static_cast<const TIO*>(v), g, beta,
      state, Hqk, Hv, dv, scale, static_cast<TIO*>(o));
  return launch_status("gdn_decode");
}

template <typename TIO, typename TS>
gdn_status dispatch_decode(const void* q, const void* k, const void* v, const float* g,
                           const float* beta, TS* state, int B, int Hqk, int Hv, int dk,
                           int dv, float scale, void* o, cudaStream_t st) {
  switch (dk) {
    case 16: return launch_decode<TIO, 16, TS>(q, k, v, g, beta, state, B, Hqk, Hv, dv, scale, o, st);
    case 32: return launch_decode<TIO, 32, TS>(q, k, v, g, beta, state, B, Hqk, Hv, dv, scale, o, st);
    case 64: return launch_decode<TIO, 64, TS>(q, k, v, g, beta, state, B, Hqk, Hv, dv, scale, o, st);
    default: return launch_decode<TIO, 128, TS>(q, k, v, g, beta, state, B, Hqk, Hv, dv, scale, o, st);
  }
}

// Host checks shared by the decode entry points; GDN_OK when the call may proceed
// (B == 0 is returned as done through *done).
gdn_status check_decode(const char* fn, const void* q, const void* k, const void* v, const float* g,
                        const float* beta, const void* state, int B, int Hqk, int Hv, int dk, int dv,
                        gdn_dtype dtype, const void* o, bool* done) {
  *done = false;
  if (B < 0) return fail(GDN_ERR_INVALID_ARG, "%s: B=%d < 0", fn, B);
  if (Hqk <= 0 || Hv <= 0 || Hv % Hqk != 0)
    return fail(GDN_ERR_INVALID_ARG, "%s: Hv=%d must be a positive multiple of Hqk=%d", fn, Hv, Hqk);
  if (!head_dim_ok(dk) || !head_dim_ok(dv))
    return fail(GDN_ERR_UNSUPPORTED, "%s: dk=%d, dv=%d (supported: 16, 32, 64, 128)", fn, dk, dv);
  if (!dtype_ok(dtype)) return fail(GDN_ERR_INVALID_ARG, "%s: unknown dtype %d", fn, (int)dtype);
  if ((int64_t)B * Hv > 0x7fffffff) return fail(GDN_ERR_INVALID_ARG, "%s: B*Hv too large", fn);
  if (B == 0) {
    *done = true;
    return ok();
  }
  if (!q || !k || !v || !g || !beta || !state || !o)
    return fail(GDN_ERR_INVALID_ARG, "%s: pointers must not be NULL", fn);
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(state))
    return fail(GDN_ERR_INVALID_ARG, "%s: q, k, v, o and state must be 16-byte aligned", fn);
  if (!aligned4(g) || !aligned4(beta)) return fail(GDN_ERR_INVALID_ARG, "%s: g and beta must be 4-byte aligned", fn);
  return GDN_OK;
}

// --------------------------------------------------------------- prefill ---
constexpr size_t kSmemLimit = kSmemOptIn;

int simt_slice_rows(int dk, int dv, int C) {
  // widest state slice whose working set fits in shared memory, at most 32 rows
  for (int dvp = dv < 32 ? dv : 32; dvp >= 8; dvp /= 2) {
    if (dv % dvp) continue;
    if ((size_t)gdn::SimtSmem(C, dk, dvp).total * sizeof(float) <= kSmemLimit) return dvp;
  }
  return 0;
}

template <typename TIO>
gdn_status launch_prefill_simt(const void* q, const void* k, const void* v, const float* g,
                               const float* beta, const float* state_in, const int32_t* cu,
                               int n_seqs, int64_t total_T, int Hqk, int Hv, int dk, int dv,
                               float scale, int C, void* o, float* state_out, cudaStream_t st) {
  const int dvp = simt_slice_rows(dk, dv, C);
  if (dvp == 0)
    return fail(GDN_ERR_UNSUPPORTED, "gdn_prefill: dk=%d dv=%d chunk=%d does not fit the SIMT kernel", dk,
                dv, C);
  const size_t smem = (size_t)gdn::SimtSmem(C, dk, dvp).total * sizeof(float);
  auto kern = gdn::prefill_simt_kernel<TIO>;
  if (gdn_status s = allow_smem(kern, "gdn_prefill")) return s;
  dim3 grid((unsigned)(dv / dvp), (unsigned)Hv, (unsigned)n_seqs);
  kern<<<grid, 256, smem, st>>>(static_cast<const TIO*>(q), static_cast<const TIO*>(k),
                                static_cast<const TIO*>(v), g, beta, state_in, cu, Hqk, Hv, dk, dv,
                                dvp, C, scale, static_cast<TIO*>(o), state_out, (long long)total_T);
  return launch_status("gdn_prefill");
}

// ------------------------------------------------- tensor-core prefill ---
// The driver's tensor-map encoder, looked up once per process (thread-safe).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 3-D map of 16-bit elements (bf16 or f16) over a token-major [T][H][D] tensor:
// dims (D, H, T), box (box_d, 1, 64).
bool make_map(CUtensorMap* m, const void* base, int D, int H, int T, int box_d, CUtensorMapDataType type) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
  cuuint32_t box[3] = {(cuuint32_t)box_d, 1, (cuuint32_t)gdn::pc::kC};
  cuuint32_t estr[3] = {1, 1, 1};
  const int row_bytes = box_d * 2;
  CUtensorMapSwizzle sw = row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                          : row_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                            : CU_TENSOR_MAP_SWIZZLE_32B;
  CUresult r = enc(m, type, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

// The prefill kernel's two bounded waits -- on a ring flag in global memory and
// on an mbarrier -- each run on something nothing will ever signal, so that the
// timeout path (error word set, kernel returns) can be exercised without a hung
// or faulted GPU.
__device__ uint32_t g_never_set;
__global__ void wait_selftest_kernel(long long max_cycles) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    gdn::sm100::wait_flag_geq(&g_never_set, 1u, max_cycles);
    gdn::sm100::mbar_init(&bar, 1);
    gdn::sm100::fence_mbar_init();
    gdn::sm100::mbar_wait(&bar, 0, max_cycles);
  }
}

bool uses_pc_prefill(gdn_dtype dtype, int dk, int dv) {
  return (dtype == GDN_BF16 || dtype == GDN_F16) && dk == 128 && dv == 128;
}


template <int DVP, typename T>
gdn_status launch_pc(const CUtensorMap& qm, const CUtensorMap& km, const CUtensorMap& vm, const CUtensorMap& om,
                     const gdn::pc::Params& prm, int grid, cudaStream_t st) {
  auto kern = gdn::pc::prefill_pc_kernel<DVP, T>;
  if (gdn_status s = allow_smem(kern, "gdn_prefill")) return s;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(gdn::pc::kThreads);
  cfg.dynamicSmemBytes = gdn::pc::Smem<DVP>::kAlloc;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;   // every CTA co-resident: CTAs wait on one another
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, qm, km, vm, om, prm);
  if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "gdn_prefill: launch failed: %s", cudaGetErrorString(e));
  return launch_status("gdn_prefill");
}

// Chooses the state slice width DVP and the number of chain CTAs. The kernel
// runs P = NC / slices chains (sequence-heads) at a time, in rounds, and
// prepares packages on the remaining CTAs; its time is about the larger of the
// two sides. Per-chunk costs (SM cycles) measured on B200: a chain step of one
// slice and the preparation of one (head, chunk) item. With several sequences a
// round lasts as long as its longest chain, so P is kept to a multiple or a
// divisor of Hv (whole sequences, or equal parts of one, per round) and a round
// of m sequences is charged the expected longest of m: 2m / (m + 1) times the
// mean length (the lengths are on the device; only their mean is known here).
struct PcPlan {
  int dvp;
  long nc;
};
PcPlan plan_pc(long chains, int64_t total_T, int n_seqs, int Hv, int sms) {
  const double kChainStep[3] = {1950.0, 2300.0, 3100.0};   // DVP 32, 64, 128
  const double kPrepItem = 10500.0;
  const double chunks = std::max(1.0, std::ceil((double)total_T / std::max(1, n_seqs) / 64.0));
  PcPlan best = {128, 1};
  double best_t = 1e300;
  for (int t = 0; t < 3; ++t) {
    const int dvp = 32 << t, slices = 128 / dvp;
    const long p_max = std::min({chains, (long)gdn::pc::kMaxPositions, ((long)sms - 8) / slices});
    for (long pos = 1; pos <= p_max; ++pos) {
      double maxf = 1.0;
      if (n_seqs > 1) {
        if (pos % Hv != 0 && Hv % pos != 0) continue;
        const double m = pos >= Hv ? (double)(pos / Hv) : 1.0;
        maxf = 2.0 * m / (m + 1.0);
      }
      const long nc = pos * slices;
      const double rounds = std::ceil((double)chains / pos);
      const double chain_t = rounds * chunks * maxf * kChainStep[t];
      const double prep_t = chains * chunks * kPrepItem / (double)(sms - nc);
      const double tt = std::max(chain_t, prep_t);
      if (tt < best_t * 0.999) {
        best_t = tt;
        best = {dvp, nc};
      }
    }
  }
  return best;
}

// The plan a launch uses: the model's choice, replaced field by field by the
// caller's request (a field of 0 keeps the model's value), clamped so that no
// position is without a chain, a chain's slices stay in one round and the
// package ring's positions suffice. The request is validated by the caller.
struct PcLaunchPlan {
  int dvp;
  long nc, rounds;
};
bool plan_request_ok(const gdn_plan* req) {
  if (!req) return true;
  return (req->dvp == 0 || req->dvp == 32 || req->dvp == 64 || req->dvp == 128) && req->n_chain_ctas >= 0;
}
PcLaunchPlan resolve_pc(long chains, int64_t total_T, int n_seqs, int Hv, int sms, const gdn_plan* req) {
  PcPlan plan = plan_pc(chains, total_T, n_seqs, Hv, sms);
  if (req && req->dvp != 0 && req->dvp != plan.dvp) {
    // another slice width: keep the model's number of chains per round
    plan.nc = plan.nc / (128 / plan.dvp) * (128 / req->dvp);
    plan.dvp = req->dvp;
  }
  const int dvp = plan.dvp, slices = 128 / dvp;
  long nc = plan.nc;
  if (req && req->n_chain_ctas > 0) nc = std::max(1, std::min(req->n_chain_ctas, sms - 1));
  nc = std::min(nc, (long)sms - 1);
  nc = std::min(nc, chains * slices);
  nc = std::min(nc, (long)gdn::pc::kMaxPositions * slices);
  nc -= nc % slices;
  if (nc < slices) nc = slices;
  return {dvp, nc, (chains * slices + nc - 1) / nc};
}

gdn_status launch_prefill_pc(const void* q, const void* k, const void* v, const float* g, const float* beta,
                             const float* state_in, const int32_t* cu, int n_seqs, int64_t total_T, int Hqk,
                             int Hv, float scale, gdn_dtype dtype, void* o, float* state_out, void* ws,
                             const gdn_plan* req, cudaStream_t st) {
  const long chains = (long)n_seqs * Hv;
  const int sms = sm_count();
  if (sms < 16) return fail(GDN_ERR_CUDA, "gdn_prefill: cannot query the multiprocessor count");
  const PcLaunchPlan lp = resolve_pc(chains, total_T, n_seqs, Hv, sms, req);
  const int dvp = lp.dvp, slices = 128 / dvp;
  const long nc = lp.nc;
  if (lp.rounds > gdn::pc::kMaxRounds)
    return fail(GDN_ERR_UNSUPPORTED, "gdn_prefill: %ld sequence-heads is more than this kernel schedules", chains);
  CUtensorMap qm, km, vm, om;
  const CUtensorMapDataType ty = dtype == GDN_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (!make_map(&qm, q, 128, Hqk, (int)total_T, 64, ty) || !make_map(&km, k, 128, Hqk, (int)total_T, 64, ty) ||
      !make_map(&vm, v, 128, Hv, (int)total_T, std::min(dvp, 64), ty) ||
      !make_map(&om, o, 128, Hv, (int)total_T, std::min(dvp, 64), ty))
    return fail(GDN_ERR_CUDA, "gdn_prefill: cuTensorMapEncodeTiled unavailable or failed");
  cudaError_t e = cudaMemsetAsync(ws, 0, gdn::pc::Workspace::zeroed_bytes(nc / slices), st);
  if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "gdn_prefill: %s", cudaGetErrorString(e));
  gdn::pc::Params prm;
  prm.g = g;
  prm.beta = beta;
  prm.state_in = state_in;
  prm.cu_seqlens = cu;
  prm.o = o;
  prm.state_out = state_out;
  prm.ws = static_cast<uint8_t*>(ws);
  prm.n_seqs = n_seqs;
  prm.Hqk = Hqk;
  prm.Hv = Hv;
  prm.total_T = (int)total_T;
  prm.scale = scale;
  prm.n_chain_ctas = (int)nc;
  if (dtype == GDN_F16) {
    if (dvp == 32) return launch_pc<32, __half>(qm, km, vm, om, prm, sms, st);
    if (dvp == 64) return launch_pc<64, __half>(qm, km, vm, om, prm, sms, st);
    return launch_pc<128, __half>(qm, km, vm, om, prm, sms, st);
  }
  if (dvp == 32) return launch_pc<32, __nv_bfloat16>(qm, km, vm, om, prm, sms, st);
  if (dvp == 64) return launch_pc<64, __nv_bfloat16>(qm, km, vm, om, prm, sms, st);
  return launch_pc<128, __nv_bfloat16>(qm, km, vm, om, prm, sms, st);
}

}  // namespace

extern "C" {

int gdn_version(void) { return (0 << 16) | 4; }

const char* gdn_last_error(void) { return t_last_error.c_str(); }

size_t gdn_prefill_workspace_bytes(int n_seqs, int Hv, int dk, int dv, gdn_dtype dtype) {
  if (n_seqs <= 0 || Hv <= 0 || !uses_pc_prefill(dtype, dk, dv)) return 0;
  return gdn::pc::Workspace::bytes(std::min((long)n_seqs * Hv, (long)gdn::pc::kMaxPositions));
}

gdn_status gdn_prefill_plan(int n_seqs, int64_t total_T, int Hv, int dk, int dv, gdn_dtype dtype, int sm_count_arg,
                            const gdn_plan* requested, int* dvp, int* n_chain_ctas, int* rounds) {
  t_last_error.clear();
  if (!dvp || !n_chain_ctas || !rounds) return fail(GDN_ERR_INVALID_ARG, "gdn_prefill_plan: null output");
  if (!plan_request_ok(requested))
    return fail(GDN_ERR_INVALID_ARG, "gdn_prefill_plan: requested dvp %d (0, 32, 64 or 128), n_chain_ctas %d (>= 0)",
                requested->dvp, requested->n_chain_ctas);
  if (n_seqs <= 0 || Hv <= 0 || total_T < 0)
    return fail(GDN_ERR_INVALID_ARG, "gdn_prefill_plan: n_seqs %d, Hv %d, total_T %lld", n_seqs, Hv,
                (long long)total_T);
  if (!uses_pc_prefill(dtype, dk, dv))
    return fail(GDN_ERR_UNSUPPORTED, "gdn_prefill_plan: the tensor-core kernel takes bf16 or f16 with dk = dv = 128");
  const int sms = sm_count_arg > 0 ? sm_count_arg : sm_count();
  if (sms < 16) return fail(GDN_ERR_INVALID_ARG, "gdn_prefill_plan: %d multiprocessors", sms);
  const PcLaunchPlan lp = resolve_pc((long)n_seqs * Hv, total_T, n_seqs, Hv, sms, requested);
  *dvp = lp.dvp;
  *n_chain_ctas = (int)lp.nc;
  *rounds = (int)std::min(lp.rounds, (long)INT32_MAX);
  return GDN_OK;
}

gdn_status gdn_prefill_ex(const void* q, const void* k, const void* v, const float* g,
                          const float* beta, const float* state_in, const int32_t* cu_seqlens,
                          int n_seqs, int64_t total_T, int Hqk, int Hv, int dk, int dv, float scale,
                          int chunk, gdn_dtype dtype, void* o, float* state_out, void* workspace,
                          size_t workspace_bytes, const gdn_plan* plan, void* stream) {
  if (!plan_request_ok(plan))
    return fail(GDN_ERR_INVALID_ARG, "gdn_prefill: plan dvp %d (0, 32, 64 or 128), n_chain_ctas %d (>= 0)",
                plan->dvp, plan->n_chain_ctas);
  if (n_seqs < 0) return fail(GDN_ERR_INVALID_ARG, "gdn_prefill: n_seqs=%d < 0", n_seqs);
  if (total_T < 0 || total_T >= (int64_t(1) << 31))
    return fail(GDN_ERR_INVALID_ARG, "gdn_prefill: total_T=%lld out of range", (long long)total_T);
  if (Hqk <= 0 || Hv <= 0 || Hv % Hqk != 0)
    return fail(GDN_ERR_INVALID_ARG, "gdn_prefill: Hv=%d must be a positive multiple of Hqk=%d", Hv, Hqk);
  if (!head_dim_ok(dk) || !head_dim_ok(dv))
    return fail(GDN_ERR_UNSUPPORTED, "gdn_prefill: dk=%d, dv=%d (supported: 16, 32, 64, 128)", dk, dv);
  if (!dtype_ok(dtype)) return fail(GDN_ERR_INVALID_ARG, "gdn_prefill: unknown dtype %d", (int)dtype);
  if (n_seqs == 0) return ok();
  if (!cu_seqlens || !state_out)
    return fail(GDN_ERR_INVALID_ARG, "gdn_prefill: cu_seqlens and state_out must not be NULL");
  if (total_T > 0 && (!q || !k || !v || !g || !beta || !o))
    return fail(GDN_ERR_INVALID_ARG, "gdn_prefill: q, k, v, g, beta and o must not be NULL");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(state_out) ||
      !aligned16(state_in))
    return fail(GDN_ERR_INVALID_ARG, "gdn_prefill: q, k, v, o and the states must be 16-byte aligned");
  if (!aligned4(g) || !aligned4(beta) || !aligned4(cu_seqlens))
    return fail(GDN_ERR_INVALID_ARG, "gdn_prefill: g, beta and cu_seqlens must be 4-byte aligned");
  if (scale <= 0.f) scale = 1.0f / sqrtf((float)dk);
  int C = chunk;
  if (C == 0) C = uses_pc_prefill(dtype, dk, dv) ? 64 : 16;
  if (C != 16 && C != 32 && C != 64)
    return fail(GDN_ERR_UNSUPPORTED, "gdn_prefill: chunk=%d (supported: 16, 32, 64)", C);
  const size_t need = gdn_prefill_workspace_bytes(n_seqs, Hv, dk, dv, dtype);
  if (need > 0 && (!workspace || workspace_bytes < need || !aligned16(workspace)))
    return fail(GDN_ERR_INVALID_ARG, "gdn_prefill: workspace needs %zu bytes (16-byte aligned), got %zu",
                need, workspace_bytes);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (uses_pc_prefill(dtype, dk, dv) && C == 64 && total_T > 0)
    return launch_prefill_pc(q, k, v, g, beta, state_in, cu_seqlens, n_seqs, total_T, Hqk, Hv, scale, dtype, o,
                             state_out, workspace, plan, st);
  if (dtype == GDN_F32)
    return launch_prefill_simt<float>(q, k, v, g, beta, state_in, cu_seqlens, n_seqs, total_T, Hqk,
                                      Hv, dk, dv, scale, C, o, state_out, st);
  if (dtype == GDN_F16)
    return launch_prefill_simt<__half>(q, k, v, g, beta, state_in, cu_seqlens, n_seqs, total_T, Hqk,
                                       Hv, dk, dv, scale, C, o, state_out, st);
  return launch_prefill_simt<__nv_bfloat16>(q, k, v, g, beta, state_in, cu_seqlens, n_seqs, total_T,
                                            Hqk, Hv, dk, dv, scale, C, o, state_out, st);
}

gdn_status gdn_prefill(const void* q, const void* k, const void* v, const float* g,
                       const float* beta, const float* state_in, const int32_t* cu_seqlens,
                       int n_seqs, int64_t total_T, int Hqk, int Hv, int dk, int dv, float scale,
                       int chunk, gdn_dtype dtype, void* o, float* state_out, void* workspace,
                       size_t workspace_bytes, void* stream) {
  return gdn_prefill_ex(q, k, v, g, beta, state_in, cu_seqlens, n_seqs, total_T, Hqk, Hv, dk, dv, scale, chunk,
                        dtype, o, state_out, workspace, workspace_bytes, nullptr, stream);
}

gdn_status gdn_decode(const void* q, const void* k, const void* v, const float* g,
                      const float* beta, float* state, int B, int Hqk, int Hv, int dk, int dv,
                      float scale, gdn_dtype dtype, void* o, void* stream) {
  bool done = false;
  if (gdn_status s = check_decode("gdn_decode", q, k, v, g, beta, state, B, Hqk, Hv, dk, dv, dtype, o, &done))
    return s;
  if (done) return ok();
  if (scale <= 0.f) scale = 1.0f / sqrtf((float)dk);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == GDN_F32)
    return dispatch_decode<float, float>(q, k, v, g, beta, state, B, Hqk, Hv, dk, dv, scale, o, st);
  if (dtype == GDN_F16)
    return dispatch_decode<__half, float>(q, k, v, g, beta, state, B, Hqk, Hv, dk, dv, scale, o, st);
  return dispatch_decode<__nv_bfloat16, float>(q, k, v, g, beta, state, B, Hqk, Hv, dk, dv, scale, o, st);
}

gdn_status gdn_decode_bf16_state(const void* q, const void* k, const void* v, const float* g,
                                 const float* beta, void* state, int B, int Hqk, int Hv, int dk, int dv,
                                 float scale, gdn_dtype dtype, void* o, void* stream) {
  bool done = false;
  if (gdn_status s =
          check_decode("gdn_decode_bf16_state", q, k, v, g, beta, state, B, Hqk, Hv, dk, dv, dtype, o, &done))
    return s;
  if (done) return ok();
  if (scale <= 0.f) scale = 1.0f / sqrtf((float)dk);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  auto* s16 = static_cast<__nv_bfloat16*>(state);
  if (dtype == GDN_F32)
    return dispatch_decode<float, __nv_bfloat16>(q, k, v, g, beta, s16, B, Hqk, Hv, dk, dv, scale, o, st);
  if (dtype == GDN_F16)
    return dispatch_decode<__half, __nv_bfloat16>(q, k, v, g, beta, s16, B, Hqk, Hv, dk, dv, scale, o, st);
  return dispatch_decode<__nv_bfloat16, __nv_bfloat16>(q, k, v, g, beta, s16, B, Hqk, Hv, dk, dv, scale, o, st);
}

gdn_status gdn_wait_selftest(int max_wait_us, void* stream) {
  if (max_wait_us < 1 || max_wait_us > 1000000)
    return fail(GDN_ERR_INVALID_ARG, "gdn_wait_selftest: max_wait_us=%d outside [1, 1000000]", max_wait_us);
  const long long cycles = (long long)max_wait_us * 2000;   // ~2 GHz SM clock
  wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(cycles);
  return launch_status("gdn_wait_selftest");
}

gdn_status gdn_device_error(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned int word = 0;
  cudaError_t e = cudaMemcpyFromSymbolAsync(&word, gdn::g_error_word, sizeof word, 0,
                                            cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "gdn_device_error: %s", cudaGetErrorString(e));
  if (word) {
    unsigned int line = 0;
    e = cudaMemcpyFromSymbolAsync(&line, gdn::g_error_line, sizeof line, 0, cudaMemcpyDeviceToHost, st);
    const unsigned int zero = 0;
    if (e == cudaSuccess)
      e = cudaMemcpyToSymbolAsync(gdn::g_error_word, &zero, sizeof zero, 0, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess)
      e = cudaMemcpyToSymbolAsync(gdn::g_error_line, &zero, sizeof zero, 0, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "gdn_device_error: %s", cudaGetErrorString(e));
    if (word & gdn::kErrCheck)
      return fail(GDN_ERR_DEVICE_CHECK, "an index check of the GDN_DEBUG build failed (source line %u, error word 0x%x)",
                  line, word);
    return fail(GDN_ERR_DEVICE_TIMEOUT, "a bounded device wait ran out (error word 0x%x)", word);
  }
  return ok();
}

int gdn_debug_checks(void) {
#ifdef GDN_DEBUG
  return 1;
#else
  return 0;
#endif
}

}  // extern "C"

// ============================================================================
// Allocation-free prefill.
//
// Some callers cannot hand the library any device memory of its own making:
// code that runs where cudaMalloc is not allowed or not wanted -- inside a
// region whose memory was planned ahead of time by an inference runtime, a
// plugin whose host framework owns every allocation, or a real-time loop where
// an allocator call could stall or fail. gdn_prefill needs a workspace (the
// package ring the preparation and chain CTAs exchange data through), so for
// those callers this file keeps one statically sized scratch array in device
// memory and gdn_prefill_noalloc runs the same kernel on it.
//
// The array lives as long as the library is loaded, on every device that
// loads it. Host code must never use the array's name as a device pointer:
// its device address is looked up with cudaGetSymbolAddress, with the device
// current. The address belongs to the CUDA context the module was loaded in,
// so it is cached per device together with that context's id and looked up
// again on every call made outside stream capture (a cheap host-side query);
// a call under capture uses the cached address, which must come from an
// earlier call in the same context. Every call shares the array: the parts
// that must start at zero are cleared by each call on its stream, and two
// calls whose kernels overlap on the GPU (different streams, or different
// host threads) race on it and must be serialised by the caller.
// ============================================================================
namespace {

// The largest workspace gdn_prefill can ask for (the ring of kMaxPositions
// positions), rounded up to whole MiB: every problem gdn_prefill runs fits.
constexpr size_t kNoAllocScratchBytes =
    (gdn::pc::Workspace::bytes(gdn::pc::kMaxPositions) + (size_t(1) << 20) - 1) & ~((size_t(1) << 20) - 1);
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
struct NoAllocAddr {
  unsigned long long ctx_id;   // the context the address was looked up in
  void* ptr;
};
std::mutex g_noalloc_mu;
NoAllocAddr g_noalloc_addr[kMaxDevices] = {};

// Id of the calling thread's current CUDA context (driver entry points looked
// up once); false if there is none or the driver lacks the query.
bool current_context_id(unsigned long long* id) {
  static std::once_flag once;
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  if (!get_current || !get_id) return false;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

gdn_status noalloc_scratch(cudaStream_t st, void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "gdn_prefill_noalloc: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices)
    return fail(GDN_ERR_UNSUPPORTED, "gdn_prefill_noalloc: device %d beyond %d", dev, kMaxDevices);
  // (a runtime call on the stream also makes the device's context current)
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  e = cudaStreamIsCapturing(st, &cap);
  if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "gdn_prefill_noalloc: %s", cudaGetErrorString(e));
  unsigned long long ctx = 0;
  if (!current_context_id(&ctx))
    return fail(GDN_ERR_CUDA, "gdn_prefill_noalloc: cannot identify the current CUDA context");
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  NoAllocAddr& a = g_noalloc_addr[dev];
  if (cap == cudaStreamCaptureStatusNone) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess || !ptr)
      return fail(GDN_ERR_CUDA, "gdn_prefill_noalloc: cudaGetSymbolAddress failed: %s", cudaGetErrorString(e));
    a = {ctx, ptr};
  } else if (!a.ptr || a.ctx_id != ctx) {
    return fail(GDN_ERR_CUDA,
                "gdn_prefill_noalloc: called under stream capture before any call outside capture in this "
                "CUDA context (the scratch address is looked up outside capture)");
  }
  *out = a.ptr;
  return GDN_OK;
}

}  // namespace

extern "C" gdn_status gdn_prefill_noalloc(const void* q, const void* k, const void* v, const float* g,
                                          const float* beta, const float* state_in,
                                          const int32_t* cu_seqlens, int n_seqs, int64_t total_T, int Hqk,
                                          int Hv, int dk, int dv, float scale, int chunk, gdn_dtype dtype,
                                          void* o, float* state_out, void* stream) {
  if (dtype != GDN_BF16 || dk != 128 || dv != 128 || (chunk != 0 && chunk != 64))
    return fail(GDN_ERR_UNSUPPORTED,
                "gdn_prefill_noalloc: only bf16 with dk = dv = 128 and chunk 64 (the tensor-core kernel)");
  if (n_seqs > 0 && Hv > 0) {
    const size_t need = gdn_prefill_workspace_bytes(n_seqs, Hv, dk, dv, dtype);
    if (need > kNoAllocScratchBytes)
      return fail(GDN_ERR_UNSUPPORTED,
                  "gdn_prefill_noalloc: %d sequences x %d heads need %zu bytes of scratch, more than the %zu "
                  "bytes built into the library; use gdn_prefill with a workspace",
                  n_seqs, Hv, need, kNoAllocScratchBytes);
  }
  void* scratch = nullptr;
  if (gdn_status s = noalloc_scratch(static_cast<cudaStream_t>(stream), &scratch)) return s;
  return gdn_prefill(q, k, v, g, beta, state_in, cu_seqlens, n_seqs, total_T, Hqk, Hv, dk, dv, scale, chunk,
                     dtype, o, state_out, scratch, kNoAllocScratchBytes, stream);
}
