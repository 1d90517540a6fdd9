// Thin wrappers over the sm_100a PTX this library uses: mbarriers, TMA
// tensor loads, and the 5th-generation tensor core (tcgen05: TMEM
// allocation, MMA issue/commit, TMEM loads, ordering fences).
//
// Shared-memory matrix descriptors follow the sm_100 UMMA format: start
// address >> 4 in bits [0,14), leading byte offset >> 4 in [16,30), stride
// byte offset >> 4 in [32,46), descriptor version 1 at bit 46, swizzle mode
// in [61,64) (2 = 128-byte, 4 = 64-byte, 6 = 32-byte). Canonical layouts
// (bytes; a "row" is one 16/32/64/128-byte swizzle row):
//   K-major, 128B swizzle : rows of 64 16-bit values along K, 8-row groups 1024 B apart
//                           (stride offset), 16-byte chunk index XOR (row & 7).
//   MN-major, S-byte swizzle: rows of S/2 16-bit values along M/N, one row per K index,
//                           8 K-rows per group (stride offset = 8 * S), further
//                           blocks of S/2 M/N elements at the leading offset.
// Every swizzled tile starts on a 1024-byte boundary.
#pragma once

#include <cuda.h>
#include <stdint.h>

#include "common.cuh"

namespace gdn {
namespace sm100 {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ------------------------------------------------------------ mbarriers ---
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// Non-blocking test of a phase (try_wait may suspend the thread for a while).
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// Waits at most about `max_cycles` SM clocks for the barrier phase with the
// given parity to complete. On timeout it records kErrTimeout in the device
// error word and returns false instead of spinning forever.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity,
                                          long long max_cycles = 4000000000ll) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > max_cycles) {
      flag_error(kErrTimeout);
      return false;
    }
  }
  return true;
}

// ------------------------------------------------------ named barriers ---
// Barrier `id` (1..15) over the first `n` threads of the CTA (n a multiple of 32).
__device__ __forceinline__ void named_bar_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
// Arrives on barrier `id` (counted among its `n` threads) without waiting.
__device__ __forceinline__ void named_bar_arrive(int id, int n) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(n) : "memory");
}
// As named_bar_sync, and returns whether `p` holds on every participating thread.
__device__ __forceinline__ bool named_bar_and(int id, int n, bool p) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred a, b;\n\t"
      "setp.ne.u32 a, %1, 0;\n\t"
      "bar.red.and.pred b, %2, %3, a;\n\t"
      "selp.u32 %0, 1, 0, b;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(p)), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

// ----------------------------------------------------------------- TMA ---
// 3-D tiled bulk tensor load global -> shared, completion counted in bytes
// on `bar`. Coordinates are element offsets, innermost first.
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int x,
                                            int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}
// Prefetch of a 3-D tile into L2 (nothing is written to shared memory and no
// completion is signalled): a later load of the same box finds it in L2.
__device__ __forceinline__ void tma_prefetch_3d(const CUtensorMap* map, int x, int y, int z) {
  asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y), "r"(z)
               : "memory");
}
__device__ __forceinline__ void prefetch_l2(const void* ptr) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<uint64_t>(ptr)) : "memory");
}
// 3-D tiled bulk tensor store shared -> global (coordinates must not be
// negative), in the thread's bulk async-group; commit and wait with the
// helpers below, from the same thread.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int x, int y, int z) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z)
               : "memory");
}
// 1-D bulk copy shared -> global (16-byte aligned addresses, size a multiple of
// 16), in the thread's bulk async-group.
__device__ __forceinline__ void bulk_store(void* dst, const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(reinterpret_cast<uint64_t>(dst)),
               "r"(smem_u32(src)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Waits until the shared memory read by this thread's committed bulk stores may be reused.
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// Waits until this thread's committed bulk stores are complete.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 1-D bulk copy global -> shared (16-byte aligned addresses, size a multiple
// of 16), completion counted in bytes on `bar`; warp-collective, one lane issues.
__device__ __forceinline__ void bulk_load_warp(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n\t}" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// ---------------------------------------------------- cross-CTA flags ---
__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
// Relaxed load: does not order the thread's later memory operations, so it does
// not stall the thread until its value is used. Pair with fence_acq_rel_gpu()
// once the value has been seen, to acquire what it publishes.
__device__ __forceinline__ uint32_t ld_relaxed_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void fence_acq_rel_gpu() {
  asm volatile("fence.acq_rel.gpu;" ::: "memory");
}
__device__ __forceinline__ void st_release_gpu(uint32_t* p, uint32_t v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void red_add_release_gpu(uint32_t* p, uint32_t v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// Waits (at most about max_cycles SM clocks) until *p >= target; records
// kErrTimeout and returns false instead of spinning forever.
__device__ __forceinline__ bool wait_flag_geq(const uint32_t* p, uint32_t target,
                                              long long max_cycles = 4000000000ll) {
  if (ld_acquire_gpu(p) >= target) return true;
  const long long t0 = clock64();
  while (ld_acquire_gpu(p) < target) {
    if (clock64() - t0 > max_cycles) {
      flag_error(kErrTimeout);
      return false;
    }
    __nanosleep(64);
  }
  return true;
}
// Global writes made visible to the generic proxy of other CTAs, read next by this
// thread's async proxy (bulk copies): order the two proxies.
__device__ __forceinline__ void fence_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Generic-proxy shared-memory writes -> visible to the async proxy (TMA, tcgen05.mma).
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------- tcgen05 ---
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem], kind::f16: 16-bit inputs (both f16 or both bf16,
// as the instruction descriptor says), fp32 accumulate; one K=16 step.
__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Warp-collective variants: every lane of the warp executes the call with the
// same (warp-uniform) operands and one elected lane issues. Keeping the whole
// warp on the issue path lets the operands stay in uniform registers; issuing
// from a single divergent thread costs tens to hundreds of cycles per
// instruction. The elected lane is the lowest active one, so a commit made
// the same way tracks the MMAs issued by the same lane.
__device__ __forceinline__ void mma_f16_warp(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                              uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred e, p;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem] (kind::f16): A read from TMEM, its M rows in
// lanes 0-127 and one K=16 step in 8 columns from a_tmem. Warp-collective.
__device__ __forceinline__ void mma_f16_tmem_a_warp(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                                    uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred e, p;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Copy 128 rows x 32 bytes of a shared-memory matrix into TMEM lanes 0-127, 8
// columns from taddr (tcgen05.cp .128x256b). With the descriptor of one K-step
// of a K-major 16-bit operand it stages that step as an A operand for
// mma_f16_tmem_a_warp; a later tcgen05.mma of the same thread is ordered after
// it. Warp-collective (one elected lane issues).
__device__ __forceinline__ void tmem_cp_128x256b_warp(uint32_t taddr, uint64_t sdesc) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.cp.cta_group::1.128x256b [%0], %1;\n\t}" ::"r"(taddr),
      "l"(sdesc)
      : "memory");
}
__device__ __forceinline__ void mma_commit_warp(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(
          smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx_warp(uint64_t* bar, uint32_t bytes) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n\t}" ::"r"(smem_u32(bar)),
      "r"(bytes)
      : "memory");
}
// Adds `bytes` to the barrier's expected transaction count without arriving
// (warp-collective, one lane issues): copies may be started before the data
// they travel with is written, and the arrival made afterwards.
__device__ __forceinline__ void mbar_expect_tx_warp(uint64_t* bar, uint32_t bytes) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;\n\t}" ::"r"(smem_u32(bar)),
      "r"(bytes)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d_warp(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y,
                                                 int z) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];\n\t}" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// An L2 policy for data that is touched exactly once (a tile read or written by
// its only reader or writer): lines brought in under it are the first that L2
// evicts, so that data read again (and the kernel's code) stays resident.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
// tma_load_3d_warp under an L2 cache policy.
__device__ __forceinline__ void tma_load_3d_warp_hint(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y,
                                                      int z, uint64_t pol) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4, %5}], [%2], %6;\n\t}" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z), "l"(pol)
      : "memory");
}
// tma_store_3d under an L2 cache policy.
__device__ __forceinline__ void tma_store_3d_hint(const CUtensorMap* map, const void* src, int x, int y, int z,
                                                  uint64_t pol) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group.L2::cache_hint [%0, {%2, %3, %4}], [%1], %5;" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z), "l"(pol)
               : "memory");
}

// Arrive once on `bar` when every tcgen05.mma issued so far by this thread completes.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// Instruction descriptor, kind::f16 with fp32 D and A, B both of the 16-bit
// type whose format code is `ab_fmt` (0 = f16, 1 = bf16; one MMA never mixes
// the two).
__host__ __device__ constexpr uint32_t idesc_f16kind(int M, int N, bool a_mn_major, bool b_mn_major,
                                                     uint32_t ab_fmt) {
  return (1u << 4)                                   // D format f32
         | (ab_fmt << 7)                             // A format
         | (ab_fmt << 10)                            // B format
         | (static_cast<uint32_t>(a_mn_major) << 15) //
         | (static_cast<uint32_t>(b_mn_major) << 16) //
         | (static_cast<uint32_t>(N >> 3) << 17)     //
         | (static_cast<uint32_t>(M >> 4) << 24);
}


enum : uint32_t { kSwizzle128 = 2, kSwizzle64 = 4, kSwizzle32 = 6 };

__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes,
                                              uint32_t swizzle) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) |
         (static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32) | (1ull << 46) |
         (static_cast<uint64_t>(swizzle) << 61);
}

// Descriptor for K-step `kk` (16 elements) of a K-major 128B-swizzled operand whose
// 64-element atom columns are `acs` bytes apart.
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t base, int kk, uint32_t acs) {
  return smem_desc(base + (kk >> 2) * acs + (kk & 3) * 32, 16, 1024, kSwizzle128);
}
// Descriptor for K-step `kk` of an MN-major operand: K-rows of `row_bytes`
// (32/64/128), further blocks of row_bytes/2 elements `lbo` bytes apart.
__device__ __forceinline__ uint64_t desc_mnmajor(uint32_t base, int kk, uint32_t row_bytes, uint32_t lbo) {
  const uint32_t sw = row_bytes == 128 ? kSwizzle128 : row_bytes == 64 ? kSwizzle64 : kSwizzle32;
  return smem_desc(base + kk * 16 * row_bytes, lbo, 8 * row_bytes, sw);
}

// Byte offset of K-step kk (16 elements) within a K-major 128B-swizzled
// operand whose 64-element atom columns are `acs` bytes apart, and within an
// MN-major operand with K-rows of `row_bytes`.
__host__ __device__ constexpr uint32_t kmajor_step(int kk, uint32_t acs) {
  return static_cast<uint32_t>(kk >> 2) * acs + static_cast<uint32_t>(kk & 3) * 32u;
}
__host__ __device__ constexpr uint32_t mnmajor_step(int kk, uint32_t row_bytes) {
  return static_cast<uint32_t>(kk) * 16u * row_bytes;
}
// A descriptor with its start address moved on by `bytes` (a multiple of 16).
// The 14-bit address field cannot carry into the next one: shared-memory
// addresses stay below 256 KB.
__device__ __forceinline__ uint64_t desc_advance(uint64_t d, uint32_t bytes) { return d + (bytes >> 4); }

// NK K-steps of D (+)= A B (kind::f16), issued by the whole warp (one elected
// lane), from descriptors a0, b0 of K-step 0 built once: each later step only
// advances their start addresses by constants. A_KM / B_KM say whether the
// operand is K-major (then A_P / B_P is its atom column spacing) or MN-major
// (then the byte length of its K-rows). acc: accumulate onto D from the first
// step on (else the first step overwrites D).
template <int NK, bool A_KM, uint32_t A_P, bool B_KM, uint32_t B_P>
__device__ __forceinline__ void mma_k(uint32_t d_tmem, uint64_t a0, uint64_t b0, uint32_t idesc, bool acc) {
#pragma unroll
  for (int kk = 0; kk < NK; ++kk) {
    const uint32_t ao = A_KM ? kmajor_step(kk, A_P) : mnmajor_step(kk, A_P);
    const uint32_t bo = B_KM ? kmajor_step(kk, B_P) : mnmajor_step(kk, B_P);
    mma_f16_warp(d_tmem, desc_advance(a0, ao), desc_advance(b0, bo), idesc, (acc || kk > 0) ? 1u : 0u);
  }
}

// The same as mma_k for NK = 4 or 8 steps whose descriptors advance by the same
// ASTEP / BSTEP 16-byte units every step, from one asm block: one elect.sync and
// the steps' address arithmetic as immediates, so that the elected lane issues the
// whole group back to back. acc as in mma_k (the first step; the others accumulate).
#define GDN_MMA_NEXT                                                       \
  "add.s64 a, a, %5;\n\t"                                                  \
  "add.s64 b, b, %6;\n\t"                                                  \
  "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, t;\n\t"
#define GDN_MMA_HEAD                                                       \
  "{\n\t.reg .pred e, p, t;\n\t.reg .b64 a, b;\n\t"                        \
  "setp.ne.b32 p, %4, 0;\n\t"                                              \
  "setp.eq.b32 t, %4, %4;\n\t"                                             \
  "mov.b64 a, %1;\n\t"                                                     \
  "mov.b64 b, %2;\n\t"                                                     \
  "elect.sync _|e, 0xffffffff;\n\t"                                        \
  "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, p;\n\t"
template <int NK, uint32_t ASTEP, uint32_t BSTEP>
__device__ __forceinline__ void mma_run_warp(uint32_t d_tmem, uint64_t a0, uint64_t b0, uint32_t idesc, uint32_t acc) {
  static_assert(NK == 4 || NK == 8, "4 or 8 steps");
  if constexpr (NK == 4) {
    asm volatile(GDN_MMA_HEAD GDN_MMA_NEXT GDN_MMA_NEXT GDN_MMA_NEXT "}" ::"r"(d_tmem), "l"(a0), "l"(b0),
                 "r"(idesc), "r"(acc), "n"(ASTEP), "n"(BSTEP)
                 : "memory");
  } else {
    asm volatile(GDN_MMA_HEAD GDN_MMA_NEXT GDN_MMA_NEXT GDN_MMA_NEXT GDN_MMA_NEXT GDN_MMA_NEXT GDN_MMA_NEXT
                     GDN_MMA_NEXT "}" ::"r"(d_tmem),
                 "l"(a0), "l"(b0), "r"(idesc), "r"(acc), "n"(ASTEP), "n"(BSTEP)
                 : "memory");
  }
}
#undef GDN_MMA_HEAD
#undef GDN_MMA_NEXT
// Eight accumulating K-steps with A in TMEM (8 columns a step from a_tmem) and B
// advancing BSTEP 16-byte units a step, from one asm block (as mma_run_warp).
#define GDN_MMA_TA_NEXT                                                    \
  "add.u32 a, a, 8;\n\t"                                                   \
  "add.s64 b, b, %4;\n\t"                                                  \
  "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %3, t;\n\t"
template <uint32_t BSTEP>
__device__ __forceinline__ void mma8_tmem_a_run_warp(uint32_t d_tmem, uint32_t a_tmem, uint64_t b0, uint32_t idesc) {
  asm volatile(
      "{\n\t.reg .pred e, t;\n\t.reg .b64 b;\n\t.reg .b32 a;\n\t"
      "setp.eq.b32 t, %3, %3;\n\t"
      "mov.b32 a, %1;\n\t"
      "mov.b64 b, %2;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %3, t;\n\t" GDN_MMA_TA_NEXT GDN_MMA_TA_NEXT GDN_MMA_TA_NEXT
          GDN_MMA_TA_NEXT GDN_MMA_TA_NEXT GDN_MMA_TA_NEXT GDN_MMA_TA_NEXT "}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b0), "r"(idesc), "n"(BSTEP)
      : "memory");
}
#undef GDN_MMA_TA_NEXT

// Byte offset of element (row, col) in a K-major 128B-swizzled operand
// (64-element atom columns `acs` bytes apart). col % 8 == 0 addresses a chunk.
__device__ __forceinline__ uint32_t sw128_off(int row, int col, uint32_t acs) {
  return (col >> 6) * acs + (row >> 3) * 1024 + (row & 7) * 128 +
         ((((col & 63) >> 3) ^ (row & 7)) << 4) + ((col & 7) << 1);
}

// Byte offset of element (row, col) of an MN-major tile whose rows are R
// bytes (32, 64 or 128) with the matching swizzle: 16-byte chunk bits [4,7)
// XOR address bits [7,10) (as many bits as the row has chunks).
template <uint32_t R>
__device__ __forceinline__ uint32_t mn_off(int row, int col) {
  static_assert(R == 32 || R == 64 || R == 128, "row bytes");
  constexpr uint32_t mask = R == 128 ? 7u : R == 64 ? 3u : 1u;
  const uint32_t o = static_cast<uint32_t>(row) * R + static_cast<uint32_t>(col) * 2u;
  return o ^ (((o >> 7) & mask) << 4);
}

// ------------------------------------------------------------ TMEM loads ---
// 32 lanes x 8 / 16 / 32 consecutive 32-bit columns, waited for before returning.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float* r) {
  uint32_t u[8];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 8; ++i) r[i] = __uint_as_float(u[i]);
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* r) {
  uint32_t u[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7]),
        "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]), "=r"(u[14]),
        "=r"(u[15])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) r[i] = __uint_as_float(u[i]);
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* r) {
  uint32_t u[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7]),
        "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]), "=r"(u[14]),
        "=r"(u[15]), "=r"(u[16]), "=r"(u[17]), "=r"(u[18]), "=r"(u[19]), "=r"(u[20]), "=r"(u[21]),
        "=r"(u[22]), "=r"(u[23]), "=r"(u[24]), "=r"(u[25]), "=r"(u[26]), "=r"(u[27]), "=r"(u[28]),
        "=r"(u[29]), "=r"(u[30]), "=r"(u[31])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) r[i] = __uint_as_float(u[i]);
}

// Load N (8, 16, 32 or a multiple of 32) consecutive columns.
// 32 lanes x 64 consecutive columns in one load.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float* r) {
  uint32_t u[64];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,"
      "%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
      "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7]),
        "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]), "=r"(u[14]), "=r"(u[15]),
        "=r"(u[16]), "=r"(u[17]), "=r"(u[18]), "=r"(u[19]), "=r"(u[20]), "=r"(u[21]), "=r"(u[22]), "=r"(u[23]),
        "=r"(u[24]), "=r"(u[25]), "=r"(u[26]), "=r"(u[27]), "=r"(u[28]), "=r"(u[29]), "=r"(u[30]), "=r"(u[31]),
        "=r"(u[32]), "=r"(u[33]), "=r"(u[34]), "=r"(u[35]), "=r"(u[36]), "=r"(u[37]), "=r"(u[38]), "=r"(u[39]),
        "=r"(u[40]), "=r"(u[41]), "=r"(u[42]), "=r"(u[43]), "=r"(u[44]), "=r"(u[45]), "=r"(u[46]), "=r"(u[47]),
        "=r"(u[48]), "=r"(u[49]), "=r"(u[50]), "=r"(u[51]), "=r"(u[52]), "=r"(u[53]), "=r"(u[54]), "=r"(u[55]),
        "=r"(u[56]), "=r"(u[57]), "=r"(u[58]), "=r"(u[59]), "=r"(u[60]), "=r"(u[61]), "=r"(u[62]), "=r"(u[63])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 64; ++i) r[i] = __uint_as_float(u[i]);
}

template <int N>
__device__ __forceinline__ void tmem_ld(uint32_t taddr, float* r) {
  if constexpr (N == 8) {
    tmem_ld8(taddr, r);
  } else if constexpr (N == 16) {
    tmem_ld16(taddr, r);
  } else if constexpr (N == 32) {
    tmem_ld32(taddr, r);
  } else {
    static_assert(N % 64 == 0, "columns");
#pragma unroll
    for (int c = 0; c < N / 64; ++c) tmem_ld64(taddr + 64 * c, r + 64 * c);
  }
}

// The 16-bit tensor-core operand types (kind::f16): format code, packing of 8
// floats into one 16-byte chunk (round to nearest even) and unpacking.
template <typename T> struct Op16;
template <> struct Op16<__nv_bfloat16> {
  static constexpr uint32_t kFmt = 1u;
  static __device__ __forceinline__ uint32_t pack2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
  }
  static __device__ __forceinline__ float2 unpack2(uint32_t u) {
    return __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&u));
  }
  static __device__ __forceinline__ unsigned short one(float x) {
    __nv_bfloat16 h = __float2bfloat16_rn(x);
    return *reinterpret_cast<unsigned short*>(&h);
  }
};
template <> struct Op16<__half> {
  static constexpr uint32_t kFmt = 0u;
  static __device__ __forceinline__ uint32_t pack2(float a, float b) {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
  }
  static __device__ __forceinline__ float2 unpack2(uint32_t u) {
    return __half22float2(*reinterpret_cast<__half2*>(&u));
  }
  static __device__ __forceinline__ unsigned short one(float x) {
    __half h = __float2half_rn(x);
    return *reinterpret_cast<unsigned short*>(&h);
  }
};
template <typename T>
__device__ __forceinline__ uint4 pack8(const float* x) {
  return make_uint4(Op16<T>::pack2(x[0], x[1]), Op16<T>::pack2(x[2], x[3]), Op16<T>::pack2(x[4], x[5]),
                    Op16<T>::pack2(x[6], x[7]));
}
// The 8 values of a 16-byte chunk of T as floats.
template <typename T>
__device__ __forceinline__ void unpack8(uint4 v, float* x) {
  const float2 a = Op16<T>::unpack2(v.x), b = Op16<T>::unpack2(v.y), c = Op16<T>::unpack2(v.z),
               d = Op16<T>::unpack2(v.w);
  x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y; x[4] = c.x; x[5] = c.y; x[6] = d.x; x[7] = d.y;
}

}  // namespace sm100
}  // namespace gdn
