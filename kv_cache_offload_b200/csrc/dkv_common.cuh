// Shared device-side helpers for libdkv (sm_100a): pool view, error bits, mbarrier,
// bulk-copy and cp.async wrappers, bounded waits.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/dkv.h"

namespace dkv {

// Status-word bits set by kernels (never trap; skip and flag instead).
enum : int {
  kErrBadTier = 1,
  kErrBadBlock = 2,
  kErrCtxTooLong = 4,
  kErrTimeout = 8,
  kErrBadPlan = 16,
  kErrDebugBounds = 32,  // a DKV_DEBUG range check failed (an indexing bug, not bad input)
};

// What a kernel needs to address the pool.
struct PoolView {
  uint16_t* tier[2];     // device-accessible bases (HBM, host alias)
  int64_t blocks[2];     // physical blocks per tier
  int32_t L, Hkv, D, T;
  int32_t layout;        // DKV_LAYOUT_*
  int* status;           // device status word
};

// Element offset of the [T][D] chunk (layer, phys, kv, g) inside a tier.
__host__ __device__ __forceinline__ int64_t chunk_offset(const PoolView& p, int tier, int layer,
                                                         int64_t phys, int kv, int g) {
  int64_t c;
  if (p.layout == DKV_LAYOUT_LAYER_FIRST)
    c = (((int64_t)layer * (tier ? p.blocks[1] : p.blocks[0]) + phys) * 2 + kv) * p.Hkv + g;
  else
    c = (((int64_t)phys * p.L + layer) * 2 + kv) * p.Hkv + g;
  return c * (int64_t)p.T * p.D;
}

// Tier base / size selected without dynamic indexing into the by-value struct (which
// would put the struct in local memory).
__host__ __device__ __forceinline__ uint16_t* tier_base(const PoolView& p, int tier) {
  return tier ? p.tier[1] : p.tier[0];
}
__host__ __device__ __forceinline__ int64_t tier_blocks(const PoolView& p, int tier) {
  return tier ? p.blocks[1] : p.blocks[0];
}

__device__ __forceinline__ void flag_error(int* status, int bits) {
  if (status) atomicOr(status, bits);
}

// Elements of a tier (every layer, K and V, every kv head, T tokens of D).
__host__ __device__ __forceinline__ int64_t tier_elems(const PoolView& p, int tier) {
  return tier_blocks(p, tier) * p.L * 2 * p.Hkv * p.T * p.D;
}

// Range checks of the DKV_DEBUG build: every block, slot and workspace access whose index
// the kernel computed is checked to lie in its buffer ([lo, hi) within [0, n)); a failing
// access is skipped and flags kErrDebugBounds (dkv_check: DKV_ERR_INTERNAL). The release
// build compiles them to `true`.
#ifdef DKV_DEBUG
__device__ __forceinline__ bool debug_in_range(int* status, int64_t lo, int64_t hi, int64_t n) {
  if (lo >= 0 && lo <= hi && hi <= n) return true;
  flag_error(status, kErrDebugBounds);
  return false;
}
#define DKV_DEBUG_RANGE(status, lo, hi, n) ::dkv::debug_in_range((status), (lo), (hi), (n))
#else
#define DKV_DEBUG_RANGE(status, lo, hi, n) true
#endif

// ---------------------------------------------------- programmatic dependent launch
// A kernel launched with programmatic stream serialization may start before the kernel
// ahead of it in the stream has finished. griddep_wait() blocks the calling thread until
// that kernel has completed and its memory is visible (a no-op for a normal launch);
// griddep_launch_dependents() lets the next such kernel start once every CTA of this grid
// has signalled (or exited). Both exist on sm_90 and later.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ------------------------------------------------------------------ shared memory

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------- mbarrier

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

// Test the phase; if it is not complete the thread sleeps until it completes or about
// `hint_ns` pass (suspend-time hint), so waiting warps do not spin on the issue slots.
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity, uint32_t hint_ns = 20000) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Wait for the phase with `parity` to complete, giving up after `limit_ns` of wall time.
// Returns false (and flags kErrTimeout) on give-up. Never spins forever.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, int* status,
                                                  uint64_t limit_ns = 4000000000ull) {
  if (mbar_try_wait(bar, parity)) return true;
  uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 15u) == 15u && globaltimer_ns() - t0 > limit_ns) {
      flag_error(status, kErrTimeout);
      return false;
    }
  }
}

// ------------------------------------------------------------------- bulk copies

// 1-D bulk copy global -> shared (TMA engine), completing `bytes` on `bar`.
// Requires 16-byte aligned addresses and bytes % 16 == 0.
__device__ __forceinline__ void bulk_g2s(void* dst_smem, const void* src_gmem, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst_smem)),
      "l"(src_gmem), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// An L2 cache policy that marks the lines it fills for first eviction (data read exactly
// once, such as cached KV streamed by the attention), so they do not displace lines other
// kernels will reuse.
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// bulk_g2s with an L2 cache-policy hint (from l2_policy_*).
__device__ __forceinline__ void bulk_g2s_hint(void* dst_smem, const void* src_gmem, uint32_t bytes, uint64_t* bar,
                                              uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::
          "r"(smem_u32(dst_smem)),
      "l"(src_gmem), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// 16-byte asynchronous copy global -> shared through the LSU (works for mapped host memory).
__device__ __forceinline__ void cp_async16(void* dst_smem, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst_smem)), "l"(src)
               : "memory");
}

// Arrive on `bar` once all of this thread's prior cp.async copies have landed; the arrival
// counts against the barrier's initial count (no pending-count increment).
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}

// Named barrier among `nthreads` threads (multiple of 32).
__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ------------------------------------------------------------------ conversions

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

}  // namespace dkv
