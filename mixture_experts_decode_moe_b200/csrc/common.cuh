// Device helpers shared by the libmoedec kernels (sm_100a only).
//
// Everything here is plumbing: bf16 bit helpers, PTX wrappers for mbarriers,
// bulk (TMA) copies, vector reductions, and a bounded grid-wide barrier for
// persistent cooperative kernels. None of it encodes the MoE arithmetic.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "moedec.h"  // include/ is on the include path

namespace moedec {

constexpr int kThreads = 256;   // threads per CTA for every persistent kernel
constexpr int kWarps = kThreads / 32;

// Status word values written by kernels (same numbering as moe_status).
constexpr uint32_t kStatusTimeout = MOE_ERR_TIMEOUT;
constexpr uint32_t kStatusBadIds = MOE_ERR_INVALID;

// Default budget for any device-side wait, in SM clock cycles (~1 s at
// 2 GHz). A wait that runs out records MOE_ERR_TIMEOUT and the kernel returns.
// A workspace may carry its own budget (WsControl::wait_budget, 0 = this).
constexpr long long kWaitBudgetCycles = 2000000000LL;

// WsControl::inject bits (set from the host for tests of the timeout path):
// every grid-wide barrier waits for one arrival more than the grid makes.
constexpr uint32_t kInjectBarrierExtraArrival = MOE_INJECT_BARRIER_EXTRA_ARRIVAL;

// Workspace control block (first 256 bytes of every workspace).
struct alignas(16) WsControl {
  uint32_t status;          // 0 = ok, else a moe_status
  uint32_t inject;          // fault-injection bits (kInject*), 0 = none
  unsigned long long bar;   // grid-barrier arrival counter (monotonic)
  unsigned long long wait_budget;  // cycles per bounded wait, 0 = kWaitBudgetCycles
  unsigned long long pad[13];
  // batch-1 decode: routed jobs handed out per layer (layer l uses
  // pool[l % 3]), in a cache line of their own
  uint32_t pool[4];
  uint32_t pad2[28];
};
static_assert(sizeof(WsControl) == 256, "control block is 256 bytes");

// ---------------------------------------------------------------- bf16

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }
__device__ __forceinline__ float bf16_to_f(uint16_t v) { return __uint_as_float(uint32_t(v) << 16); }

// fp32 -> bf16, round to nearest even (finite inputs; NaN kept quiet).
__device__ __forceinline__ uint16_t f_to_bf16(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7F800000u) == 0x7F800000u) return uint16_t((u >> 16) | ((u & 0xFFFFu) ? 0x40u : 0u));
  u += 0x7FFFu + ((u >> 16) & 1u);
  return uint16_t(u >> 16);
}

// Unpack 8 bf16 (one 16-byte vector) into fp32.
__device__ __forceinline__ void unpack8(const uint4& v, float* f) {
  f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x);
  f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
  f[4] = bf16_lo(v.z); f[5] = bf16_hi(v.z);
  f[6] = bf16_lo(v.w); f[7] = bf16_hi(v.w);
}

// Order-preserving map fp32 -> u32 (larger float => larger key; -0 == +0).
__device__ __forceinline__ uint32_t float_key(float f) {
  uint32_t u = __float_as_uint(f + 0.0f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ---------------------------------------------------------------- PTX wrappers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// try_wait with a suspend-time hint: the thread sleeps in hardware until the
// phase completes or about `ns` nanoseconds pass, instead of spinning.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t ns) {
  uint32_t ok;
  asm volatile(
      "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3; selp.u32 %0, 1, 0, p; }"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(ns)
      : "memory");
  return ok != 0;
}

// The wait budget of a workspace (read once per kernel).
__device__ __forceinline__ long long ctl_wait_budget(const WsControl* ctl) {
  const unsigned long long b = ctl->wait_budget;
  return b ? (long long)(b > 0x7fffffffffffffffull ? 0x7fffffffffffffffull : b) : kWaitBudgetCycles;
}

// Bounded wait on an mbarrier phase. Returns false if the budget ran out.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, long long budget = kWaitBudgetCycles) {
  if (mbar_try_wait_sleep(bar, parity, 20000)) return true;
  long long t0 = clock64();
  while (!mbar_try_wait_sleep(bar, parity, 20000)) {
    if (clock64() - t0 > budget) return false;
  }
  return true;
}

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ uint64_t policy_evict_normal() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// 1-D bulk copy global -> this CTA's shared memory, completing on `bar`.
// dst, src 16-byte aligned; bytes a multiple of 16. No multicast.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                         uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// Prefetch [src, src + bytes) from global memory into L2 (no shared memory
// involved, no completion to wait for). src 16-byte aligned, bytes a
// multiple of 16.
__device__ __forceinline__ void prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

__device__ __forceinline__ unsigned long long atom_add_release_gpu(unsigned long long* p,
                                                                   unsigned long long v) {
  unsigned long long old;
  asm volatile("atom.add.release.gpu.global.u64 %0, [%1], %2;" : "=l"(old) : "l"(p), "l"(v) : "memory");
  return old;
}
__device__ __forceinline__ unsigned long long ld_acquire_gpu(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void set_status(WsControl* ctl, uint32_t code) {
  atomicCAS(&ctl->status, 0u, code);
}

}  // namespace moedec
