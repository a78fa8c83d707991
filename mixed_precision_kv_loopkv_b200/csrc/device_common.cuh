// Device helpers shared by the LoopKV kernels (sm_100a).
//
// Thin inline-PTX wrappers: mbarriers, 1-D bulk copies (TMA, no multicast)
// into the CTA's own shared memory, cluster barriers and distributed shared
// memory stores, programmatic dependent launch, and waits bounded by the
// global timer so that no kernel can spin forever.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "loopkv.h"

namespace loopkv {

constexpr int kGroup = 32;  // quantisation group: tokens (keys) or channels (values)
constexpr int kBlock = 16;  // tokens per paged block
constexpr unsigned long long kWaitTimeoutNs = 2000000000ull;  // 2 s

// Record layout of one (block, head) of a stored cell; see loopkv.h.
template <int KIND, int D>
struct Rec {
  static constexpr int kRow = D / 4;                  // bytes of one 2-bit plane row
  static constexpr int kPlane = kBlock * kRow;        // one 2-bit plane
  static constexpr int kKMeta = (D / 2) * 4;          // half the channels' (scale, min)
  static constexpr int kVMeta = kBlock * (D / kGroup) * 4;
  static constexpr int kBf16Rows = kBlock * D * 2;
  // 4-bit
  static constexpr int kQ4KHi = 0;
  static constexpr int kQ4KLo = kPlane;
  static constexpr int kQ4KMeta = 2 * kPlane;
  static constexpr int kQ4VHi = 2 * kPlane + kKMeta;
  static constexpr int kQ4VMeta = 3 * kPlane + kKMeta;
  static constexpr int kQ4VLo = 3 * kPlane + kKMeta + kVMeta;
  // 2-bit
  static constexpr int kQ2K = 0;
  static constexpr int kQ2KMeta = kPlane;
  static constexpr int kQ2V = kPlane + kKMeta;
  static constexpr int kQ2VMeta = 2 * kPlane + kKMeta;
  // bf16
  static constexpr int kBfK = 0;
  static constexpr int kBfV = kBf16Rows;

  static constexpr int kBytes = KIND == LOOPKV_CELL_Q4 ? 4 * kPlane + kKMeta + kVMeta
                               : KIND == LOOPKV_CELL_Q2 ? 2 * kPlane + kKMeta + kVMeta
                                                        : 2 * kBf16Rows;
  // where each section sits, independent of kind
  static constexpr int kKHi = KIND == LOOPKV_CELL_Q4 ? kQ4KHi : kQ2K;
  static constexpr int kKMetaOff = KIND == LOOPKV_CELL_Q4 ? kQ4KMeta : kQ2KMeta;
  static constexpr int kVHi = KIND == LOOPKV_CELL_Q4 ? kQ4VHi : kQ2V;
  static constexpr int kVMetaOff = KIND == LOOPKV_CELL_Q4 ? kQ4VMeta : kQ2VMeta;
};

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint16_t bf16_bits_rn(float x) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_timer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Wait for the phase with the given parity; false if it did not complete
// within kWaitTimeoutNs.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_timer_ns();
  for (;;) {
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (global_timer_ns() - t0 > kWaitTimeoutNs) return false;
  }
}

// ------------------------------------------------------- bulk copy (1-D TMA)
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
// Global -> this CTA's shared memory, completion counted on `bar`.  Both
// addresses 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar), "l"(policy)
      : "memory");
}

// Orders this thread's earlier generic-proxy global writes before later
// async-proxy (bulk copy) reads of the same bytes.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// blockIdx.y read afresh (not merged with earlier reads, so that it need not
// stay in a register in between)
__device__ __forceinline__ int cta_id_y() {
  int r;
  asm volatile("mov.u32 %0, %%ctaid.y;" : "=r"(r));
  return r;
}

// ----------------------------------------------------------------- cluster
// Every thread of every CTA of the cluster must call this (no early exits).
__device__ __forceinline__ void cluster_sync_all() {
  __syncwarp();
  asm volatile(
      "barrier.cluster.arrive.release.aligned;\n\t"
      "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Split cluster barrier.  The relaxed arrival at kernel start, waited on
// before the first store into a peer, proves that every CTA of the cluster
// has started; release / acquire pairs order the exchanges after it.
__device__ __forceinline__ void cluster_arrive_relaxed() {
  __syncwarp();
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  __syncwarp();
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive_release() {
  __syncwarp();
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
  __syncwarp();
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t peer_addr(uint32_t local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}

// Stores into a peer CTA's shared memory (visible to it after the next
// cluster barrier).  v4: 16-byte aligned address.
__device__ __forceinline__ void st_peer_f32(uint32_t addr, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}
__device__ __forceinline__ void st_peer_s32(uint32_t addr, int v) {
  asm volatile("st.shared::cluster.s32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void st_peer_v4(uint32_t addr, float4 v) {
  asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(v.x), "f"(v.y),
               "f"(v.z), "f"(v.w)
               : "memory");
}
// Atomic OR into a word of a cluster CTA's shared memory (this CTA's own
// included); visible after the next release / acquire cluster barrier.
__device__ __forceinline__ void or_peer_u32(uint32_t addr, uint32_t v) {
  asm volatile("red.relaxed.cluster.shared::cluster.or.b32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// ------------------------------------------------ programmatic dependent launch
// Both are no-ops when the kernel was launched without the attribute.
__device__ __forceinline__ void pdl_wait_prior_grid() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void pdl_allow_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// --------------------------------------------------------------------- math
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void flag_error(int32_t* err, int bits) {
  if (err) atomicOr(err, bits);
}

}  // namespace loopkv
