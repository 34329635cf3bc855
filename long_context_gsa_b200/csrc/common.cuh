// common.cuh -- device helpers shared by the GSA kernels (sm_100a).
//
// Bulk (TMA-engine) copies with mbarrier completion, bounded waits that
// record a status bit instead of hanging, programmatic-dependent-launch
// controls, bf16 unpacking, warp reductions and a base-2 exponential.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/gsa.h"

namespace gsa {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Longest time a thread waits on an mbarrier (or a counter another CTA
// advances) before it gives up and flags GSA_DEVERR_TIMEOUT (nanoseconds of
// %globaltimer).  A test build may shorten it with -DGSA_WAIT_LIMIT_NS.
#ifndef GSA_WAIT_LIMIT_NS
#define GSA_WAIT_LIMIT_NS 2000000000ull
#endif
constexpr uint64_t kWaitLimitNs = GSA_WAIT_LIMIT_NS;

// Extra transaction bytes that some copy barriers expect: 0 in the library.
// The failure-detection test builds a variant with 16, so those barriers
// never complete (their copies land, the count stays short) and the bounded
// waits must expire, flag GSA_DEVERR_TIMEOUT and let the kernel return.
#ifndef GSA_TEST_STALL_BYTES
#define GSA_TEST_STALL_BYTES 0u
#endif

// Test builds only: with 1, the fused decode's scoring tail never publishes
// row 0 in the ready list, so the unfold CTA that waits for the last slot
// must run out of its wait, flag GSA_DEVERR_TIMEOUT and return.
#ifndef GSA_TEST_SKIP_PUBLISH
#define GSA_TEST_SKIP_PUBLISH 0
#endif

// Partial softmax record: base-2 max, sum, then `d` accumulator floats.
// Stored as float[d + 4] (the two pad floats keep the accumulator 16-byte
// aligned).  Logits are kept in the base-2 domain: z2 = scale*log2(e)*q.k.
constexpr int kPartHeader = 4;

__device__ __forceinline__ float neg_inf() { return __int_as_float(0xff800000u); }

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Acquire load of a flag or counter another CTA updates (gpu scope).
__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t *p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Release store of a flag another CTA acquires (gpu scope).
__device__ __forceinline__ void st_release_u32(uint32_t *p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// The ready list of the fused decode step: the scoring kernel's tail
// publishes each selected row (row + 1, in completion order) and the unfold
// CTAs take them in that order.  Words [rows .. rows + 2] are the
// publisher's slot counter, the unfold's ticket counter and its done
// counter; the unfold's last CTA clears the whole list.
struct ReadyList {
  uint32_t *w;  // [rows + 4] or null
  int32_t rows;
};

__device__ __forceinline__ void flag_error(uint32_t *status, uint32_t bits);

// Publish `row` (its outputs written and fenced by every writer).
__device__ __forceinline__ void ready_publish(const ReadyList &r, int row, uint32_t *status) {
  if (GSA_TEST_SKIP_PUBLISH && row == 0) return;
  const uint32_t pos = atomicAdd(&r.w[r.rows], 1u);
  if (pos < static_cast<uint32_t>(r.rows))
    st_release_u32(&r.w[pos], static_cast<uint32_t>(row) + 1u);
  else
    flag_error(status, GSA_DEVERR_CAPACITY);  // a list left over from a failed call
}

__device__ __forceinline__ void flag_error(uint32_t *status, uint32_t bits) {
  if (status) atomicOr(status, bits);
}

// ---- mbarrier + bulk copy ------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for phase `parity` of `bar`; false if kWaitLimitNs passed first.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0 && global_timer_ns() - t0 > kWaitLimitNs) return false;
  }
}

// Global -> shared bulk copy through the TMA engine; completion is counted
// on `bar` as transaction bytes.  dst, src 16-byte aligned, bytes % 16 == 0.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// ---- programmatic dependent launch ----------------------------------------
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---- arithmetic -----------------------------------------------------------
// 2^x on the SFU (ex2.approx, flush-to-zero); 2^-inf = 0.
__device__ __forceinline__ float exp2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// bf16 pair in one 32-bit word -> two floats (exact).
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Eight elements (16 bytes) of T as floats.
template <typename T>
struct Vec16;

template <>
struct Vec16<__nv_bfloat16> {
  static constexpr int kElems = 8;
  __device__ __forceinline__ static void unpack(const uint4 &w, float *f) {
    f[0] = bf16_lo(w.x); f[1] = bf16_hi(w.x);
    f[2] = bf16_lo(w.y); f[3] = bf16_hi(w.y);
    f[4] = bf16_lo(w.z); f[5] = bf16_hi(w.z);
    f[6] = bf16_lo(w.w); f[7] = bf16_hi(w.w);
  }
};

template <>
struct Vec16<float> {
  static constexpr int kElems = 4;
  __device__ __forceinline__ static void unpack(const uint4 &w, float *f) {
    f[0] = __uint_as_float(w.x); f[1] = __uint_as_float(w.y);
    f[2] = __uint_as_float(w.z); f[3] = __uint_as_float(w.w);
  }
};

__device__ __forceinline__ uint4 ldg_nc_v4(const void *p) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ uint4 lds_v4(const void *p) { return *reinterpret_cast<const uint4 *>(p); }

// Order-preserving map of a finite float to uint32 (larger float -> larger
// key); -0 is canonicalised to +0 first.
__device__ __forceinline__ uint32_t float_to_key(float s) {
  uint32_t u = __float_as_uint(s == 0.0f ? 0.0f : s);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_to_float(uint32_t k) {
  uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
  return __uint_as_float(u);
}

// Store one float of the attention output in the requested dtype.
__device__ __forceinline__ void store_out(void *out, size_t i, float v, int out_bf16) {
  if (out_bf16)
    reinterpret_cast<__nv_bfloat16 *>(out)[i] = __float2bfloat16_rn(v);
  else
    reinterpret_cast<float *>(out)[i] = v;
}

}  // namespace gsa
