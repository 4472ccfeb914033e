// Device helpers shared by the libduo kernels (sm_100a): bulk copies into
// shared memory, mbarriers with bounded waits, bf16 unpacking, packed fp32
// arithmetic.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kernels.h"

namespace duo {

// An mbarrier wait gives up after about kWaitNs nanoseconds of polling (read
// from the global timer), records its code in the error word and returns false.
constexpr uint64_t kWaitNs = 1000000000ull;

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
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

// Bounded wait for the phase with the given parity to complete.  Returns false
// (and records `code` in the error word) if it did not within limit_ns.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, int *err, int code,
                                          uint64_t limit_ns = kWaitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (;;) {
    for (int i = 0; i < 256; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (global_ns() - t0 > limit_ns) break;
  }
  if (err) atomicOr(err, code);
  return false;
}

// One-dimensional bulk copy global -> shared, completing `bytes` of
// transaction count on `bar`.  dst, src 16-byte aligned, bytes % 16 == 0.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes,
                                         uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

// Two bf16 packed in a 32-bit word -> (low element, high element) as fp32.
// bf16 is the upper half of an fp32, so this is exact bit placement.
__device__ __forceinline__ float2 bf16x2_to_f2(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) { return __fmul2_rn(a, b); }

// 2^x through the hardware's approximate base-2 exponential instruction.
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float fast_log2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Unpack one 16-byte chunk into fp32 pairs: 8 bf16 -> 4 pairs, 4 f32 -> 2 pairs.
template <typename T>
struct Chunk;

template <>
struct Chunk<__nv_bfloat16> {
  static constexpr int kPairs = 4;
  __device__ __forceinline__ static void unpack(const uint4 &c, float2 (&f)[4]) {
    f[0] = bf16x2_to_f2(c.x);
    f[1] = bf16x2_to_f2(c.y);
    f[2] = bf16x2_to_f2(c.z);
    f[3] = bf16x2_to_f2(c.w);
  }
};

template <>
struct Chunk<float> {
  static constexpr int kPairs = 2;
  __device__ __forceinline__ static void unpack(const uint4 &c, float2 (&f)[2]) {
    f[0] = make_float2(__uint_as_float(c.x), __uint_as_float(c.y));
    f[1] = make_float2(__uint_as_float(c.z), __uint_as_float(c.w));
  }
};

__device__ __forceinline__ void store_out(float *p, float v) { *p = v; }
__device__ __forceinline__ void store_out(__nv_bfloat16 *p, float v) { *p = __float2bfloat16_rn(v); }

__device__ __forceinline__ float load_in(const float *p) { return *p; }
__device__ __forceinline__ float load_in(const __nv_bfloat16 *p) { return __bfloat162float(*p); }

// Storage row of retrieval key `key` of (batch row b, retrieval head pidx);
// see RetMap.
__device__ __forceinline__ int64_t ret_row(const RetMap &m, int b, int pidx, int64_t key) {
  if (!m.table) return ((int64_t)b * m.n_ret + pidx) * m.cap + key;
  const int64_t blk = m.table[(int64_t)b * m.stride + (key >> kPageShift)];
  return ((blk * m.n_ret + pidx) << kPageShift) + (key & (kPageTokens - 1));
}

// Ring slot of position p in a streaming head's buffer: sinks first, then
// an R-slot ring.
__device__ __forceinline__ int64_t ring_slot(int64_t p, int S, int R) {
  return p < S ? p : S + (p - S) % R;
}

}  // namespace duo
