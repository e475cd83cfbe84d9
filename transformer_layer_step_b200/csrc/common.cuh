// common.cuh — device helpers shared by the layer's kernels (sm_100a only).
//
// PTX wrappers for mbarriers, TMA tensor loads and the tcgen05 (5th-gen
// tensor core + tensor memory) instructions, 16-bit conversions, and the
// library's device error word.  Every wait on an mbarrier is bounded: after
// ~2 s of %globaltimer it records an error bit and gives up instead of
// hanging the GPU.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gptlayer.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "this library targets sm_100a only"
#endif

namespace gptl {

// Library-wide device error word (bit 0: a pipeline wait timed out; bit 1: an
// internal index check failed).  Read by gptl_read_device_error().
__device__ int g_device_error;

enum : int { kErrTimeout = 1, kErrIndex = 2 };

constexpr unsigned long long kWaitTimeoutNs = 2000000000ull;   // 2 s

__device__ __forceinline__ void set_device_error(int bit) { atomicOr(&g_device_error, bit); }

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long globaltimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
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

// As mbar_try_wait, but with a 20 ns suspend-time hint: the thread is
// suspended at most ~20 ns before it looks again.  Measured on B200, this
// shortens the hand-off between pipeline roles against the default (longer)
// suspend of a plain try_wait, and against a non-blocking test_wait spin.
__device__ __forceinline__ bool mbar_try_wait_short(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(20u)
      : "memory");
  return ok != 0;
}

// Wait until the phase with the given parity has completed.  Returns false
// (and records kErrTimeout) after kWaitTimeoutNs, or at once when *abort is
// set by another role of the same CTA.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int *abort) {
#pragma unroll 1
  for (int i = 0; i < 256; ++i)
    if (mbar_try_wait_short(bar, parity)) return true;
  const unsigned long long t0 = globaltimer();
#pragma unroll 1
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 1024; ++i)
      if (mbar_try_wait_short(bar, parity)) return true;
    if (*abort) return false;
    if (globaltimer() - t0 > kWaitTimeoutNs) {
      set_device_error(kErrTimeout);
      *abort = 1;
      return false;
    }
  }
}

// Bounded wait used on the abort path (the abort flag is already set).
__device__ __forceinline__ bool mbar_wait_drain(uint32_t bar, uint32_t parity) {
  const unsigned long long t0 = globaltimer();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer() - t0 > kWaitTimeoutNs) return false;
  return true;
}

// --------------------------------------------------------------------- TMA
// 3-D tiled tensor load into shared memory, completing on an mbarrier.
// Every CTA loads its own operands from this GPU's memory.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *map, int x, int y,
                                            int z, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}

// 4-D tiled tensor store from shared memory, tracked by this thread's bulk
// async-groups (commit with bulk_commit, wait with bulk_wait_read/bulk_wait).
// Elements of the box outside the tensor's extents are not written.
__device__ __forceinline__ void tma_store_4d(const CUtensorMap *map, uint32_t src, int x, int y,
                                             int z, int w) {
  asm volatile(
      "cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(src), "r"(x), "r"(y), "r"(z), "r"(w)
      : "memory");
}
// The same store with an L2 eviction-priority hint (a createpolicy value):
// outputs that nothing reads soon (the weight gradients, read by the
// optimizer step) leave L2 first and do not push the operands out.
__device__ __forceinline__ void tma_store_4d_hint(const CUtensorMap *map, uint32_t src, int x, int y,
                                                  int z, int w, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.4d.global.shared::cta.bulk_group.L2::cache_hint"
      " [%0, {%2, %3, %4, %5}], [%1], %6;" ::"l"(reinterpret_cast<uint64_t>(map)),
      "r"(src), "r"(x), "r"(y), "r"(z), "r"(w), "l"(policy)
      : "memory");
}
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Wait until at most N of this thread's committed groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// Wait until all of this thread's committed groups have completed.
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ----------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem], kind::f16 (fp16/bf16 inputs, fp32 accumulate)
__device__ __forceinline__ void tc_mma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on an mbarrier when all previously issued tcgen05 ops of this
// thread have completed.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}

// 32 lanes x 32 bit, 16 consecutive columns: thread i of the warp gets TMEM
// lane (lane_base + i), columns col .. col+15.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32"
      " {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 32 lanes x 32 bit, 16 consecutive columns, registers -> TMEM (the inverse
// of tmem_ld16); complete with tmem_wait_st().
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32"
      " [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Makes this thread's generic-proxy shared-memory writes visible to the
// async proxy (the tensor core reading an operand tile).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

// Shared-memory matrix descriptor (tcgen05 "version 1" format):
//   [0,14) start>>4  [16,30) leading byte offset>>4  [32,46) stride byte
//   offset>>4  [46,48) version=1  [49,52) base offset=0  [61,64) layout
// layout: 2 = 128B swizzle, 4 = 64B swizzle, 6 = 32B swizzle.
__device__ __forceinline__ uint64_t make_smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo,
                                                   uint32_t layout) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFF);
  d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)(layout & 7) << 61;
  return d;
}

// ------------------------------------------------------------ conversions
template <typename T> struct Cvt;
template <> struct Cvt<__half> {
  static __device__ __forceinline__ float to_f(__half v) { return __half2float(v); }
  static __device__ __forceinline__ __half from_f(float v) { return __float2half_rn(v); }
  static __device__ __forceinline__ uint32_t pack2(float a, float b) {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
  }
  static __device__ __forceinline__ float2 unpack2(uint32_t u) {
    __half2 h = *reinterpret_cast<__half2 *>(&u);
    return __half22float2(h);
  }
};
template <> struct Cvt<__nv_bfloat16> {
  static __device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
  static __device__ __forceinline__ __nv_bfloat16 from_f(float v) { return __float2bfloat16_rn(v); }
  static __device__ __forceinline__ uint32_t pack2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
  }
  static __device__ __forceinline__ float2 unpack2(uint32_t u) {
    __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162 *>(&u);
    return __bfloat1622float2(h);
  }
};

// 8 packed 16-bit values (one 16-byte vector) <-> 8 floats
template <typename T>
__device__ __forceinline__ void unpack8(const uint4 &u, float (&f)[8]) {
  float2 a = Cvt<T>::unpack2(u.x), b = Cvt<T>::unpack2(u.y), c = Cvt<T>::unpack2(u.z),
         d = Cvt<T>::unpack2(u.w);
  f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y; f[4] = c.x; f[5] = c.y; f[6] = d.x; f[7] = d.y;
}
template <typename T>
__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  uint4 u;
  u.x = Cvt<T>::pack2(f[0], f[1]);
  u.y = Cvt<T>::pack2(f[2], f[3]);
  u.z = Cvt<T>::pack2(f[4], f[5]);
  u.w = Cvt<T>::pack2(f[6], f[7]);
  return u;
}

// Single-instruction base-2 exponential and reciprocal of the SFU
// (ex2.approx / rcp.approx, flush-to-zero): relative error about 2^-22.
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// GeLU, tanh form (GPT-2 / Megatron fused bias-GeLU), and its derivative.
// With u = sqrt(2/pi) (z + 0.044715 z^3), 0.5 (1 + tanh u) is the logistic
// sigmoid s = 1 / (1 + e^{-2u}), so GeLU(z) = z s and
// GeLU'(z) = s + z s (1 - s) 2u'(z), 2u'(z) = 2 sqrt(2/pi) (1 + 3 * 0.044715 z^2).
// e^{-2u} is taken as 2^{z (k1 + k2 z^2)}, k1 = -2 sqrt(2/pi) / ln 2, k2 = 0.044715 k1.
// Far below zero e^{-2u} overflows to +inf and s to 0: GeLU -> -0, GeLU' -> 0.
__device__ __forceinline__ float gelu_sigmoid(float z) {
  const float k1 = -2.3022082f, k2 = -0.10294324f;
  return rcp_approx(1.0f + ex2_approx(z * fmaf(k2, z * z, k1)));
}
__device__ __forceinline__ float gelu_f(float z) { return z * gelu_sigmoid(z); }
// The polynomial's argument is clamped to |z| <= 1e4 so that z^2 cannot
// overflow; beyond |z| ~ 40 the term it scales is multiplied by exactly 0
// (s = 0 below, 1 - s = 0 above), and a NaN still reaches the result through s.
__device__ __forceinline__ float gelu_prime_f(float z) {
  const float c2 = 1.5957692f, c6 = 0.21406445f;   // 2 sqrt(2/pi), 6 * 0.044715 sqrt(2/pi)
  const float s = gelu_sigmoid(z);
  const float zc = fminf(fmaxf(z, -1e4f), 1e4f);
  return s * fmaf(z * (1.0f - s), fmaf(c6, zc * zc, c2), 1.0f);
}

// Sum of v[j] over the warp's 32 lanes for each of the 16 columns j, in five
// exchange steps (16 shuffles): each step hands half of the remaining
// columns to the partner lane and keeps the other half.  Lane l ends with
// the sum of column (l >> 1) & 15 (lanes l and l ^ 1 hold the same value);
// the order of the additions is fixed.
__device__ __forceinline__ float warp_colsum16(const float (&v)[16], int lane) {
  float s8[8], s4[4], s2[2];
  const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4, b1 = lane & 2;
#pragma unroll
  for (int i = 0; i < 8; ++i)
    s8[i] = (b4 ? v[i + 8] : v[i]) + __shfl_xor_sync(0xffffffffu, b4 ? v[i] : v[i + 8], 16);
#pragma unroll
  for (int i = 0; i < 4; ++i)
    s4[i] = (b3 ? s8[i + 4] : s8[i]) + __shfl_xor_sync(0xffffffffu, b3 ? s8[i] : s8[i + 4], 8);
#pragma unroll
  for (int i = 0; i < 2; ++i)
    s2[i] = (b2 ? s4[i + 2] : s4[i]) + __shfl_xor_sync(0xffffffffu, b2 ? s4[i] : s4[i + 2], 4);
  const float s1 = (b1 ? s2[1] : s2[0]) + __shfl_xor_sync(0xffffffffu, b1 ? s2[0] : s2[1], 2);
  return s1 + __shfl_xor_sync(0xffffffffu, s1, 1);
}

}  // namespace gptl
