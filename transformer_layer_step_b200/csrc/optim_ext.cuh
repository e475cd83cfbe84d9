// Optimizer-side extensions of the layer step: gradient clipping by global
// norm and gradient accumulation over micro-batches.
//
// "Training GPT-2 with Megatron-LM" adds --clip-grad 1.0 against NaN losses
// (troubleshooting list) and accumulates gradients over micro-batches
// (§4.3, --gradient-accumulation-steps); "Megatron-LM overview" §5.1 names
// over-strong clipping as a cause of non-convergence.  The clip is the usual
// global-norm one: the unscaled gradient g = grad / S of the whole parameter
// arena is multiplied by max_norm / (||g|| + 1e-6) when that is below 1.
//
// Included by libgptlayer.cu after gptlayer.cu, in the same translation unit,
// so the entry points below share the library's argument checks, device
// check and launch recorder.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "gptlayer.h"

namespace gptl {

// Layout of the caller's clip workspace (GPTL_CLIP_WORKSPACE_BYTES).
constexpr int kClipNormOff = 0;        // float: ||grad / S||_2
constexpr int kClipCoefOff = 4;        // float: clip coefficient (<= 1)
constexpr int kClipStateOff = 16;      // gptl_scaler_state seen by the Adam pass
constexpr int kClipPartsOff = 64;      // double[kClipMaxParts]: per-block sums of squares
constexpr int kClipMaxParts = (GPTL_CLIP_WORKSPACE_BYTES - kClipPartsOff) / 8;
static_assert(kClipStateOff + (int)sizeof(gptl_scaler_state) <= kClipPartsOff, "clip workspace");

// One pass over the fp32 (scaled) gradient arena: found_inf |= any element
// is inf or NaN, and part[blockIdx.x] = sum of grad^2 over the elements this
// block visits, in float64.  Each thread adds its grid-stride elements in
// index order, then the block adds its threads' sums in a fixed tree, so the
// result depends only on the grid size.
__global__ void __launch_bounds__(256) norm_overflow_kernel(const float4 *__restrict__ g,
                                                            long long n4, int *__restrict__ found,
                                                            double *__restrict__ part) {
  __shared__ double warp_sum[8];
  bool bad = false;
  double acc = 0.0;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
       i += (long long)gridDim.x * blockDim.x) {
    const float4 v = __ldcs(g + i);
    const uint32_t e = 0x7F800000u;
    bad |= ((__float_as_uint(v.x) & e) == e) | ((__float_as_uint(v.y) & e) == e) |
           ((__float_as_uint(v.z) & e) == e) | ((__float_as_uint(v.w) & e) == e);
    acc += (double)v.x * (double)v.x;
    acc += (double)v.y * (double)v.y;
    acc += (double)v.z * (double)v.z;
    acc += (double)v.w * (double)v.w;
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(found, 1);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_down_sync(0xffffffffu, acc, o);
  if (lane == 0) warp_sum[warp] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double s = 0.0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) s += warp_sum[w];
    part[blockIdx.x] = s;
  }
}

// One block: adds the nparts partial sums in a fixed order, then writes the
// norm of the unscaled gradient, the clip coefficient, and the scaler state
// the Adam pass reads: the caller's state with its scale divided by the
// coefficient, so that Adam's grad / scale is (grad / S) * coef.  With no
// clipping the coefficient is exactly 1 and the state is the caller's.
__global__ void __launch_bounds__(256) clip_state_kernel(const double *__restrict__ part,
                                                         int nparts,
                                                         const gptl_scaler_state *__restrict__ st,
                                                         float max_norm, uint8_t *__restrict__ ws) {
  __shared__ double warp_sum[8];
  double acc = 0.0;
  for (int i = threadIdx.x; i < nparts; i += blockDim.x) acc += part[i];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_down_sync(0xffffffffu, acc, o);
  if (lane == 0) warp_sum[warp] = acc;
  __syncthreads();
  if (threadIdx.x != 0) return;
  double sumsq = 0.0;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) sumsq += warp_sum[w];
  const double S = (double)st->scale;
  const double norm = sqrt(sumsq) / S;
  const double c = (double)max_norm / (norm + 1e-6);
  const float coef = c < 1.0 ? (float)c : 1.0f;
  *reinterpret_cast<float *>(ws + kClipNormOff) = (float)norm;
  *reinterpret_cast<float *>(ws + kClipCoefOff) = coef;
  gptl_scaler_state eff = *st;
  if (coef < 1.0f) eff.scale = st->scale / coef;
  *reinterpret_cast<gptl_scaler_state *>(ws + kClipStateOff) = eff;
}

// acc[i] += grad[i], fp32, one rounding per element.
__global__ void __launch_bounds__(256) accumulate_kernel(float4 *__restrict__ acc,
                                                         const float4 *__restrict__ g,
                                                         long long n4) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
       i += (long long)gridDim.x * blockDim.x) {
    const float4 b = __ldcs(g + i);
    float4 a = acc[i];
    a.x += b.x;
    a.y += b.y;
    a.z += b.z;
    a.w += b.w;
    acc[i] = a;
  }
}

}  // namespace gptl

extern "C" {

int adam_step_fp32_master_clip(size_t n_params, float *master, float *m, float *v,
                               const float *grad, void *w16, gptl_dtype dtype, float lr,
                               float beta1, float beta2, float eps, float weight_decay,
                               float max_norm, void *clip_ws, gptl_scaler_state *st,
                               gptl_stream_t stream) {
  if (!master || !m || !v || !grad || !w16 || !st || !clip_ws) return GPTL_E_NULL;
  if (dtype != GPTL_FP16 && dtype != GPTL_BF16) return GPTL_E_DTYPE;
  if (!aligned16(master) || !aligned16(m) || !aligned16(v) || !aligned16(grad) || !aligned16(w16) ||
      !aligned16(clip_ws) || (reinterpret_cast<uintptr_t>(st) & 3u))
    return GPTL_E_ALIGN;
  if (n_params == 0 || n_params % 4 || !(lr >= 0.f) || !(beta1 >= 0.f && beta1 < 1.f) ||
      !(beta2 >= 0.f && beta2 < 1.f) || !(eps >= 0.f) || !(weight_decay >= 0.f) ||
      !(max_norm > 0.f) || !(max_norm <= 3.0e38f))
    return GPTL_E_ARG;
  int sms = 0;
  GPTL_TRY(device_check(&sms));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t *ws = static_cast<uint8_t *>(clip_ws);
  double *parts = reinterpret_cast<double *>(ws + kClipPartsOff);
  const long long n4 = (long long)(n_params / 4);

  TagScope tag_scope(GPTL_TAG_O1_OVERFLOW);
  GPTL_CK(cudaMemsetAsync(&st->found_inf, 0, sizeof(int), s));
  long long nb = (n4 + 255) / 256;
  if (nb > 4 * sms) nb = 4 * sms;
  if (nb > kClipMaxParts) nb = kClipMaxParts;
  prof_start(s);
  norm_overflow_kernel<<<(unsigned)nb, 256, 0, s>>>(reinterpret_cast<const float4 *>(grad), n4,
                                                    &st->found_inf, parts);
  GPTL_CK(cudaGetLastError());
  prof_launched(s, GPTL_KIND_OVERFLOW);
  clip_state_kernel<<<1, 256, 0, s>>>(parts, (int)nb, st, max_norm, ws);
  GPTL_CK(cudaGetLastError());
  prof_launched(s, GPTL_KIND_CLIP);

  g_tag = GPTL_TAG_O2_ADAM;
  const gptl_scaler_state *eff = reinterpret_cast<const gptl_scaler_state *>(ws + kClipStateOff);
  long long blocks = (n4 + 255) / 256;
  if (blocks > 8 * sms) blocks = 8 * sms;
  AdamArgs a{lr, beta1, beta2, eps, weight_decay};
  if (dtype == GPTL_FP16)
    adam_kernel<__half><<<(unsigned)blocks, 256, 0, s>>>(
        reinterpret_cast<float4 *>(master), reinterpret_cast<float4 *>(m),
        reinterpret_cast<float4 *>(v), reinterpret_cast<const float4 *>(grad),
        static_cast<__half *>(w16), n4, a, eff);
  else
    adam_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, s>>>(
        reinterpret_cast<float4 *>(master), reinterpret_cast<float4 *>(m),
        reinterpret_cast<float4 *>(v), reinterpret_cast<const float4 *>(grad),
        static_cast<__nv_bfloat16 *>(w16), n4, a, eff);
  GPTL_CK(cudaGetLastError());
  prof_launched(s, GPTL_KIND_ADAM);
  return GPTL_OK;
}

int gptl_grad_accumulate(size_t n, float *acc, const float *grad, gptl_stream_t stream) {
  if (!acc || !grad) return GPTL_E_NULL;
  if (!aligned16(acc) || !aligned16(grad)) return GPTL_E_ALIGN;
  if (n == 0 || n % 4) return GPTL_E_ARG;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(acc), g0 = reinterpret_cast<uintptr_t>(grad);
  if (a0 < g0 + n * sizeof(float) && g0 < a0 + n * sizeof(float)) return GPTL_E_ARG;
  int sms = 0;
  GPTL_TRY(device_check(&sms));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const long long n4 = (long long)(n / 4);
  long long blocks = (n4 + 255) / 256;
  if (blocks > 8 * sms) blocks = 8 * sms;
  prof_start(s);
  accumulate_kernel<<<(unsigned)blocks, 256, 0, s>>>(reinterpret_cast<float4 *>(acc),
                                                     reinterpret_cast<const float4 *>(grad), n4);
  GPTL_CK(cudaGetLastError());
  prof_launched(s, GPTL_KIND_ACCUMULATE);
  return GPTL_OK;
}

}  // extern "C"
