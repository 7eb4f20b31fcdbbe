// dp_ddim.cu -- the sampler update between two denoising steps.
//
// DistriFusion's results use a 50-step DDIM sampler ("DistriFusion",
// atlas.scime.ai summary, Key results and the GroupNorm ablation rows); every
// step of it runs the displaced U-Net once and then moves the latent from
// timestep t to the previous one.  The update is the deterministic DDIM step
// (eta = 0; Song, Meng and Ermon, "Denoising Diffusion Implicit Models",
// ICLR 2021, the generative process of section 4.1 with sigma = 0):
//   x0_hat = (x_t - sqrt(1 - abar_t) eps) / sqrt(abar_t)
//   x_prev = sqrt(abar_prev) x0_hat + sqrt(1 - abar_prev) eps
// which is linear in (x_t, eps): x_prev = ca x_t + ce eps with
//   ca = sqrt(abar_prev / abar_t),
//   ce = sqrt(1 - abar_prev) - sqrt(abar_prev (1 - abar_t) / abar_t).
// The host folds the schedule into (ca, ce) in double precision; the kernel
// is one fused multiply-add per element in fp32, so it is HBM-bound: read x
// and eps, write x_prev.  The update is elementwise, so every band runs it
// on its own rows with no context from other bands.
#include <cmath>

#include "dp_common.cuh"
#include "dp_internal.h"

namespace dp {

__device__ __forceinline__ float ddim_one(float x, float e, float ca, float ce) { return fmaf(ca, x, ce * e); }

// bf16: 8 elements per 16-byte vector; the ragged tail (n % 8) goes element by element
__global__ void __launch_bounds__(256) ddim_bf16_kernel(const __nv_bfloat16* x, const __nv_bfloat16* __restrict__ eps,
                                                        __nv_bfloat16* y, size_t n, float ca, float ce) {
  griddep_wait();
  griddep_trigger();
  const size_t nv = n / 8;
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  const size_t tid = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const uint4* xv = reinterpret_cast<const uint4*>(x);
  const uint4* ev = reinterpret_cast<const uint4*>(eps);
  uint4* yv = reinterpret_cast<uint4*>(y);
  for (size_t i = tid; i < nv; i += stride) {
    const uint4 a = xv[i], b = ev[i];
    const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
    uint32_t o[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float x0 = __uint_as_float(wa[k] << 16), x1 = __uint_as_float(wa[k] & 0xffff0000u);
      const float e0 = __uint_as_float(wb[k] << 16), e1 = __uint_as_float(wb[k] & 0xffff0000u);
      o[k] = pack_bf16x2(ddim_one(x0, e0, ca, ce), ddim_one(x1, e1, ca, ce));
    }
    yv[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
  for (size_t i = nv * 8 + tid; i < n; i += stride)
    y[i] = __float2bfloat16_rn(ddim_one(__bfloat162float(x[i]), __bfloat162float(eps[i]), ca, ce));
}

// fp32: 4 elements per 16-byte vector, then the tail
__global__ void __launch_bounds__(256) ddim_f32_kernel(const float* x, const float* __restrict__ eps, float* y,
                                                       size_t n, float ca, float ce) {
  griddep_wait();
  griddep_trigger();
  const size_t nv = n / 4;
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  const size_t tid = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const float4* xv = reinterpret_cast<const float4*>(x);
  const float4* ev = reinterpret_cast<const float4*>(eps);
  float4* yv = reinterpret_cast<float4*>(y);
  for (size_t i = tid; i < nv; i += stride) {
    const float4 a = xv[i], b = ev[i];
    yv[i] = make_float4(ddim_one(a.x, b.x, ca, ce), ddim_one(a.y, b.y, ca, ce), ddim_one(a.z, b.z, ca, ce),
                        ddim_one(a.w, b.w, ca, ce));
  }
  for (size_t i = nv * 4 + tid; i < n; i += stride) y[i] = ddim_one(x[i], eps[i], ca, ce);
}

}  // namespace dp

extern "C" {

int dp_ddim_step(const void* x, const void* eps, void* x_prev, size_t n, double abar_t, double abar_prev,
                 int dtype, void* stream) {
  if (!x || !eps || !x_prev) return dp::set_error(DP_ERR_INVALID_ARG, "ddim: null pointer");
  if (dtype != DP_BF16 && dtype != DP_FP32) return dp::set_error(DP_ERR_INVALID_ARG, "ddim: bad dtype");
  if (!(abar_t > 0.0 && abar_t <= 1.0) || !(abar_prev > 0.0 && abar_prev <= 1.0))
    return dp::set_error(DP_ERR_INVALID_ARG, "ddim: alpha-bar values must lie in (0, 1]");
  if (!dp::aligned16(x) || !dp::aligned16(eps) || !dp::aligned16(x_prev))
    return dp::set_error(DP_ERR_UNSUPPORTED, "ddim: pointers must be 16-byte aligned");
  const size_t es = dtype == DP_FP32 ? 4 : 2;
  if (n > (static_cast<size_t>(-1) >> 3)) return dp::set_error(DP_ERR_INVALID_ARG, "ddim: n too large");
  const size_t bytes = n * es;
  const char* xb = static_cast<const char*>(x);
  const char* eb = static_cast<const char*>(eps);
  const char* yb = static_cast<const char*>(x_prev);
  if (yb < eb + bytes && eb < yb + bytes) return dp::set_error(DP_ERR_INVALID_ARG, "ddim: x_prev overlaps eps");
  if (yb != xb && yb < xb + bytes && xb < yb + bytes)
    return dp::set_error(DP_ERR_INVALID_ARG, "ddim: x_prev overlaps x without being x");
  if (n == 0) return DP_OK;
  const float ca = static_cast<float>(std::sqrt(abar_prev / abar_t));
  const float ce =
      static_cast<float>(std::sqrt(1.0 - abar_prev) - std::sqrt(abar_prev * (1.0 - abar_t) / abar_t));
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t vec = 16 / es;
  size_t blocks = (n / vec + 255) / 256;
  const size_t cap = static_cast<size_t>(dp::num_sms()) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks == 0) blocks = 1;
  dp::mark_launch(st);
  if (dtype == DP_FP32)
    return dp::launch_kernel(dp::ddim_f32_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, st, false,
                             "ddim launch", static_cast<const float*>(x), static_cast<const float*>(eps),
                             static_cast<float*>(x_prev), n, ca, ce);
  return dp::launch_kernel(dp::ddim_bf16_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, st, false,
                           "ddim launch", static_cast<const __nv_bfloat16*>(x),
                           static_cast<const __nv_bfloat16*>(eps), static_cast<__nv_bfloat16*>(x_prev), n, ca,
                           ce);
}

}  // extern "C"
