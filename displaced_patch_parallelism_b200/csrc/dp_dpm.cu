// dp_dpm.cu -- the multistep second-order DPM-Solver++ update between two
// denoising steps.
//
// The pages' warm-up ablation runs DistriFusion with a "10-step DPM-Solver"
// ("DistriFusion", atlas.scime.ai summary, the warm-up ablation rows).  The
// update is the multistep second-order DPM-Solver++ in data prediction (Lu,
// Zhou, Bao, Chen, Li and Zhu, "DPM-Solver++: Fast Solver for Guided Sampling
// of Diffusion Probabilistic Models"): one model evaluation per step, the
// previous step's data prediction supplying the second-order term.  With
// alpha = sqrt(abar), sigma = sqrt(1 - abar), lambda = log(alpha / sigma) and
// h = lambda_t - lambda_s, from level s to the less noisy level t:
//   x0  = (x - sigma_s eps) / alpha_s                 (this step's prediction)
//   D   = x0 + c2 (x0 - x0_prev),   c2 = h / (2 (lambda_s - lambda_prev))
//                                   (c2 = 0: a first-order step)
//   x_t = (sigma_t / sigma_s) x + alpha_t (1 - exp(-h)) D
// and the final step to abar_t = 1 returns x0.  The host folds the schedule
// into five fp32 coefficients (computed in double); per element the kernel
// reads x, eps and x0_prev, and writes x_t and x0 (which the next step reads
// as its x0_prev) -- three fused multiply-adds, HBM-bound.  Elementwise, so
// every band updates its own rows with no context from other bands.
#include <cmath>

#include "dp_common.cuh"
#include "dp_internal.h"

namespace dp {

struct DpmCoef {
  float cx, ce;   // x0 = cx x + ce eps
  float c2;       // D = x0 + c2 (x0 - x0_prev)
  float a, b;     // x_t = a x + b D
};

__device__ __forceinline__ void dpm_one(float x, float e, float xp, const DpmCoef& k, float* xt, float* x0) {
  const float p = fmaf(k.cx, x, k.ce * e);
  // a first-order step ignores x0_prev, whatever the buffer holds
  const float d = k.c2 != 0.f ? fmaf(k.c2, p - xp, p) : p;
  *x0 = p;
  *xt = fmaf(k.a, x, k.b * d);
}

// bf16: 8 elements per 16-byte vector, the ragged tail element by element.
// x_t may be x (in place): each element is read before it is written.
__global__ void __launch_bounds__(256) dpm_bf16_kernel(const __nv_bfloat16* x, const __nv_bfloat16* __restrict__ eps,
                                                       __nv_bfloat16* x0b, __nv_bfloat16* xt, size_t n, DpmCoef k) {
  griddep_wait();
  griddep_trigger();
  const size_t nv = n / 8;
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  const size_t tid = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  for (size_t i = tid; i < nv; i += stride) {
    const uint4 a = reinterpret_cast<const uint4*>(x)[i];
    const uint4 b = reinterpret_cast<const uint4*>(eps)[i];
    const uint4 c = reinterpret_cast<const uint4*>(x0b)[i];
    const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w}, wc[4] = {c.x, c.y, c.z, c.w};
    uint32_t ot[4], o0[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float t0, t1, p0, p1;
      dpm_one(__uint_as_float(wa[q] << 16), __uint_as_float(wb[q] << 16), __uint_as_float(wc[q] << 16), k, &t0, &p0);
      dpm_one(__uint_as_float(wa[q] & 0xffff0000u), __uint_as_float(wb[q] & 0xffff0000u),
              __uint_as_float(wc[q] & 0xffff0000u), k, &t1, &p1);
      ot[q] = pack_bf16x2(t0, t1);
      o0[q] = pack_bf16x2(p0, p1);
    }
    reinterpret_cast<uint4*>(xt)[i] = make_uint4(ot[0], ot[1], ot[2], ot[3]);
    reinterpret_cast<uint4*>(x0b)[i] = make_uint4(o0[0], o0[1], o0[2], o0[3]);
  }
  for (size_t i = nv * 8 + tid; i < n; i += stride) {
    float t, p;
    dpm_one(__bfloat162float(x[i]), __bfloat162float(eps[i]), __bfloat162float(x0b[i]), k, &t, &p);
    xt[i] = __float2bfloat16_rn(t);
    x0b[i] = __float2bfloat16_rn(p);
  }
}

__global__ void __launch_bounds__(256) dpm_f32_kernel(const float* x, const float* __restrict__ eps, float* x0b,
                                                      float* xt, size_t n, DpmCoef k) {
  griddep_wait();
  griddep_trigger();
  const size_t nv = n / 4;
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  const size_t tid = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  for (size_t i = tid; i < nv; i += stride) {
    const float4 a = reinterpret_cast<const float4*>(x)[i];
    const float4 b = reinterpret_cast<const float4*>(eps)[i];
    const float4 c = reinterpret_cast<const float4*>(x0b)[i];
    float4 t, p;
    dpm_one(a.x, b.x, c.x, k, &t.x, &p.x);
    dpm_one(a.y, b.y, c.y, k, &t.y, &p.y);
    dpm_one(a.z, b.z, c.z, k, &t.z, &p.z);
    dpm_one(a.w, b.w, c.w, k, &t.w, &p.w);
    reinterpret_cast<float4*>(xt)[i] = t;
    reinterpret_cast<float4*>(x0b)[i] = p;
  }
  for (size_t i = nv * 4 + tid; i < n; i += stride) dpm_one(x[i], eps[i], x0b[i], k, &xt[i], &x0b[i]);
}

}  // namespace dp

extern "C" {

int dp_dpm_solver_step(const void* x, const void* eps, void* x0_buf, void* x_next, size_t n, double abar_prev,
                       double abar_s, double abar_t, int dtype, void* stream) {
  if (!x || !eps || !x0_buf || !x_next) return dp::set_error(DP_ERR_INVALID_ARG, "dpm: null pointer");
  if (dtype != DP_BF16 && dtype != DP_FP32) return dp::set_error(DP_ERR_INVALID_ARG, "dpm: bad dtype");
  if (!(abar_s > 0.0 && abar_s < 1.0) || !(abar_t > abar_s && abar_t <= 1.0))
    return dp::set_error(DP_ERR_INVALID_ARG, "dpm: need 0 < abar_s < abar_t <= 1");
  if (abar_prev != 0.0 && !(abar_prev > 0.0 && abar_prev < abar_s))
    return dp::set_error(DP_ERR_INVALID_ARG, "dpm: abar_prev must be 0 (first order) or in (0, abar_s)");
  if (!dp::aligned16(x) || !dp::aligned16(eps) || !dp::aligned16(x0_buf) || !dp::aligned16(x_next))
    return dp::set_error(DP_ERR_UNSUPPORTED, "dpm: pointers must be 16-byte aligned");
  const size_t es = dtype == DP_FP32 ? 4 : 2;
  if (n > (static_cast<size_t>(-1) >> 3)) return dp::set_error(DP_ERR_INVALID_ARG, "dpm: n too large");
  const size_t bytes = n * es;
  auto overlap = [&](const void* a, const void* b) {
    const char* pa = static_cast<const char*>(a);
    const char* pb = static_cast<const char*>(b);
    return pa < pb + bytes && pb < pa + bytes;
  };
  if (overlap(x0_buf, x) || overlap(x0_buf, eps) || overlap(x0_buf, x_next) || overlap(x_next, eps))
    return dp::set_error(DP_ERR_INVALID_ARG, "dpm: x0_buf or x_next overlaps another buffer");
  if (x_next != x && overlap(x_next, x))
    return dp::set_error(DP_ERR_INVALID_ARG, "dpm: x_next overlaps x without being x");
  if (n == 0) return DP_OK;
  const double a_s = std::sqrt(abar_s), s_s = std::sqrt(1.0 - abar_s);
  dp::DpmCoef k;
  k.cx = static_cast<float>(1.0 / a_s);
  k.ce = static_cast<float>(-s_s / a_s);
  if (abar_t >= 1.0) {   // the final step: the clean sample, first order
    k.c2 = 0.f;
    k.a = 0.f;
    k.b = 1.f;
  } else {
    const double a_t = std::sqrt(abar_t), s_t = std::sqrt(1.0 - abar_t);
    const double lam_s = std::log(a_s / s_s), lam_t = std::log(a_t / s_t), h = lam_t - lam_s;
    double c2 = 0.0;
    if (abar_prev > 0.0) {
      const double lam_p = std::log(std::sqrt(abar_prev) / std::sqrt(1.0 - abar_prev));
      c2 = h / (2.0 * (lam_s - lam_p));
    }
    k.c2 = static_cast<float>(c2);
    k.a = static_cast<float>(s_t / s_s);
    k.b = static_cast<float>(a_t * -std::expm1(-h));
  }
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  size_t blocks = (n / (16 / es) + 255) / 256;
  const size_t cap = static_cast<size_t>(dp::num_sms()) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks == 0) blocks = 1;
  dp::mark_launch(st);
  if (dtype == DP_FP32)
    return dp::launch_kernel(dp::dpm_f32_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, st, false,
                             "dpm launch", static_cast<const float*>(x), static_cast<const float*>(eps),
                             static_cast<float*>(x0_buf), static_cast<float*>(x_next), n, k);
  return dp::launch_kernel(dp::dpm_bf16_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, st, false,
                           "dpm launch", static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(eps),
                           static_cast<__nv_bfloat16*>(x0_buf), static_cast<__nv_bfloat16*>(x_next), n, k);
}

}  // extern "C"
