// dp_token.cu -- per-token operators of the SDXL-shaped transformer block.
//
// DistriFusion runs SDXL ("DistriFusion", study.space summary, Experiments),
// whose transformer blocks normalise every token with a LayerNorm and end
// with a GELU-gated feed-forward.  Both act on one token at a time, so
// unlike GroupNorm and self-attention they need no context from other bands
// and no stale copy: they run on the fresh tokens of every band alike.
//
//  * layernorm_kernel: one warp per token; the token's C values stay in
//    registers (16-byte vectors, C <= 2048), the mean and then the variance
//    of the deviations come from warp shuffles (two passes over registers, no
//    E[x^2] - E[x]^2 cancellation), and y = (x - mean) rstd gamma + beta is
//    stored as bf16.  HBM-bound: read and write each token once.
//  * geglu_kernel: y = a * gelu(g) for h = [a | g] (two halves of 2F
//    columns), exact GELU through erff; 16-byte vectors.  HBM-bound.
#include <cstring>

#include "dp_common.cuh"
#include "dp_internal.h"

namespace dp {

constexpr int kLnMaxVec = kLnMaxC / (32 * 8);   // 16-byte vectors per lane

template <int NV>
__global__ void __launch_bounds__(256) layernorm_kernel(const __nv_bfloat16* __restrict__ x,
                                                        __nv_bfloat16* __restrict__ y,
                                                        const float* __restrict__ gamma,
                                                        const float* __restrict__ beta, int T,
                                                        int C, float eps) {
  // gamma and beta are weights, never written by the kernel before this one:
  // staged while that kernel finishes, so the token's end needs no memory trip
  __shared__ __align__(16) float sg[kLnMaxC], sb[kLnMaxC];
  for (int c = 4 * threadIdx.x; c < C; c += 4 * blockDim.x) {
    *reinterpret_cast<float4*>(sg + c) = __ldg(reinterpret_cast<const float4*>(gamma + c));
    *reinterpret_cast<float4*>(sb + c) = __ldg(reinterpret_cast<const float4*>(beta + c));
  }
  __syncthreads();
  griddep_wait();
  griddep_trigger();
  const int warp = static_cast<int>((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int lane = lane_id();
  if (warp >= T) return;   // after the block's only barrier
  const int nvec = C / 8;
  const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<size_t>(warp) * C);
  float v[NV][8];
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int e = lane + 32 * i;
    if (e < nvec) {
      const uint4 u = src[e];
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        v[i][2 * k] = __uint_as_float(w[k] << 16);
        v[i][2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
        s += v[i][2 * k] + v[i][2 * k + 1];
      }
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  const float mean = s / C;
  float q = 0.f;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    if (lane + 32 * i < nvec) {
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float d = v[i][k] - mean;
        q = fmaf(d, d, q);
      }
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) q += __shfl_xor_sync(0xffffffffu, q, off);
  const float rstd = rsqrtf(q / C + eps);
  uint4* dst = reinterpret_cast<uint4*>(y + static_cast<size_t>(warp) * C);
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int e = lane + 32 * i;
    if (e < nvec) {
      const float4 g0 = reinterpret_cast<const float4*>(sg)[2 * e];
      const float4 g1 = reinterpret_cast<const float4*>(sg)[2 * e + 1];
      const float4 b0 = reinterpret_cast<const float4*>(sb)[2 * e];
      const float4 b1 = reinterpret_cast<const float4*>(sb)[2 * e + 1];
      const float g[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
      const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
      float o[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) o[k] = fmaf((v[i][k] - mean) * rstd, g[k], b[k]);
      dst[e] = make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]), pack_bf16x2(o[4], o[5]),
                          pack_bf16x2(o[6], o[7]));
    }
  }
}

// IL = false: h's row is [a (F values) | g (F values)].  IL = true: value and
// gate columns interleaved in blocks of 16 (columns 32k..32k+15 are a for
// outputs 16k..16k+15, columns 32k+16..32k+31 the matching g), the layout a
// transformer block's feed-forward projection writes.
template <bool IL>
__global__ void __launch_bounds__(256) geglu_kernel(const __nv_bfloat16* __restrict__ h,
                                                    __nv_bfloat16* __restrict__ y, int T, int F) {
  griddep_wait();
  griddep_trigger();
  const int fv = F / 8;
  const size_t n = static_cast<size_t>(T) * fv;
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t t = i / fv, c = i - t * fv;
    const uint4* row = reinterpret_cast<const uint4*>(h + t * 2 * F);
    // 8 outputs per vector: IL takes the half-block c & 1 of block c / 2
    const uint4 a = IL ? row[4 * (c >> 1) + (c & 1)] : row[c];
    const uint4 g = IL ? row[4 * (c >> 1) + 2 + (c & 1)] : row[fv + c];
    const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wg[4] = {g.x, g.y, g.z, g.w};
    uint32_t o[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float a0 = __uint_as_float(wa[k] << 16), a1 = __uint_as_float(wa[k] & 0xffff0000u);
      const float g0 = __uint_as_float(wg[k] << 16), g1 = __uint_as_float(wg[k] & 0xffff0000u);
      o[k] = pack_bf16x2(a0 * gelu_exact(g0), a1 * gelu_exact(g1));
    }
    reinterpret_cast<uint4*>(y + t * F)[c] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

int geglu_launch(const void* h, void* y, int T, int F, bool interleaved, cudaStream_t st) {
  const size_t n = static_cast<size_t>(T) * (F / 8);
  size_t blocks = (n + 255) / 256;
  const size_t cap = static_cast<size_t>(num_sms()) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks == 0) blocks = 1;
  mark_launch(st);
  const auto* hb = static_cast<const __nv_bfloat16*>(h);
  auto* yb = static_cast<__nv_bfloat16*>(y);
  if (interleaved)
    return launch_kernel(geglu_kernel<true>, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, st, false,
                         "geglu launch", hb, yb, T, F);
  return launch_kernel(geglu_kernel<false>, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, st, false,
                       "geglu launch", hb, yb, T, F);
}

}  // namespace dp

extern "C" {

int dp_layernorm(const void* x, void* y, const float* gamma, const float* beta, int T, int C,
                 float eps, void* stream) {
  if (!x || !y || !gamma || !beta) return dp::set_error(DP_ERR_INVALID_ARG, "layernorm: null pointer");
  if (T <= 0 || C <= 0) return dp::set_error(DP_ERR_INVALID_ARG, "layernorm: bad size");
  if (C % 8 || C > 32 * 8 * dp::kLnMaxVec)
    return dp::set_error(DP_ERR_UNSUPPORTED, "layernorm: C must be a multiple of 8 and at most %d",
                         32 * 8 * dp::kLnMaxVec);
  if (!(eps > 0.f)) return dp::set_error(DP_ERR_INVALID_ARG, "layernorm: eps must be > 0");
  if (!dp::aligned16(x) || !dp::aligned16(y) || !dp::aligned16(gamma) || !dp::aligned16(beta))
    return dp::set_error(DP_ERR_UNSUPPORTED, "layernorm: pointers must be 16-byte aligned");
  {
    // each warp reads its token before writing it, but another warp's rows may be
    // read after this one's are written: y may not overlap x at all
    const char* xb8 = static_cast<const char*>(x);
    const char* yb8 = static_cast<const char*>(y);
    const size_t bytes = static_cast<size_t>(T) * C * 2;
    if (xb8 < yb8 + bytes && yb8 < xb8 + bytes)
      return dp::set_error(DP_ERR_INVALID_ARG, "layernorm: y overlaps x");
  }
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  const unsigned blocks = static_cast<unsigned>((static_cast<long>(T) * 32 + 255) / 256);
  const int nv = (C / 8 + 31) / 32;
  const auto* xb = static_cast<const __nv_bfloat16*>(x);
  auto* yb = static_cast<__nv_bfloat16*>(y);
  dp::mark_launch(st);
  if (nv <= 2)
    return dp::launch_kernel(dp::layernorm_kernel<2>, dim3(blocks), dim3(256), 0, st, false,
                             "layernorm launch", xb, yb, gamma, beta, T, C, eps);
  if (nv <= 4)
    return dp::launch_kernel(dp::layernorm_kernel<4>, dim3(blocks), dim3(256), 0, st, false,
                             "layernorm launch", xb, yb, gamma, beta, T, C, eps);
  return dp::launch_kernel(dp::layernorm_kernel<8>, dim3(blocks), dim3(256), 0, st, false,
                           "layernorm launch", xb, yb, gamma, beta, T, C, eps);
}

int dp_geglu(const void* h, void* y, int T, int F, void* stream) {
  if (!h || !y) return dp::set_error(DP_ERR_INVALID_ARG, "geglu: null pointer");
  if (T <= 0 || F <= 0) return dp::set_error(DP_ERR_INVALID_ARG, "geglu: bad size");
  if (F % 8) return dp::set_error(DP_ERR_UNSUPPORTED, "geglu: F must be a multiple of 8");
  if (!dp::aligned16(h) || !dp::aligned16(y))
    return dp::set_error(DP_ERR_UNSUPPORTED, "geglu: pointers must be 16-byte aligned");
  const char* hb = static_cast<const char*>(h);
  const char* yb = static_cast<const char*>(y);
  const size_t hbytes = static_cast<size_t>(T) * 2 * F * 2, ybytes = static_cast<size_t>(T) * F * 2;
  if (hb < yb + ybytes && yb < hb + hbytes) return dp::set_error(DP_ERR_INVALID_ARG, "geglu: y overlaps h");
  return dp::geglu_launch(h, y, T, F, false, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
