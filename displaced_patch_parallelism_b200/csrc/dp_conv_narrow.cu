// dp_conv_narrow.cu -- the stale-halo 3x3 conv to a handful of output
// channels, on the CUDA cores.
//
// A U-Net's last conv maps its 320 channels back to the 4 latent channels:
// N = 4 is far below a tensor-core tile, and at a 128x128 latent the conv is
// 0.4 GFLOP, so it runs as fp32 fused multiply-adds.  Same halo rule as the
// tensor-core conv ("DistriFusion", study.space summary, Method): input row
// rho of another band comes from the fresh input (sync), the previous step's
// input (displaced) or nowhere (naive); outside the image it is zero padding.
//
// A block owns 64 output pixels of one row; its 256 threads are the 64
// pixels x 4 slices of the input channels.  The channels are walked 16 at a
// time: the filter slice [tap][16][CO] goes to shared memory as fp32, and
// slice s of pixel px accumulates channels 4s..4s+3 of the 16 (a warp covers
// 8 pixels x 4 slices, so each tap's load is 8 whole 32-byte pixel rows of
// the chunk).  The four slices' partial sums meet in shared memory at the end.
#include "dp_common.cuh"
#include "dp_internal.h"

namespace dp {

constexpr int kNarrowPx = 64;    // output pixels of a block
constexpr int kNarrowCi = 16;    // input channels staged at a time
constexpr int kNarrowMaxCo = 16;

__device__ __forceinline__ void load4(const __nv_bfloat16* p, float* v) {
  const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
  v[0] = __uint_as_float(u.x << 16);
  v[1] = __uint_as_float(u.x & 0xffff0000u);
  v[2] = __uint_as_float(u.y << 16);
  v[3] = __uint_as_float(u.y & 0xffff0000u);
}
__device__ __forceinline__ void load4(const float* p, float* v) {
  const float4 u = __ldg(reinterpret_cast<const float4*>(p));
  v[0] = u.x;
  v[1] = u.y;
  v[2] = u.z;
  v[3] = u.w;
}
__device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ void from_f(float v, __nv_bfloat16* o) { *o = __float2bfloat16_rn(v); }
__device__ __forceinline__ void from_f(float v, float* o) { *o = v; }

template <typename T, int CO>
__global__ void __launch_bounds__(256) conv3x3_narrow_kernel(
    const T* __restrict__ af, const T* __restrict__ as, const T* __restrict__ w, const float* __restrict__ bias,
    const T* __restrict__ residual, T* __restrict__ out, int H, int W, int Ho, int Wo, int Cin, int Cout,
    int stride, int hb_in, int hb_out, int mode) {
  __shared__ __align__(16) float s_w[9][kNarrowCi][CO];
  __shared__ float s_red[4][kNarrowPx][CO + 1];
  griddep_wait();
  griddep_trigger();
  const int px = threadIdx.x >> 2, slice = threadIdx.x & 3;
  const int r = blockIdx.y, c = blockIdx.x * kNarrowPx + px;
  const int band = r / hb_out;
  // the source of each of the three input rows: fresh, stale or none
  const T* src[3];
#pragma unroll
  for (int kh = 0; kh < 3; ++kh) {
    const int rho = stride * r + kh - 1;
    src[kh] = nullptr;
    if (rho < 0 || rho >= H) continue;
    if (rho / hb_in == band || mode == DP_MODE_SYNC) src[kh] = af + static_cast<size_t>(rho) * W * Cin;
    else if (mode == DP_MODE_DISPLACED) src[kh] = as + static_cast<size_t>(rho) * W * Cin;
  }
  float acc[CO];
#pragma unroll
  for (int j = 0; j < CO; ++j) acc[j] = 0.f;
  for (int ci0 = 0; ci0 < Cin; ci0 += kNarrowCi) {
    // the filter slice: all of a thread's loads issued before its stores
    constexpr int kWIter = (9 * kNarrowCi * CO + 255) / 256;
    float vw[kWIter];
#pragma unroll
    for (int j = 0; j < kWIter; ++j) {
      const int i = threadIdx.x + 256 * j;
      const int co = i % CO, rest = i / CO;
      const int ci = rest % kNarrowCi, tap = rest / kNarrowCi;
      vw[j] = co < Cout && tap < 9 ? to_f(w[(static_cast<size_t>(co) * 9 + tap) * Cin + ci0 + ci]) : 0.f;
    }
#pragma unroll
    for (int j = 0; j < kWIter; ++j) {
      const int i = threadIdx.x + 256 * j;
      const int co = i % CO, rest = i / CO;
      const int ci = rest % kNarrowCi, tap = rest / kNarrowCi;
      if (tap < 9) s_w[tap][ci][co] = vw[j];
    }
    __syncthreads();
    if (c < Wo) {
#pragma unroll
      for (int kh = 0; kh < 3; ++kh) {
        if (!src[kh]) continue;
#pragma unroll
        for (int kw = 0; kw < 3; ++kw) {
          const int col = stride * c + kw - 1;
          if (col < 0 || col >= W) continue;
          float v[4];
          load4(src[kh] + static_cast<size_t>(col) * Cin + ci0 + 4 * slice, v);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float* wr = &s_w[kh * 3 + kw][4 * slice + q][0];
#pragma unroll
            for (int j = 0; j < CO; j += 4) {
              const float4 wq = *reinterpret_cast<const float4*>(wr + j);
              acc[j] = fmaf(v[q], wq.x, acc[j]);
              acc[j + 1] = fmaf(v[q], wq.y, acc[j + 1]);
              acc[j + 2] = fmaf(v[q], wq.z, acc[j + 2]);
              acc[j + 3] = fmaf(v[q], wq.w, acc[j + 3]);
            }
          }
        }
      }
    }
    __syncthreads();   // the next channel slice overwrites the filter staging
  }
#pragma unroll
  for (int j = 0; j < CO; ++j) s_red[slice][px][j] = acc[j];
  __syncthreads();
  // thread t writes output channel t % CO of pixel t / CO (fewer threads than outputs never
  // happens: 64 pixels x CO <= 1024 = 4 passes of 256)
  for (int i = threadIdx.x; i < kNarrowPx * CO; i += blockDim.x) {
    const int p = i / CO, j = i % CO;
    const int cc = blockIdx.x * kNarrowPx + p;
    if (cc >= Wo || j >= Cout) continue;
    float s = s_red[0][p][j] + s_red[1][p][j] + s_red[2][p][j] + s_red[3][p][j];
    if (bias) s += __ldg(bias + j);
    const size_t o = (static_cast<size_t>(r) * Wo + cc) * Cout + j;
    if (residual) s += to_f(residual[o]);
    from_f(s, out + o);
  }
}

template <typename T>
int narrow_launch_t(const void* af, const void* as, const void* w, const float* bias, const void* res, void* out,
                    int H, int W, int Cin, int Cout, int stride, int P, int mode, cudaStream_t st) {
  const int Ho = (H - 1) / stride + 1, Wo = (W - 1) / stride + 1;
  const dim3 grid((Wo + kNarrowPx - 1) / kNarrowPx, Ho);
  const T* a = static_cast<const T*>(af);
  const T* s = static_cast<const T*>(as ? as : af);
  mark_launch(st);
#define DP_NARROW_CASE(CO)                                                                              \
  return launch_kernel(conv3x3_narrow_kernel<T, CO>, grid, dim3(256), 0, st, false, "narrow conv launch", a, s, \
                       static_cast<const T*>(w), bias, static_cast<const T*>(res), static_cast<T*>(out), H, W, \
                       Ho, Wo, Cin, Cout, stride, H / P, Ho / P, mode)
  if (Cout <= 4) DP_NARROW_CASE(4);
  if (Cout <= 8) DP_NARROW_CASE(8);
  DP_NARROW_CASE(16);
#undef DP_NARROW_CASE
}

bool conv3x3_is_narrow(int Cout) { return Cout > 0 && Cout <= kNarrowMaxCo; }

int conv3x3_narrow_launch(const void* a_fresh, const void* a_stale, const void* weight, const float* bias,
                          const void* residual, void* out, int H, int W, int Cin, int Cout, int stride, int P,
                          int mode, int dtype, cudaStream_t stream) {
  if (!conv3x3_is_narrow(Cout) || Cin % kNarrowCi)
    return set_error(DP_ERR_UNSUPPORTED, "narrow conv: needs Cout <= %d and Cin %% %d == 0", kNarrowMaxCo,
                     kNarrowCi);
  if (dtype == DP_FP32)
    return narrow_launch_t<float>(a_fresh, a_stale, weight, bias, residual, out, H, W, Cin, Cout, stride, P,
                                  mode, stream);
  return narrow_launch_t<__nv_bfloat16>(a_fresh, a_stale, weight, bias, residual, out, H, W, Cin, Cout, stride,
                                        P, mode, stream);
}

}  // namespace dp
