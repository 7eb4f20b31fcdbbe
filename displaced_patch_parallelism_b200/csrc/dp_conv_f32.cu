// dp_conv_f32.cu -- the stale-halo 3x3 conv in fp32 on the CUDA cores.
//
// Same operation and halo rule as the bf16 tensor-core conv ("DistriFusion",
// study.space summary, Method): output row r of band p reads input row
// rho = stride*r + kh - 1 from the fresh buffer when it lies in band p,
// otherwise from the fresh buffer (sync), the stale buffer (displaced) or
// nowhere (naive: zeros); outside the image it is zero padding.  Storage and
// arithmetic are fp32 (fp32 fused multiply-adds, no narrower operand format):
// the fp32 workloads state fp32, and at their sizes (tens of MFLOP) latency,
// not the math, sets the time.
//
// A block computes one output row x 32 columns x 16 output channels with 256
// threads.  It walks the input channels 16 at a time: the three input rows
// the row window needs ([kh][ci][column], zero where the halo rule or the
// image edge says so) and the filter slice ([tap][ci][co]) go to shared
// memory, the next slice's loads already in flight into registers.  Thread
// t owns two neighbouring columns (t % 16) x four output channels
// ((t / 16) % 4) and one quarter of each 16-channel slice (t / 64): eight
// independent accumulators, so a thread's fused multiply-adds do not wait on
// one another.  The four quarters' sums meet in shared memory at the end and
// are added in quarter order.
#include "dp_common.cuh"
#include "dp_internal.h"

namespace dp {

constexpr int kF32Px = 32;    // output columns of a block
constexpr int kF32Co = 16;    // output channels of a block
constexpr int kF32Ci = 16;    // input channels staged at a time

__global__ void __launch_bounds__(256) conv3x3_f32_kernel(
    const float* __restrict__ af, const float* __restrict__ as, const float* __restrict__ w,
    const float* __restrict__ bias, const float* __restrict__ residual, float* __restrict__ out,
    int H, int W, int Ho, int Wo, int Cin, int Cout, int stride, int hb_in, int hb_out, int mode) {
  constexpr int kMaxSpan = 2 * (kF32Px - 1) + 3;            // input columns of a window, stride <= 2
  __shared__ float s_in[3][kF32Ci][kMaxSpan + 1];
  __shared__ __align__(16) float s_w[9][kF32Ci][kF32Co];
  __shared__ __align__(16) float s_red[4][kF32Px][kF32Co];   // the quarters' sums
  griddep_wait();
  griddep_trigger();
  const int c0 = blockIdx.x * kF32Px, r = blockIdx.y, co0 = blockIdx.z * kF32Co;
  const int pp = threadIdx.x & 15, cq = (threadIdx.x >> 4) & 3, part = threadIdx.x >> 6;
  const int span = stride * (kF32Px - 1) + 3;
  const int band = r / hb_out;
  // the source of each of the three input rows: fresh, stale or none
  const float* src[3];
  int rows[3];
#pragma unroll
  for (int kh = 0; kh < 3; ++kh) {
    const int rho = stride * r + kh - 1;
    rows[kh] = rho;
    src[kh] = nullptr;
    if (rho < 0 || rho >= H) continue;
    if (rho / hb_in == band || mode == DP_MODE_SYNC) src[kh] = af;
    else if (mode == DP_MODE_DISPLACED) src[kh] = as;
  }
  float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
  constexpr int kInIter = (3 * kMaxSpan * kF32Ci + 255) / 256;   // staging loads per thread
  constexpr int kWIter = 9 * kF32Ci * kF32Co / 256;
  // staging loads of the slice starting at channel ci0 into registers
  float vin[kInIter], vw[kWIter];
  auto load_slice = [&](int ci0) {
#pragma unroll
    for (int j = 0; j < kInIter; ++j) {
      const int i = threadIdx.x + 256 * j;   // consecutive threads: consecutive channels of a pixel
      const int ci = i % kF32Ci, rest = i / kF32Ci;
      const int px = rest % span, kh = rest / span;
      const int col = stride * c0 + px - 1;
      vin[j] = 0.f;
      if (kh < 3 && src[kh] && col >= 0 && col < W)
        vin[j] = __ldg(src[kh] + (static_cast<size_t>(rows[kh]) * W + col) * Cin + ci0 + ci);
    }
#pragma unroll
    for (int j = 0; j < kWIter; ++j) {
      const int i = threadIdx.x + 256 * j;   // filter slice [tap][ci][co] of this block's channels
      const int ci = i % kF32Ci, rest = i / kF32Ci;
      const int tap = rest % 9, co = rest / 9;
      vw[j] = __ldg(w + (static_cast<size_t>(co0 + co) * 9 + tap) * Cin + ci0 + ci);
    }
  };
  load_slice(0);
  for (int ci0 = 0; ci0 < Cin; ci0 += kF32Ci) {
#pragma unroll
    for (int j = 0; j < kInIter; ++j) {
      const int i = threadIdx.x + 256 * j;
      const int ci = i % kF32Ci, rest = i / kF32Ci;
      const int px = rest % span, kh = rest / span;
      if (kh < 3) s_in[kh][ci][px] = vin[j];
    }
#pragma unroll
    for (int j = 0; j < kWIter; ++j) {
      const int i = threadIdx.x + 256 * j;
      const int ci = i % kF32Ci, rest = i / kF32Ci;
      const int tap = rest % 9, co = rest / 9;
      s_w[tap][ci][co] = vw[j];
    }
    // the next slice's loads fly while this one is computed
    if (ci0 + kF32Ci < Cin) load_slice(ci0 + kF32Ci);
    __syncthreads();
#pragma unroll
    for (int kh = 0; kh < 3; ++kh)
#pragma unroll
      for (int kw = 0; kw < 3; ++kw) {
        const int px0 = stride * (2 * pp) + kw, px1 = px0 + stride;
#pragma unroll
        for (int k = 0; k < kF32Ci / 4; ++k) {
          const int ci = 4 * part + k;   // this thread's quarter of the slice
          const float v0 = s_in[kh][ci][px0], v1 = s_in[kh][ci][px1];
          const float4 wq = *reinterpret_cast<const float4*>(&s_w[kh * 3 + kw][ci][4 * cq]);
          acc[0][0] = fmaf(v0, wq.x, acc[0][0]);
          acc[0][1] = fmaf(v0, wq.y, acc[0][1]);
          acc[0][2] = fmaf(v0, wq.z, acc[0][2]);
          acc[0][3] = fmaf(v0, wq.w, acc[0][3]);
          acc[1][0] = fmaf(v1, wq.x, acc[1][0]);
          acc[1][1] = fmaf(v1, wq.y, acc[1][1]);
          acc[1][2] = fmaf(v1, wq.z, acc[1][2]);
          acc[1][3] = fmaf(v1, wq.w, acc[1][3]);
        }
      }
    __syncthreads();   // the next channel slice overwrites the staging
  }
#pragma unroll
  for (int i = 0; i < 2; ++i)
    *reinterpret_cast<float4*>(&s_red[part][2 * pp + i][4 * cq]) =
        make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
  __syncthreads();
  // 32 columns x 16 channels as float4s: threads 0..127 each add the four quarters of one
  for (int t = threadIdx.x; t < kF32Px * kF32Co / 4; t += blockDim.x) {
    const int px = t / (kF32Co / 4), q4 = t % (kF32Co / 4);
    const int c = c0 + px;
    if (c >= Wo) continue;
    float4 s = *reinterpret_cast<const float4*>(&s_red[0][px][4 * q4]);
#pragma unroll
    for (int g = 1; g < 4; ++g) {
      const float4 v = *reinterpret_cast<const float4*>(&s_red[g][px][4 * q4]);
      s.x += v.x;
      s.y += v.y;
      s.z += v.z;
      s.w += v.w;
    }
    const int co = co0 + 4 * q4;
    const size_t o = (static_cast<size_t>(r) * Wo + c) * Cout + co;
    float4 b4 = make_float4(0.f, 0.f, 0.f, 0.f);
    if (bias) b4 = *reinterpret_cast<const float4*>(bias + co);
    float4 res = make_float4(0.f, 0.f, 0.f, 0.f);
    if (residual) res = *reinterpret_cast<const float4*>(residual + o);
    *reinterpret_cast<float4*>(out + o) =
        make_float4(s.x + b4.x + res.x, s.y + b4.y + res.y, s.z + b4.z + res.z, s.w + b4.w + res.w);
  }
}

int conv3x3_f32_launch(const void* a_fresh, const void* a_stale, const void* weight, const float* bias,
                       const void* residual, void* out, int H, int W, int Cin, int Cout, int stride, int P,
                       int mode, cudaStream_t stream) {
  if (Cin % kF32Ci || Cout % kF32Co)
    return set_error(DP_ERR_UNSUPPORTED, "fp32 conv: needs Cin %% %d == 0 and Cout %% %d == 0", kF32Ci,
                     kF32Co);
  if (bias && !aligned16(bias)) return set_error(DP_ERR_UNSUPPORTED, "fp32 conv: bias not 16-byte aligned");
  const int Ho = (H - 1) / stride + 1, Wo = (W - 1) / stride + 1;
  const dim3 grid((Wo + kF32Px - 1) / kF32Px, Ho, Cout / kF32Co);
  mark_launch(stream);
  return launch_kernel(conv3x3_f32_kernel, grid, dim3(256), 0, stream, false, "fp32 conv launch",
                       static_cast<const float*>(a_fresh),
                       static_cast<const float*>(a_stale ? a_stale : a_fresh),
                       static_cast<const float*>(weight), bias, static_cast<const float*>(residual),
                       static_cast<float*>(out), H, W, Ho, Wo, Cin, Cout, stride, H / P, Ho / P, mode);
}

}  // namespace dp
