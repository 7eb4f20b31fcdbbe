// dp_conv_small.cu -- direct 3x3 conv for a handful of input channels.
//
// The latent entering a U-Net has 4 channels; a 3x3 conv from it has
// K = 36, too short for a tensor-core tile, so it runs on the CUDA cores.
// Same halo rule as the tensor-core conv ("DistriFusion", study.space
// summary, Method): rows of other bands come from the fresh input (sync), the
// previous step's input (displaced) or nowhere (naive).
//
// Up to 8 input channels: the register kernel below.  Otherwise one thread
// computes 32 consecutive output channels of one pixel; a warp holds
// 32 neighbouring pixels of the same channel group, so every weight it reads
// from shared memory is the same address for all lanes (a broadcast), and its
// input loads are adjacent pixels.  The filter slice of the block's channel
// group sits in shared memory as fp32, laid out [tap][ci][32].
#include "dp_common.cuh"
#include "dp_internal.h"

namespace dp {

constexpr int kSmallCo = 32;   // output channels per thread

__global__ void __launch_bounds__(256) conv3x3_small_kernel(
    const __nv_bfloat16* __restrict__ af, const __nv_bfloat16* __restrict__ as,
    const __nv_bfloat16* __restrict__ w, const float* __restrict__ bias,
    __nv_bfloat16* __restrict__ out, int H, int W, int Cin, int Cout, int hb, int mode) {
  extern __shared__ float sw[];   // [9][Cin][32] for channel group blockIdx.y
  griddep_wait();
  griddep_trigger();
  const int co0 = blockIdx.y * kSmallCo;
  const int nw = 9 * Cin * kSmallCo;
  for (int i = threadIdx.x; i < nw; i += blockDim.x) {
    const int j = i % kSmallCo, k = i / kSmallCo;   // k = tap * Cin + ci
    const int tap = k / Cin, ci = k % Cin;
    sw[i] = __bfloat162float(w[(static_cast<size_t>(co0 + j) * 9 + tap) * Cin + ci]);
  }
  __syncthreads();
  const long pix = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (pix >= static_cast<long>(H) * W) return;
  const int r = static_cast<int>(pix / W), c = static_cast<int>(pix % W);
  const int band = r / hb;
  float acc[kSmallCo];
#pragma unroll
  for (int j = 0; j < kSmallCo; ++j) acc[j] = bias ? __ldg(bias + co0 + j) : 0.f;
  for (int kh = 0; kh < 3; ++kh) {
    const int rho = r + kh - 1;
    if (rho < 0 || rho >= H) continue;
    const __nv_bfloat16* src = af;
    if (rho / hb != band) {
      if (mode == DP_MODE_DISPLACED) src = as;
      else if (mode == DP_MODE_NAIVE) continue;
    }
    for (int kw = 0; kw < 3; ++kw) {
      const int col = c + kw - 1;
      if (col < 0 || col >= W) continue;
      const __nv_bfloat16* px = src + (static_cast<size_t>(rho) * W + col) * Cin;
      const float* wt = sw + (kh * 3 + kw) * Cin * kSmallCo;
      for (int ci = 0; ci < Cin; ++ci) {
        const float v = __bfloat162float(px[ci]);
#pragma unroll
        for (int j = 0; j < kSmallCo; ++j) acc[j] = fmaf(v, wt[ci * kSmallCo + j], acc[j]);
      }
    }
  }
  uint4* dst = reinterpret_cast<uint4*>(out + pix * Cout + co0);
#pragma unroll
  for (int q = 0; q < kSmallCo / 8; ++q) {
    uint4 u;
    u.x = pack_bf16x2(acc[8 * q], acc[8 * q + 1]);
    u.y = pack_bf16x2(acc[8 * q + 2], acc[8 * q + 3]);
    u.z = pack_bf16x2(acc[8 * q + 4], acc[8 * q + 5]);
    u.w = pack_bf16x2(acc[8 * q + 6], acc[8 * q + 7]);
    dst[q] = u;
  }
}

// Register variant for up to 8 input channels (the latent input conv has
// 4): a block takes 64 pixels of one output row; the 3 input rows it needs
// (66 pixels, channels padded to CIN with zeros) are staged in shared memory
// as fp32 with the halo rule applied.  A warp owns a group of 32 output
// channels for the whole tile (a lane owns one channel and keeps its 9 x CIN
// filter taps in registers, loaded once).  It walks the tile 4 pixels at a
// time: per input row it reads the 6 pixels those 4 outputs touch as 16-byte
// shared-memory broadcasts (CIN / 4 vectors each) and does 3 x 4 x CIN FMAs
// per vector read.  A warp's 32 lanes store 32 consecutive channels of one
// pixel.
constexpr int kRegTile = 64;

template <int CIN>
__global__ void __launch_bounds__(320) conv3x3_small_reg_kernel(
    const __nv_bfloat16* __restrict__ af, const __nv_bfloat16* __restrict__ as,
    const __nv_bfloat16* __restrict__ w, const float* __restrict__ bias,
    __nv_bfloat16* __restrict__ out, int H, int W, int Cin, int Cout, int hb, int mode) {
  static_assert(CIN % 4 == 0, "float4 staging");
  constexpr int NV = CIN / 4;
  __shared__ __align__(16) float4 sx[3][kRegTile + 2][NV];
  const int r = blockIdx.y, c0 = blockIdx.x * kRegTile;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
  griddep_wait();
  griddep_trigger();
  const int band = r / hb;
  float* sxf = reinterpret_cast<float*>(sx);
  for (int i = threadIdx.x; i < 3 * (kRegTile + 2) * CIN; i += blockDim.x) {
    const int ci = i % CIN, px = (i / CIN) % (kRegTile + 2), kh = i / (CIN * (kRegTile + 2));
    const int rho = r + kh - 1, col = c0 + px - 1;
    float v = 0.f;
    if (ci < Cin && rho >= 0 && rho < H && col >= 0 && col < W) {
      const __nv_bfloat16* src = af;
      bool use = true;
      if (rho / hb != band) {
        if (mode == DP_MODE_DISPLACED) src = as;
        else if (mode == DP_MODE_NAIVE) use = false;
      }
      if (use) v = __bfloat162float(src[(static_cast<size_t>(rho) * W + col) * Cin + ci]);
    }
    sxf[i] = v;
  }
  __syncthreads();
  const int groups = Cout / 32;
  const int npx = min(kRegTile, W - c0);
  for (int g = warp; g < groups; g += nwarps) {
    const int co = g * 32 + lane;
    float wr[9 * CIN];
    if (Cin == CIN && (reinterpret_cast<uintptr_t>(w) & 7u) == 0) {
      // the lane's 9 x CIN taps are contiguous: 8-byte loads (a quarter of
      // the sectors that 2-byte loads at this lane stride touch)
      const uint2* wv = reinterpret_cast<const uint2*>(w + static_cast<size_t>(co) * 9 * CIN);
#pragma unroll
      for (int i = 0; i < 9 * CIN / 4; ++i) {
        const uint2 u = __ldg(wv + i);
        const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
        const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
        wr[4 * i] = lo.x;
        wr[4 * i + 1] = lo.y;
        wr[4 * i + 2] = hi.x;
        wr[4 * i + 3] = hi.y;
      }
    } else {
#pragma unroll
      for (int k = 0; k < 9; ++k)
#pragma unroll
        for (int ci = 0; ci < CIN; ++ci)
          wr[k * CIN + ci] = ci < Cin ? __bfloat162float(w[(static_cast<size_t>(co) * 9 + k) * Cin + ci]) : 0.f;
    }
    const float b0 = bias ? __ldg(bias + co) : 0.f;
    __nv_bfloat16* orow = out + (static_cast<size_t>(r) * W + c0) * Cout + co;
    for (int px = 0; px < npx; px += 4) {
      float acc[4] = {b0, b0, b0, b0};
#pragma unroll
      for (int kh = 0; kh < 3; ++kh) {
        float4 xv[6][NV];
#pragma unroll
        for (int t = 0; t < 6; ++t)
#pragma unroll
          for (int q = 0; q < NV; ++q) xv[t][q] = sx[kh][px + t][q];
#pragma unroll
        for (int kw = 0; kw < 3; ++kw)
#pragma unroll
          for (int q = 0; q < NV; ++q) {
            const float* wk = wr + (kh * 3 + kw) * CIN + 4 * q;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const float4 x = xv[u + kw][q];
              acc[u] = fmaf(x.x, wk[0], acc[u]);
              acc[u] = fmaf(x.y, wk[1], acc[u]);
              acc[u] = fmaf(x.z, wk[2], acc[u]);
              acc[u] = fmaf(x.w, wk[3], acc[u]);
            }
          }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (px + u < npx) orow[static_cast<size_t>(px + u) * Cout] = __float2bfloat16_rn(acc[u]);
    }
  }
}

int conv3x3_small_launch(const void* af, const void* as, const void* w, const float* bias,
                         void* out, int H, int W, int Cin, int Cout, int P, int mode,
                         cudaStream_t stream) {
  const auto* a0 = static_cast<const __nv_bfloat16*>(af);
  const auto* a1 = static_cast<const __nv_bfloat16*>(as ? as : af);
  const auto* wt = static_cast<const __nv_bfloat16*>(w);
  auto* o = static_cast<__nv_bfloat16*>(out);
  if (Cin <= 8) {
    const dim3 grid(static_cast<unsigned>((W + kRegTile - 1) / kRegTile), static_cast<unsigned>(H));
    mark_launch(stream);
    if (Cin <= 4)
      return launch_kernel(conv3x3_small_reg_kernel<4>, grid, dim3(320), 0, stream, false,
                           "small conv launch", a0, a1, wt, bias, o, H, W, Cin, Cout, H / P, mode);
    return launch_kernel(conv3x3_small_reg_kernel<8>, grid, dim3(320), 0, stream, false,
                         "small conv launch", a0, a1, wt, bias, o, H, W, Cin, Cout, H / P, mode);
  }
  const size_t smem = static_cast<size_t>(9) * Cin * kSmallCo * sizeof(float);
  const dim3 grid(static_cast<unsigned>((static_cast<long>(H) * W + 255) / 256), Cout / kSmallCo);
  mark_launch(stream);
  return launch_kernel(conv3x3_small_kernel, grid, dim3(256), smem, stream, false, "small conv launch",
                       a0, a1, wt, bias, o, H, W, Cin, Cout, H / P, mode);
}

}  // namespace dp

extern "C" int dp_conv3x3_halo_small(const void* a_fresh, const void* a_stale, const void* weight,
                                     const float* bias, void* out, int H, int W, int Cin,
                                     int Cout, int P, int mode, void* stream) {
  if (!a_fresh || !weight || !out) return dp::set_error(DP_ERR_INVALID_ARG, "small conv: null pointer");
  if (H <= 0 || W <= 0 || Cin <= 0 || Cout <= 0 || P <= 0)
    return dp::set_error(DP_ERR_INVALID_ARG, "small conv: non-positive size");
  if (mode < DP_MODE_SYNC || mode > DP_MODE_NAIVE)
    return dp::set_error(DP_ERR_INVALID_ARG, "small conv: bad mode %d", mode);
  if (mode == DP_MODE_DISPLACED && !a_stale)
    return dp::set_error(DP_ERR_INVALID_ARG, "small conv: displaced mode needs the stale buffer");
  if (Cin > 16 || Cout % 32)
    return dp::set_error(DP_ERR_UNSUPPORTED, "small conv: needs Cin <= 16 and Cout %% 32 == 0");
  if (H % P) return dp::set_error(DP_ERR_UNSUPPORTED, "small conv: H %% P != 0");
  if (!dp::aligned16(out)) return dp::set_error(DP_ERR_UNSUPPORTED, "small conv: out not 16-byte aligned");
  if (out == a_fresh || out == a_stale) return dp::set_error(DP_ERR_INVALID_ARG, "small conv: out aliases an input");
  return dp::conv3x3_small_launch(a_fresh, a_stale, weight, bias, out, H, W, Cin, Cout, P, mode,
                                  static_cast<cudaStream_t>(stream));
}
