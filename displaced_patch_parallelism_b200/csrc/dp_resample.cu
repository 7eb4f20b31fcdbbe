// dp_resample.cu -- the two data movements of a U-Net's up path: channel
// concatenation of the running tensor with a skip connection, and
// nearest-neighbour 2x upsampling.
//
// Both act on each pixel's rows inside its own band (an up-level band is the
// 2x image of the same band one level down), so a displaced step needs no
// context from other bands for them ("DistriFusion", study.space summary,
// Method: only GroupNorm statistics, conv halos and attention keys/values
// cross bands).  Both are pure copies: HBM-bound, 16-byte vectors, a grid
// of a few waves over the SMs walking the output with a grid stride.
#include "dp_common.cuh"
#include "dp_internal.h"

namespace dp {

// out[pix] = [a[pix] (Ca elements) | b[pix] (Cb elements)], in 16-byte vectors
// (va = Ca / vec and vb = Cb / vec vectors per pixel).
__global__ void __launch_bounds__(256) concat_kernel(const uint4* __restrict__ a, const uint4* __restrict__ b,
                                                     uint4* __restrict__ out, size_t npix, int va, int vb) {
  griddep_wait();
  griddep_trigger();
  const int vo = va + vb;
  const size_t n = npix * vo;
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride) {
    const size_t pix = i / vo;
    const int j = static_cast<int>(i - pix * vo);
    out[i] = j < va ? __ldg(a + pix * va + j) : __ldg(b + pix * vb + (j - va));
  }
}

// out[2i + di][2j + dj] = x[i][j]: each thread reads one 16-byte vector of x
// and writes it to the four output pixels it covers.
__global__ void __launch_bounds__(256) upsample2x_kernel(const uint4* __restrict__ x, uint4* __restrict__ out,
                                                         int H, int W, int vc) {
  griddep_wait();
  griddep_trigger();
  const size_t n = static_cast<size_t>(H) * W * vc;
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  const size_t row_out = static_cast<size_t>(2 * W) * vc;   // vectors in one output row
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride) {
    const size_t pix = i / vc;
    const int c = static_cast<int>(i - pix * vc);
    const int r = static_cast<int>(pix / W), col = static_cast<int>(pix - static_cast<size_t>(r) * W);
    const uint4 v = __ldg(x + i);
    uint4* o = out + static_cast<size_t>(2 * r) * row_out + static_cast<size_t>(2 * col) * vc + c;
    o[0] = v;
    o[vc] = v;
    o[row_out] = v;
    o[row_out + vc] = v;
  }
}

unsigned copy_grid(size_t vectors) {
  size_t blocks = (vectors + 255) / 256;
  const size_t cap = static_cast<size_t>(num_sms()) * 8;
  if (blocks > cap) blocks = cap;
  return static_cast<unsigned>(blocks ? blocks : 1);
}

int concat_launch(const void* a, const void* b, void* out, size_t npix, int Ca, int Cb, int dtype,
                  cudaStream_t st) {
  const int vec = dtype == DP_FP32 ? 4 : 8;
  mark_launch(st);
  const size_t nv = npix * ((Ca + Cb) / vec);
  return launch_kernel(concat_kernel, dim3(copy_grid(nv)), dim3(256), 0, st, false, "concat launch",
                       static_cast<const uint4*>(a), static_cast<const uint4*>(b), static_cast<uint4*>(out),
                       npix, Ca / vec, Cb / vec);
}

int upsample2x_launch(const void* x, void* out, int H, int W, int C, int dtype, cudaStream_t st) {
  const int vec = dtype == DP_FP32 ? 4 : 8;
  mark_launch(st);
  const size_t nv = static_cast<size_t>(H) * W * (C / vec);
  return launch_kernel(upsample2x_kernel, dim3(copy_grid(nv)), dim3(256), 0, st, false, "upsample launch",
                       static_cast<const uint4*>(x), static_cast<uint4*>(out), H, W, C / vec);
}

namespace {

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const char* pa = static_cast<const char*>(a);
  const char* pb = static_cast<const char*>(b);
  return pa < pb + nb && pb < pa + na;
}

}  // namespace
}  // namespace dp

extern "C" {

int dp_concat_channels(const void* a, const void* b, void* out, size_t npix, int Ca, int Cb, int dtype,
                       void* stream) {
  if (!a || !b || !out) return dp::set_error(DP_ERR_INVALID_ARG, "concat: null pointer");
  if (dtype != DP_BF16 && dtype != DP_FP32) return dp::set_error(DP_ERR_INVALID_ARG, "concat: bad dtype");
  if (Ca <= 0 || Cb <= 0) return dp::set_error(DP_ERR_INVALID_ARG, "concat: non-positive channels");
  const int vec = dtype == DP_FP32 ? 4 : 8;
  if (Ca % vec || Cb % vec)
    return dp::set_error(DP_ERR_UNSUPPORTED, "concat: channel counts must be multiples of %d", vec);
  if (!dp::aligned16(a) || !dp::aligned16(b) || !dp::aligned16(out))
    return dp::set_error(DP_ERR_UNSUPPORTED, "concat: pointers must be 16-byte aligned");
  if (npix > (static_cast<size_t>(1) << 40)) return dp::set_error(DP_ERR_INVALID_ARG, "concat: npix too large");
  const size_t es = dtype == DP_FP32 ? 4 : 2;
  const size_t oa = npix * Ca * es, ob = npix * Cb * es, oo = npix * (Ca + Cb) * es;
  if (dp::overlaps(out, oo, a, oa) || dp::overlaps(out, oo, b, ob))
    return dp::set_error(DP_ERR_INVALID_ARG, "concat: out overlaps an input");
  if (npix == 0) return DP_OK;
  return dp::concat_launch(a, b, out, npix, Ca, Cb, dtype, static_cast<cudaStream_t>(stream));
}

int dp_upsample_nearest2x(const void* x, void* out, int H, int W, int C, int dtype, void* stream) {
  if (!x || !out) return dp::set_error(DP_ERR_INVALID_ARG, "upsample: null pointer");
  if (dtype != DP_BF16 && dtype != DP_FP32) return dp::set_error(DP_ERR_INVALID_ARG, "upsample: bad dtype");
  if (H <= 0 || W <= 0 || C <= 0) return dp::set_error(DP_ERR_INVALID_ARG, "upsample: non-positive size");
  if (H > (1 << 20) || W > (1 << 20)) return dp::set_error(DP_ERR_INVALID_ARG, "upsample: size too large");
  const int vec = dtype == DP_FP32 ? 4 : 8;
  if (C % vec) return dp::set_error(DP_ERR_UNSUPPORTED, "upsample: C must be a multiple of %d", vec);
  if (!dp::aligned16(x) || !dp::aligned16(out))
    return dp::set_error(DP_ERR_UNSUPPORTED, "upsample: pointers must be 16-byte aligned");
  const size_t es = dtype == DP_FP32 ? 4 : 2;
  const size_t nx = static_cast<size_t>(H) * W * C * es;
  if (dp::overlaps(out, 4 * nx, x, nx)) return dp::set_error(DP_ERR_INVALID_ARG, "upsample: out overlaps x");
  return dp::upsample2x_launch(x, out, H, W, C, dtype, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
