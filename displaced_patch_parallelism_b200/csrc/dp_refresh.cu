// dp_refresh.cu -- the stale-buffer refresh.
//
// In DistriFusion every device AllGathers its fresh activations asynchronously
// so that the next step can use them as stale context ("DistriFusion",
// atlas.scime.ai summary, Approach; its limitations note that the NCCL
// kernels doing so occupy SMs).  With all bands on one GPU the gathered
// result is simply the fresh buffer itself: the block step refreshes by
// flipping a ping-pong pair, and this explicit copy exists for callers that
// keep a single stale buffer per layer.  It is a plain HBM-bound copy with
// 16-byte vectors and enough loads in flight per thread to cover latency.
#include "dp_common.cuh"
#include "dp_internal.h"

namespace dp {

__global__ void __launch_bounds__(256) copy16_kernel(const uint4* __restrict__ src,
                                                     uint4* __restrict__ dst, size_t n16) {
  griddep_wait();
  griddep_trigger();
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  for (; i + 3 * stride < n16; i += 4 * stride) {
    uint4 a = __ldcs(src + i), b = __ldcs(src + i + stride);
    uint4 c = __ldcs(src + i + 2 * stride), d = __ldcs(src + i + 3 * stride);
    dst[i] = a;
    dst[i + stride] = b;
    dst[i + 2 * stride] = c;
    dst[i + 3 * stride] = d;
  }
  for (; i < n16; i += stride) dst[i] = __ldcs(src + i);
}

// Halo refresh: edge e (between bands e and e+1) owns the contiguous rows
// [(e+1) hb - above, (e+1) hb + below); blockIdx.y is the edge, the x blocks
// stride over that range's 16-byte vectors.
__global__ void __launch_bounds__(256) halo_copy_kernel(const uint4* __restrict__ src,
                                                        uint4* __restrict__ dst, size_t edge0_16,
                                                        size_t band16, size_t range16) {
  griddep_wait();
  griddep_trigger();
  const size_t base = edge0_16 + static_cast<size_t>(blockIdx.y) * band16;
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < range16;
       i += static_cast<size_t>(gridDim.x) * blockDim.x)
    dst[base + i] = __ldcs(src + base + i);
}

__global__ void refresh_stats_kernel(const float* __restrict__ fresh_local,
                                     float* __restrict__ stale_local,
                                     float* __restrict__ stale_global, int P, int G) {
  griddep_wait();
  griddep_trigger();
  for (int i = threadIdx.x; i < P * G * 2; i += blockDim.x) stale_local[i] = fresh_local[i];
  for (int i = threadIdx.x; i < G * 2; i += blockDim.x) {
    const int g = i / 2, k = i % 2;
    double s = 0.0;
    for (int p = 0; p < P; ++p) s += fresh_local[(p * G + g) * 2 + k];
    stale_global[i] = static_cast<float>(s / P);
  }
}

int copy_launch(const void* src, void* dst, size_t bytes, cudaStream_t stream) {
  const size_t n16 = bytes / 16;
  if (n16 == 0) return DP_OK;
  size_t blocks = (n16 + 255) / 256;
  const size_t cap = static_cast<size_t>(num_sms()) * 8;
  if (blocks > cap) blocks = cap;
  mark_launch(stream);
  return launch_kernel(copy16_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, stream, false,
                       "refresh launch", static_cast<const uint4*>(src), static_cast<uint4*>(dst), n16);
}

}  // namespace dp

extern "C" {

int dp_refresh_stale(const void* fresh, void* stale, size_t row_bytes, int rows, int P, int band,
                     void* stream) {
  if (!fresh || !stale) return dp::set_error(DP_ERR_INVALID_ARG, "refresh: null buffer");
  if (rows < 0 || P <= 0) return dp::set_error(DP_ERR_INVALID_ARG, "refresh: bad rows/P");
  if (rows % P) return dp::set_error(DP_ERR_UNSUPPORTED, "refresh: rows %% P != 0");
  if (band < -1 || band >= P) return dp::set_error(DP_ERR_INVALID_ARG, "refresh: bad band %d", band);
  if (row_bytes % 16 || !dp::aligned16(fresh) || !dp::aligned16(stale))
    return dp::set_error(DP_ERR_UNSUPPORTED, "refresh: rows and pointers must be 16-byte aligned");
  const size_t band_bytes = row_bytes * static_cast<size_t>(rows / P);
  const size_t total = band == -1 ? band_bytes * P : band_bytes;
  const size_t off = band == -1 ? 0 : band_bytes * band;
  const char* f = static_cast<const char*>(fresh) + off;
  char* s = static_cast<char*>(stale) + off;
  if ((f < s + total) && (s < f + total))
    return dp::set_error(DP_ERR_INVALID_ARG, "refresh: fresh and stale overlap");
  return dp::copy_launch(f, s, total, static_cast<cudaStream_t>(stream));
}

int dp_refresh_halo(const void* fresh, void* stale, size_t row_bytes, int rows, int P, int above,
                    int below, void* stream) {
  if (!fresh || !stale) return dp::set_error(DP_ERR_INVALID_ARG, "refresh_halo: null buffer");
  if (rows < 0 || P <= 0 || above < 0 || below < 0)
    return dp::set_error(DP_ERR_INVALID_ARG, "refresh_halo: bad rows/P/above/below");
  if (rows % P) return dp::set_error(DP_ERR_UNSUPPORTED, "refresh_halo: rows %% P != 0");
  const int hb = rows / P;
  if (above > hb || below > hb)
    return dp::set_error(DP_ERR_INVALID_ARG, "refresh_halo: halo deeper than a band (%d rows)", hb);
  if (row_bytes % 16 || !dp::aligned16(fresh) || !dp::aligned16(stale))
    return dp::set_error(DP_ERR_UNSUPPORTED, "refresh_halo: rows and pointers must be 16-byte aligned");
  const size_t total = row_bytes * static_cast<size_t>(rows);
  const char* f = static_cast<const char*>(fresh);
  char* s = static_cast<char*>(stale);
  if ((f < s + total) && (s < f + total))
    return dp::set_error(DP_ERR_INVALID_ARG, "refresh_halo: fresh and stale overlap");
  if (P == 1 || above + below == 0 || row_bytes == 0) return DP_OK;   // no band edge to refresh
  const size_t row16 = row_bytes / 16;
  const size_t range16 = static_cast<size_t>(above + below) * row16;
  const size_t edge0_16 = (static_cast<size_t>(hb) - above) * row16;
  size_t bx = (range16 + 255) / 256;   // about one vector per thread
  if (bx > 1024) bx = 1024;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  dp::mark_launch(st);
  return dp::launch_kernel(dp::halo_copy_kernel, dim3(static_cast<unsigned>(bx), P - 1), dim3(256), 0,
                           st, false, "refresh_halo launch", static_cast<const uint4*>(fresh),
                           static_cast<uint4*>(stale), edge0_16, static_cast<size_t>(hb) * row16,
                           range16);
}

int dp_refresh_stats(const float* fresh_local, float* stale_local, float* stale_global, int P,
                     int G, void* stream) {
  if (!fresh_local || !stale_local || !stale_global)
    return dp::set_error(DP_ERR_INVALID_ARG, "refresh_stats: null pointer");
  if (P <= 0 || G <= 0) return dp::set_error(DP_ERR_INVALID_ARG, "refresh_stats: bad P/G");
  dp::mark_launch(static_cast<cudaStream_t>(stream));
  return dp::launch_kernel(dp::refresh_stats_kernel, dim3(1), dim3(256), 0,
                           static_cast<cudaStream_t>(stream), false, "refresh_stats launch",
                           fresh_local, stale_local, stale_global, P, G);
}

}  // extern "C"
