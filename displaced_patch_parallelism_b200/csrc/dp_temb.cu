// dp_temb.cu -- the time-embedding term of an SDXL-shaped ResBlock.
//
// DistriFusion runs SDXL ("DistriFusion", study.space summary, Experiments).
// An SDXL ResBlock adds a projection of the step's time embedding,
// temb_w silu(temb) + temb_b, to every pixel of its first conv's output.  The
// term is one vector per step, the same for every band, so it needs no stale
// copy: the kernel folds it and the conv's own bias into one fp32 bias vector,
// and the conv's epilogue adds that vector as it adds any bias.
//
//  * temb_bias_kernel: each block stages silu(temb) in shared memory once,
//    then each warp reduces one output channel's row of temb_w (lanes stride
//    the row, so the loads are coalesced) with a shuffle tree.  The kernel
//    reads temb_w once (Cout * Ct * 4 bytes): HBM-bound and a few
//    microseconds at SDXL sizes.
#include "dp_common.cuh"
#include "dp_internal.h"

namespace dp {

constexpr int kTembMaxDim = 8192;   // silu(temb) staged in shared memory: 32 KB at most

__global__ void __launch_bounds__(256) temb_bias_kernel(const float* __restrict__ temb,
                                                        const float* __restrict__ temb_w,
                                                        const float* __restrict__ temb_b,
                                                        const float* __restrict__ conv_b,
                                                        float* __restrict__ bias, int Ct, int Cout) {
  extern __shared__ float s_act[];
  griddep_wait();
  griddep_trigger();
  for (int j = threadIdx.x; j < Ct; j += blockDim.x) {
    const float t = temb[j];
    s_act[j] = t / (1.f + expf(-t));
  }
  __syncthreads();
  const int c = static_cast<int>(blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5));
  const int lane = lane_id();
  if (c >= Cout) return;   // the whole warp leaves together
  const float* row = temb_w + static_cast<size_t>(c) * Ct;
  float s = 0.f;
  for (int j = lane; j < Ct; j += 32) s = fmaf(row[j], s_act[j], s);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if (lane == 0) bias[c] = s + (temb_b ? temb_b[c] : 0.f) + (conv_b ? conv_b[c] : 0.f);
}

int temb_bias_launch(const float* temb, const float* temb_w, const float* temb_b, const float* conv_b,
                     float* bias, int Ct, int Cout, cudaStream_t st) {
  const unsigned blocks = static_cast<unsigned>((Cout + 7) / 8);   // 8 warps, one channel each
  mark_launch(st);
  return launch_kernel(temb_bias_kernel, dim3(blocks), dim3(256), static_cast<size_t>(Ct) * sizeof(float),
                       st, false, "time-embedding bias launch", temb, temb_w, temb_b, conv_b, bias, Ct,
                       Cout);
}

int temb_bias_validate(const void* temb, const void* temb_w, const void* temb_b, const void* conv_b,
                       const void* bias, int Ct, int Cout) {
  if (!temb || !temb_w || !bias) return set_error(DP_ERR_INVALID_ARG, "time embedding: null pointer");
  if (Ct < 1 || Ct > kTembMaxDim || Cout < 1)
    return set_error(DP_ERR_INVALID_ARG, "time embedding: need 1 <= Ct <= %d and Cout >= 1", kTembMaxDim);
  const char* b = static_cast<const char*>(bias);
  const size_t bbytes = static_cast<size_t>(Cout) * sizeof(float);
  auto overlaps = [&](const void* p, size_t bytes) {
    const char* q = static_cast<const char*>(p);
    return p && q < b + bbytes && b < q + bytes;
  };
  if (overlaps(temb, static_cast<size_t>(Ct) * sizeof(float)) ||
      overlaps(temb_w, static_cast<size_t>(Cout) * Ct * sizeof(float)) || overlaps(temb_b, bbytes) ||
      overlaps(conv_b, bbytes))
    return set_error(DP_ERR_INVALID_ARG, "time embedding: bias overlaps an input");
  return DP_OK;
}

}  // namespace dp

extern "C" {

int dp_time_embedding_bias(const float* temb, const float* temb_w, const float* temb_b,
                           const float* conv_b, float* bias, int Ct, int Cout, void* stream) {
  const int rc = dp::temb_bias_validate(temb, temb_w, temb_b, conv_b, bias, Ct, Cout);
  if (rc) return rc;
  return dp::temb_bias_launch(temb, temb_w, temb_b, conv_b, bias, Ct, Cout,
                              static_cast<cudaStream_t>(stream));
}

}  // extern "C"
