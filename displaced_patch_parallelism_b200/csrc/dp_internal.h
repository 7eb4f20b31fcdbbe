// dp_internal.h -- launchers shared between the library's translation units.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace dp {

// Widest token dp_layernorm takes: a warp holds one token, 8 bf16 per lane
// per 16-byte vector, at most 8 vectors per lane.
constexpr int kLnMaxC = 32 * 8 * 8;

size_t gn_acc_bytes(int P, int G);
size_t gn_workspace_bytes(int P, int G);
bool gn_cluster_plan(int H, int W, int C, int G, int P, int dtype, int mode, int* cpb, int* chunk,
                     int* threads, size_t* smem);
bool gn_fused_plan(int H, int W, int C, int G, int P, int dtype, int* blocks, int* chunk,
                   int* threads, size_t* smem);
int gn_launch(const void* x, void* y, const float* gamma, const float* beta, int H, int W, int C,
              int G, int P, float eps, float w, int silu, int mode, int dtype,
              const float* stale_global, const float* stale_local, float* fresh_local,
              float* fresh_global, float* used, void* workspace, size_t workspace_bytes,
              cudaStream_t stream);
int conv3x3_validate(const void* a_fresh, const void* a_stale, const void* weight,
                     const void* residual, const void* out, int H, int W, int Cin, int Cout,
                     int stride, int P, int mode, int dtype);
size_t gemm_workspace_bytes();
// the 3x3 halo conv in fp32 on the CUDA cores (fp32 storage)
int conv3x3_f32_launch(const void* a_fresh, const void* a_stale, const void* weight, const float* bias,
                       const void* residual, void* out, int H, int W, int Cin, int Cout, int stride, int P,
                       int mode, cudaStream_t stream);
// the 3x3 halo conv to Cout <= 16 channels on the CUDA cores (any storage type)
bool conv3x3_is_narrow(int Cout);
int conv3x3_narrow_launch(const void* a_fresh, const void* a_stale, const void* weight, const float* bias,
                          const void* residual, void* out, int H, int W, int Cin, int Cout, int stride, int P,
                          int mode, int dtype, cudaStream_t stream);
// the up path's copies: channel concatenation and nearest 2x upsampling
int concat_launch(const void* a, const void* b, void* out, size_t npix, int Ca, int Cb, int dtype,
                  cudaStream_t st);
int upsample2x_launch(const void* x, void* out, int H, int W, int C, int dtype, cudaStream_t st);
// GroupNorm statistics alone (the first kernel of the two-kernel path): fresh
// moments, used moments and (if given) the whole-image moments; no apply.
int gn_stats_launch(const void* x, int H, int W, int C, int G, int P, float w, int mode, int dtype,
                    const float* stale_global, const float* stale_local, float* fresh_local,
                    float* fresh_global, float* used, void* workspace, cudaStream_t stream);
// 3x3 conv (stride 1) of GroupNorm(x) (+SiLU), normalised in the conv's
// operand path from the used moments; the band-edge rows of the normalised
// input go to a_next (if not null).  Eligible shapes: conv3x3_gn_eligible.
bool conv3x3_gn_eligible(int H, int W, int Cin, int Cout, int G, int dtype);
int conv3x3_gn_launch(const void* x, const void* a_stale, void* a_next, const float* used,
                      const float* gamma, const float* beta, int G, float eps, int silu,
                      const void* weight, const float* bias, const void* residual, void* out, int H,
                      int W, int Cin, int Cout, int P, int mode, cudaStream_t stream);
// K runs of a conv / projection (1: no split; more: the GEMM is followed by
// the split-K finish kernel).
int conv3x3_splits(int H, int W, int Cin, int Cout, int stride, int dtype, bool can_split);
int linear_splits(int M, int N, int K, int split, bool can_split);
int conv3x3_launch(const void* a_fresh, const void* a_stale, const void* weight,
                   const float* bias, const void* residual, void* out, int H, int W, int Cin,
                   int Cout, int stride, int P, int mode, int dtype, void* workspace,
                   size_t workspace_bytes, cudaStream_t stream);
int linear_launch(const void* x, const void* weight, const float* bias, const void* residual,
                  void* out0, void* out1, void* out2, int M, int N, int K, int split,
                  void* workspace, size_t workspace_bytes, cudaStream_t stream);
int attn_validate(const void* q, const void* kf, const void* vf, const void* ks, const void* vs,
                  const void* o, int T, int heads, int head_dim, int P, int mode);
size_t attn_workspace_bytes();
// bias[c] = conv_b[c] + temb_b[c] + temb_w[c] . silu(temb) (fp32; temb_b and
// conv_b may be null); the validate call checks sizes, nulls and aliasing
int temb_bias_validate(const void* temb, const void* temb_w, const void* temb_b, const void* conv_b,
                       const void* bias, int Ct, int Cout);
int temb_bias_launch(const float* temb, const float* temb_w, const float* temb_b, const float* conv_b,
                     float* bias, int Ct, int Cout, cudaStream_t st);
// attention of T queries over Tk keys (Tk = T: self-attention; with mode SYNC
// and P = 1 and Tk != T: cross-attention over a context every band sees)
int attn_launch_tk(const void* q, const void* kf, const void* vf, const void* ks, const void* vs,
                   void* o, int T, int Tk, int heads, int P, float scale, int mode, void* workspace,
                   size_t workspace_bytes, cudaStream_t stream);
int attn_launch(const void* q, const void* kf, const void* vf, const void* ks, const void* vs,
                void* o, int T, int heads, int P, float scale, int mode, void* workspace,
                size_t workspace_bytes, cudaStream_t stream);
// the feed-forward's projection with the gated GELU in its epilogue (weight and
// bias rows interleaved in blocks of 16), and the stand-alone gated GELU
bool linear_geglu_fusable(int M, int F, int K);
int linear_geglu_launch(const void* x, const void* weight, const float* bias, void* y, int M, int F, int K,
                        cudaStream_t stream);
int geglu_launch(const void* h, void* y, int T, int F, bool interleaved, cudaStream_t st);
void recorder_begin(void* const* events, int n);
int recorder_end();
int copy_launch(const void* src, void* dst, size_t bytes, cudaStream_t stream);

}  // namespace dp
