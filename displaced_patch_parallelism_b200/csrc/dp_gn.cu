// dp_gn.cu -- corrected asynchronous GroupNorm fused with SiLU and the cast.
//
// Method: "DistriFusion: Distributed Parallel Inference for High-Resolution
// Diffusion Models", atlas.scime.ai summary (Approach: a corrected
// asynchronous GroupNorm fixes the statistics; ablation rows: on-device-only
// statistics, stale-only statistics and a synchronous exact pass are the
// alternatives).  Each band normalises with the previous step's whole-image
// moments corrected by the drift of its own fresh moments:
//     used[p][g] = stale_global[g] + w * (fresh_local[p][g] - stale_local[p][g])
// on the raw moments (E[x], E[x^2]).
//
// Two bandwidth-bound kernels:
//  1. gn_stats: per-(band, group) sums of x and x^2.  Every thread keeps one
//     16-byte channel vector of a pixel fixed (block size = a multiple of the
//     vectors per pixel), so it accumulates per-channel sums in registers and
//     never has to split a vector across groups (C/G = 10 at C = 320).  The
//     block folds lanes into channels and channels into groups, then adds
//     its group sums into an fp64 accumulator with atomics; the last block to
//     finish (atomic ticket) turns the sums into the fresh moments and the
//     moments each band uses, and clears the accumulator for the next call.
//  2. gn_apply: y = x * scale_c + shift_c (+ SiLU), cast and stored with
//     16-byte vectors.  Blocks walk the image in the reverse order of the
//     stats pass so that the most recently read part of x is still in L2.
#include <math.h>

#include <mutex>

#include "dp_common.cuh"
#include "dp_internal.h"

namespace dp {

constexpr int kGnMaxSplits = 64;   // blocks per band

template <typename T>
struct Vec;
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ __forceinline__ static void load(const __nv_bfloat16* p, float (&v)[8]) {
    uint4 u = *reinterpret_cast<const uint4*>(p);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 f = __bfloat1622float2(h[i]);
      v[2 * i] = f.x;
      v[2 * i + 1] = f.y;
    }
  }
  __device__ __forceinline__ static void store(__nv_bfloat16* p, const float (&v)[8]) {
    uint4 u;
    u.x = pack_bf16x2(v[0], v[1]);
    u.y = pack_bf16x2(v[2], v[3]);
    u.z = pack_bf16x2(v[4], v[5]);
    u.w = pack_bf16x2(v[6], v[7]);
    *reinterpret_cast<uint4*>(p) = u;
  }
};
template <>
struct Vec<float> {
  static constexpr int N = 4;
  __device__ __forceinline__ static void load(const float* p, float (&v)[4]) {
    float4 u = *reinterpret_cast<const float4*>(p);
    v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w;
  }
  __device__ __forceinline__ static void store(float* p, const float (&v)[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  }
};

struct GnArgs {
  int HWp;      // pixels per band
  int C, G, P;
  int S;        // blocks per band
  int vpp;      // 16-byte vectors per pixel
  int lanes;    // pixel lanes per block (blockDim = vpp * lanes)
  float eps, w;
  int silu, mode;
};

template <typename T>
__global__ void __launch_bounds__(1024) gn_stats_kernel(const T* __restrict__ x, GnArgs a,
                                                        double* __restrict__ acc,
                                                        unsigned* __restrict__ counter,
                                                        const float* __restrict__ stale_global,
                                                        const float* __restrict__ stale_local,
                                                        float* __restrict__ fresh_local,
                                                        float* __restrict__ fresh_global,
                                                        float* __restrict__ used) {
  constexpr int V = Vec<T>::N;
  extern __shared__ __align__(16) unsigned char gn_smem[];
  float* ssum = reinterpret_cast<float*>(gn_smem);           // [lanes][C]
  float* ssq = ssum + a.lanes * a.C;                          // [lanes][C]
  __shared__ int s_last;

  const int p = blockIdx.x / a.S, s = blockIdx.x % a.S;
  const int v = threadIdx.x % a.vpp, pl = threadIdx.x / a.vpp;
  const int chunk = (a.HWp + a.S - 1) / a.S;
  const int beg = s * chunk;
  const int end = min(a.HWp, beg + chunk);
  const T* xb = x + (static_cast<size_t>(p) * a.HWp) * a.C + v * V;

  float sum[V], sq[V];
#pragma unroll
  for (int j = 0; j < V; ++j) sum[j] = sq[j] = 0.f;
  int pix = beg + pl;
  for (; pix + 3 * a.lanes < end; pix += 4 * a.lanes) {
    float t[4][V];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      Vec<T>::load(xb + static_cast<size_t>(pix + u * a.lanes) * a.C, t[u]);
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int j = 0; j < V; ++j) {
        sum[j] += t[u][j];
        sq[j] = fmaf(t[u][j], t[u][j], sq[j]);
      }
  }
  for (; pix < end; pix += a.lanes) {
    float t[V];
    Vec<T>::load(xb + static_cast<size_t>(pix) * a.C, t);
#pragma unroll
    for (int j = 0; j < V; ++j) {
      sum[j] += t[j];
      sq[j] = fmaf(t[j], t[j], sq[j]);
    }
  }
#pragma unroll
  for (int j = 0; j < V; ++j) {
    ssum[pl * a.C + v * V + j] = sum[j];
    ssq[pl * a.C + v * V + j] = sq[j];
  }
  __syncthreads();
  // lanes -> channels (row 0 of the scratch), then channels -> groups
  for (int c = threadIdx.x; c < a.C; c += blockDim.x) {
    float cs = 0.f, cq = 0.f;
    for (int l = 0; l < a.lanes; ++l) {
      cs += ssum[l * a.C + c];
      cq += ssq[l * a.C + c];
    }
    ssum[c] = cs;
    ssq[c] = cq;
  }
  __syncthreads();
  const int cg = a.C / a.G;
  for (int g = threadIdx.x; g < a.G; g += blockDim.x) {
    double ds = 0.0, dq = 0.0;
    for (int c = g * cg; c < (g + 1) * cg; ++c) {
      ds += ssum[c];
      dq += ssq[c];
    }
    atomicAdd(acc + (p * a.G + g) * 2, ds);
    atomicAdd(acc + (p * a.G + g) * 2 + 1, dq);
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = (atomicAdd(counter, 1u) == gridDim.x - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  // Last block: fresh moments, then the moments every band normalises with.
  double* f = reinterpret_cast<double*>(gn_smem);   // [P][G][2]
  const double n = static_cast<double>(a.HWp) * cg;
  for (int i = threadIdx.x; i < a.P * a.G * 2; i += blockDim.x) {
    const double m = __ldcg(acc + i) / n;
    acc[i] = 0.0;                                    // ready for the next call
    f[i] = m;
    fresh_local[i] = static_cast<float>(m);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < a.P * a.G; i += blockDim.x) {
    const int pp = i / a.G, g = i % a.G;
    double gm1 = 0.0, gm2 = 0.0;
    for (int q = 0; q < a.P; ++q) {
      gm1 += f[2 * (q * a.G + g)];
      gm2 += f[2 * (q * a.G + g) + 1];
    }
    gm1 /= a.P;
    gm2 /= a.P;
    double m1, m2;
    if (a.mode == DP_MODE_SYNC) {
      m1 = gm1;
      m2 = gm2;
    } else if (a.mode == DP_MODE_DISPLACED) {
      m1 = static_cast<double>(stale_global[2 * g]) +
           a.w * (f[2 * i] - static_cast<double>(stale_local[2 * i]));
      m2 = static_cast<double>(stale_global[2 * g + 1]) +
           a.w * (f[2 * i + 1] - static_cast<double>(stale_local[2 * i + 1]));
    } else {
      m1 = f[2 * i];
      m2 = f[2 * i + 1];
    }
    double var = m2 - m1 * m1;
    if (var < 0.0) var = f[2 * i + 1] - f[2 * i] * f[2 * i];
    used[2 * i] = static_cast<float>(m1);
    used[2 * i + 1] = static_cast<float>(var);
    if (fresh_global && pp == 0) {
      fresh_global[2 * g] = static_cast<float>(gm1);
      fresh_global[2 * g + 1] = static_cast<float>(gm2);
    }
  }
  if (threadIdx.x == 0) *counter = 0u;  // ready for the next call
}

template <typename T>
__global__ void __launch_bounds__(1024) gn_apply_kernel(const T* __restrict__ x, T* __restrict__ y,
                                                        const float* __restrict__ gamma,
                                                        const float* __restrict__ beta,
                                                        const float* __restrict__ used,
                                                        GnArgs a) {
  constexpr int V = Vec<T>::N;
  extern __shared__ __align__(16) unsigned char gn_smem[];
  float* sscale = reinterpret_cast<float*>(gn_smem);
  float* sshift = sscale + a.C;
  const int b = gridDim.x - 1 - blockIdx.x;   // reverse walk: L2-hot tail first
  const int p = b / a.S, s = b % a.S;
  const int cg = a.C / a.G;
  for (int c = threadIdx.x; c < a.C; c += blockDim.x) {
    const int g = c / cg;
    const float mean = used[2 * (p * a.G + g)];
    const float var = used[2 * (p * a.G + g) + 1];
    const float sc = rsqrtf(var + a.eps) * gamma[c];
    sscale[c] = sc;
    sshift[c] = beta[c] - mean * sc;
  }
  __syncthreads();
  const int v = threadIdx.x % a.vpp, pl = threadIdx.x / a.vpp;
  float sc[V], sh[V];
#pragma unroll
  for (int j = 0; j < V; ++j) {
    sc[j] = sscale[v * V + j];
    sh[j] = sshift[v * V + j];
  }
  const int chunk = (a.HWp + a.S - 1) / a.S;
  const int beg = s * chunk;
  const int end = min(a.HWp, beg + chunk);
  const size_t off = (static_cast<size_t>(p) * a.HWp) * a.C + v * V;
  const T* xb = x + off;
  T* yb = y + off;
  auto body = [&](float (&t)[V]) {
#pragma unroll
    for (int j = 0; j < V; ++j) {
      float z = fmaf(t[j], sc[j], sh[j]);
      if (a.silu) z = __fdividef(z, 1.0f + __expf(-z));
      t[j] = z;
    }
  };
  int pix = beg + pl;
  for (; pix + 3 * a.lanes < end; pix += 4 * a.lanes) {
    float t[4][V];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      Vec<T>::load(xb + static_cast<size_t>(pix + u * a.lanes) * a.C, t[u]);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      body(t[u]);
      Vec<T>::store(yb + static_cast<size_t>(pix + u * a.lanes) * a.C, t[u]);
    }
  }
  for (; pix < end; pix += a.lanes) {
    float t[V];
    Vec<T>::load(xb + static_cast<size_t>(pix) * a.C, t);
    body(t);
    Vec<T>::store(yb + static_cast<size_t>(pix) * a.C, t);
  }
}

static int gn_plan(int H, int W, int C, int G, int P, int dtype, GnArgs* a) {
  const int V = dtype == DP_BF16 ? 8 : 4;
  a->HWp = (H / P) * W;
  a->C = C;
  a->G = G;
  a->P = P;
  a->vpp = C / V;
  a->lanes = a->vpp >= 512 ? 1 : 512 / a->vpp;
  if (a->vpp * a->lanes > 1024) a->lanes = 1024 / a->vpp;
  // One full wave of resident blocks (2 per SM at up to 1024 threads each).
  int s = (2 * num_sms()) / P;
  const int by_work = (a->HWp + 4 * a->lanes - 1) / (4 * a->lanes);
  if (s > by_work) s = by_work;
  if (s > kGnMaxSplits) s = kGnMaxSplits;
  a->S = s < 1 ? 1 : s;
  return DP_OK;
}

static int gn_validate(const void* x, const void* y, int H, int W, int C, int G, int P,
                       int dtype, int mode) {
  if (!x || !y) return set_error(DP_ERR_INVALID_ARG, "groupnorm: null x/y");
  if (H <= 0 || W <= 0 || C <= 0 || G <= 0 || P <= 0)
    return set_error(DP_ERR_INVALID_ARG, "groupnorm: non-positive size");
  if (mode < DP_MODE_SYNC || mode > DP_MODE_NAIVE)
    return set_error(DP_ERR_INVALID_ARG, "groupnorm: bad mode %d", mode);
  if (dtype != DP_BF16 && dtype != DP_FP32)
    return set_error(DP_ERR_INVALID_ARG, "groupnorm: bad dtype %d", dtype);
  if (H % P) return set_error(DP_ERR_UNSUPPORTED, "groupnorm: H %% P != 0");
  if (C % G) return set_error(DP_ERR_UNSUPPORTED, "groupnorm: C %% G != 0");
  const int V = dtype == DP_BF16 ? 8 : 4;
  if (C % V) return set_error(DP_ERR_UNSUPPORTED, "groupnorm: C must be a multiple of %d", V);
  if (C / V > 1024) return set_error(DP_ERR_UNSUPPORTED, "groupnorm: C too large");
  if (P * G > 4096) return set_error(DP_ERR_UNSUPPORTED, "groupnorm: P*G too large");
  if (!aligned16(x) || !aligned16(y)) return set_error(DP_ERR_UNSUPPORTED, "groupnorm: x/y not 16-byte aligned");
  return DP_OK;
}

size_t gn_workspace_bytes(int P, int G) {
  return 256 + static_cast<size_t>(P) * G * 2 * sizeof(double);
}

// Internal entry shared by the ABI call and the block step.
int gn_launch(const void* x, void* y, const float* gamma, const float* beta, int H, int W, int C,
              int G, int P, float eps, float w, int silu, int mode, int dtype,
              const float* stale_global, const float* stale_local, float* fresh_local,
              float* fresh_global, float* used, void* workspace, cudaStream_t stream) {
  GnArgs a;
  gn_plan(H, W, C, G, P, dtype, &a);
  a.eps = eps;
  a.w = w;
  a.silu = silu;
  a.mode = mode;
  unsigned* counter = static_cast<unsigned*>(workspace);
  double* acc = reinterpret_cast<double*>(static_cast<char*>(workspace) + 256);
  const int threads = a.vpp * a.lanes;
  const int blocks = a.P * a.S;
  size_t smem_stats = static_cast<size_t>(a.lanes) * C * 2 * sizeof(float);
  const size_t smem_fin = static_cast<size_t>(P) * G * 2 * sizeof(double);
  if (smem_fin > smem_stats) smem_stats = smem_fin;
  const size_t smem_apply = static_cast<size_t>(C) * 2 * sizeof(float);
  if (smem_stats > 48 * 1024 || smem_apply > 48 * 1024) {
    static bool attr_done[2] = {false, false};
    if (!attr_done[dtype]) {
      if (dtype == DP_BF16) {
        cudaFuncSetAttribute(gn_stats_kernel<__nv_bfloat16>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, 160 * 1024);
        cudaFuncSetAttribute(gn_apply_kernel<__nv_bfloat16>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, 160 * 1024);
      } else {
        cudaFuncSetAttribute(gn_stats_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             160 * 1024);
        cudaFuncSetAttribute(gn_apply_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             160 * 1024);
      }
      attr_done[dtype] = true;
    }
  }
  if (dtype == DP_BF16) {
    mark_launch(stream);
    gn_stats_kernel<__nv_bfloat16><<<blocks, threads, smem_stats, stream>>>(
        static_cast<const __nv_bfloat16*>(x), a, acc, counter, stale_global, stale_local,
        fresh_local, fresh_global, used);
    mark_launch(stream);
    gn_apply_kernel<__nv_bfloat16><<<blocks, threads, smem_apply, stream>>>(
        static_cast<const __nv_bfloat16*>(x), static_cast<__nv_bfloat16*>(y), gamma, beta, used,
        a);
  } else {
    mark_launch(stream);
    gn_stats_kernel<float><<<blocks, threads, smem_stats, stream>>>(
        static_cast<const float*>(x), a, acc, counter, stale_global, stale_local, fresh_local,
        fresh_global, used);
    mark_launch(stream);
    gn_apply_kernel<float><<<blocks, threads, smem_apply, stream>>>(
        static_cast<const float*>(x), static_cast<float*>(y), gamma, beta, used, a);
  }
  return cuda_check(cudaGetLastError(), "groupnorm launch");
}

// ---------------------------------------------------------------------------
// Scratch for callers that cannot allocate device memory.  It is a fixed
// file-scope array that every GPU loading this library holds until the
// process exits.  Host code must not hand the array's name to a kernel: on
// the host that name is only a stand-in, so its device address is looked up
// once per device with cudaGetSymbolAddress and that address is passed on.
constexpr size_t kGnStaticScratchBytes = 32 * 1024;
static __device__ __align__(256) unsigned char g_gn_static_scratch[kGnStaticScratchBytes];

static int gn_static_scratch(void** out) {
  static void* ptrs[64] = {nullptr};
  static std::mutex mu;
  int dev = 0;
  int rc = cuda_check(cudaGetDevice(&dev), "noalloc groupnorm: current device");
  if (rc) return rc;
  if (dev < 0 || dev >= 64) return set_error(DP_ERR_UNSUPPORTED, "noalloc groupnorm: device %d", dev);
  std::lock_guard<std::mutex> lock(mu);
  if (!ptrs[dev]) {
    void* p = nullptr;
    rc = cuda_check(cudaGetSymbolAddress(&p, g_gn_static_scratch),
                    "noalloc groupnorm: scratch address");
    if (rc) return rc;
    ptrs[dev] = p;
  }
  *out = ptrs[dev];
  return DP_OK;
}

}  // namespace dp

extern "C" {

size_t dp_groupnorm_workspace_size(int H, int W, int C, int G, int P) {
  (void)H;
  (void)W;
  (void)C;
  if (P <= 0 || G <= 0) return 0;
  return dp::gn_workspace_bytes(P, G);
}

int dp_groupnorm_async(const void* x, void* y, const float* gamma, const float* beta, int H,
                       int W, int C, int G, int P, float eps, float w, int silu, int mode,
                       int dtype, const float* stale_global, const float* stale_local,
                       float* fresh_local, float* used_stats, void* workspace,
                       size_t workspace_bytes, void* stream) {
  int rc = dp::gn_validate(x, y, H, W, C, G, P, dtype, mode);
  if (rc) return rc;
  if (!gamma || !beta || !fresh_local || !used_stats || !workspace)
    return dp::set_error(DP_ERR_INVALID_ARG, "groupnorm: null gamma/beta/fresh_local/used/workspace");
  if (mode == DP_MODE_DISPLACED && (!stale_global || !stale_local))
    return dp::set_error(DP_ERR_INVALID_ARG, "groupnorm: displaced mode needs stale statistics");
  if (workspace_bytes < dp::gn_workspace_bytes(P, G))
    return dp::set_error(DP_ERR_INVALID_ARG, "groupnorm: workspace too small (%zu < %zu)",
                         workspace_bytes, dp::gn_workspace_bytes(P, G));
  if (!(eps > 0.f)) return dp::set_error(DP_ERR_INVALID_ARG, "groupnorm: eps must be > 0");
  return dp::gn_launch(x, y, gamma, beta, H, W, C, G, P, eps, w, silu, mode, dtype, stale_global,
                       stale_local, fresh_local, nullptr, used_stats, workspace,
                       static_cast<cudaStream_t>(stream));
}

int dp_groupnorm_async_noalloc(const void* x, void* y, const float* gamma, const float* beta,
                               int H, int W, int C, int G, int P, float eps, float w, int silu,
                               int mode, int dtype, const float* stale_global,
                               const float* stale_local, float* fresh_local, float* used_stats,
                               void* stream) {
  int rc = dp::gn_validate(x, y, H, W, C, G, P, dtype, mode);
  if (rc) return rc;
  if (!gamma || !beta || !fresh_local || !used_stats)
    return dp::set_error(DP_ERR_INVALID_ARG, "noalloc groupnorm: null gamma/beta/fresh_local/used");
  if (mode == DP_MODE_DISPLACED && (!stale_global || !stale_local))
    return dp::set_error(DP_ERR_INVALID_ARG, "noalloc groupnorm: displaced mode needs stale statistics");
  if (!(eps > 0.f)) return dp::set_error(DP_ERR_INVALID_ARG, "noalloc groupnorm: eps must be > 0");
  const size_t need = dp::gn_workspace_bytes(P, G);
  if (need > dp::kGnStaticScratchBytes)
    return dp::set_error(DP_ERR_UNSUPPORTED,
                         "noalloc groupnorm: P=%d, G=%d needs %zu bytes of scratch; the static "
                         "scratch holds %zu",
                         P, G, need, dp::kGnStaticScratchBytes);
  void* scratch = nullptr;
  rc = dp::gn_static_scratch(&scratch);
  if (rc) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // The completion ticket and the fp64 accumulator must start at zero; a call
  // that did not complete could have left them elsewhere.
  rc = dp::cuda_check(cudaMemsetAsync(scratch, 0, need, s), "noalloc groupnorm: clear scratch");
  if (rc) return rc;
  return dp::gn_launch(x, y, gamma, beta, H, W, C, G, P, eps, w, silu, mode, dtype, stale_global,
                       stale_local, fresh_local, nullptr, used_stats, scratch, s);
}

}  // extern "C"
