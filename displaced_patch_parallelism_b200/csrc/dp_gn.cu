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
// Two bandwidth-bound kernels (for tensors too large for the single-pass
// variant further down), one block per SM, each streaming its share of a
// band through a ring of shared-memory buffers filled by bulk copies:
//  1. gn_stats: per-(band, group) sums of x and x^2.  Every thread keeps one
//     16-byte channel vector fixed (block size = a multiple of the vectors per
//     pixel), so it accumulates per-channel sums in registers and never has
//     to split a vector across groups (C/G = 10 at C = 320).  The block folds
//     lanes into channels and channels into groups, then adds its group sums
//     into an fp64 accumulator with atomics; the last block to finish (atomic
//     ticket) turns the sums into the fresh moments and the moments each band
//     uses, and clears the accumulator for the next call.
//  2. gn_apply: y = x * scale_c + shift_c (+ SiLU), cast and stored with
//     coalesced 16-byte vectors.  Blocks walk the image in the reverse order
//     of the stats pass so that the most recently read part of x is still in
//     L2.
#include <math.h>

#include <mutex>

#include "dp_common.cuh"
#include "dp_gn_apply.cuh"
#include "dp_internal.h"

namespace dp {

constexpr int kGnMaxSplits = 64;   // blocks per band
// Each (band, group) accumulator (sum, sum of squares) gets its own 128-byte
// line so that the atomics of many blocks spread over L2 slices instead of
// queueing on the few lines a packed array would occupy.
constexpr int kAccStride = 16;     // doubles between consecutive (band, group) pairs

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

// Per-thread sums of x and x^2 over pixels for one 16-byte channel vector;
// bf16 pairs go through packed fp32x2 adds and fmas.
template <typename T>
struct VecAcc;
template <>
struct VecAcc<__nv_bfloat16> {
  uint64_t s[4] = {0, 0, 0, 0}, q[4] = {0, 0, 0, 0};
  __device__ __forceinline__ void add(const __nv_bfloat16* p) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint64_t x2 = bf16x2_to_f2(w[k]);
      s[k] = f2_add(s[k], x2);
      q[k] = f2_fma(x2, x2, q[k]);
    }
  }
  __device__ __forceinline__ void get(float (&sum)[8], float (&sq)[8]) const {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      f2_unpack(s[k], sum[2 * k], sum[2 * k + 1]);
      f2_unpack(q[k], sq[2 * k], sq[2 * k + 1]);
    }
  }
};
template <>
struct VecAcc<float> {
  float s[4] = {0.f, 0.f, 0.f, 0.f}, q[4] = {0.f, 0.f, 0.f, 0.f};
  __device__ __forceinline__ void add(const float* p) {
    const float4 u = *reinterpret_cast<const float4*>(p);
    const float t[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      s[k] += t[k];
      q[k] = fmaf(t[k], t[k], q[k]);
    }
  }
  __device__ __forceinline__ void get(float (&sum)[4], float (&sq)[4]) const {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      sum[k] = s[k];
      sq[k] = q[k];
    }
  }
};

struct GnArgs {
  int HWp;      // pixels per band
  int C, G, P;
  int S;        // blocks per band
  int vpp;      // 16-byte vectors per pixel
  int lanes;    // pixel lanes per block (blockDim = vpp * lanes)
  int piece;    // pixels per bulk copy (at most 32 KiB)
  float eps, w;
  int silu, mode;
};

// The two-pass kernels stream their share of x through a ring of kGnStages
// shared-memory buffers filled by bulk copies (one block per SM, about
// 128 KiB in flight per SM), so the number of bytes in flight no longer
// depends on how many loads each thread keeps outstanding.
constexpr int kGnStages = 4;
constexpr int kGnPieceBytes = 32768;

// Ring of one block's pixel range [beg, end) of band p.
template <typename T>
struct GnRing {
  T* buf;              // [kGnStages][piece][C]
  uint64_t* full;      // [kGnStages]
  const T* src;        // first pixel of the range
  int n, piece, C;     // pixels in the range, pixels per piece
  __device__ int pieces() const { return (n + piece - 1) / piece; }
  __device__ int count(int k) const { return min(piece, n - k * piece); }
  __device__ T* stage(int k) const { return buf + static_cast<size_t>(k % kGnStages) * piece * C; }
  // thread 0: copy piece k into its stage
  __device__ void issue(int k) const {
    const uint32_t bytes = static_cast<uint32_t>(count(k)) * C * sizeof(T);
    uint64_t* bar = &full[k % kGnStages];
    mbar_arrive_expect_tx(bar, bytes);
    bulk_load(stage(k), src + static_cast<size_t>(k) * piece * C, bytes, bar);
  }
  __device__ bool wait(int k, int* status) const {
    int no_abort = 0;
    return mbar_wait(&full[k % kGnStages], (k / kGnStages) & 1, &no_abort, status);
  }
};

template <typename T>
__global__ void __launch_bounds__(1024) gn_stats_kernel(const T* __restrict__ x, GnArgs a,
                                                        double* __restrict__ acc,
                                                        unsigned* __restrict__ counter,
                                                        const float* __restrict__ stale_global,
                                                        const float* __restrict__ stale_local,
                                                        float* __restrict__ fresh_local,
                                                        float* __restrict__ fresh_global,
                                                        float* __restrict__ used,
                                                        int* __restrict__ status) {
  constexpr int V = Vec<T>::N;
  extern __shared__ __align__(128) unsigned char gn_smem[];
  T* ring = reinterpret_cast<T*>(gn_smem);                     // [kGnStages][piece][C]
  float* ssum = reinterpret_cast<float*>(gn_smem + static_cast<size_t>(kGnStages) * a.piece * a.C * sizeof(T));
  float* ssq = ssum + a.lanes * a.C;                          // [lanes][C]
  __shared__ int s_last;
  __shared__ __align__(8) uint64_t full[kGnStages];

  if (threadIdx.x == 0) {
    for (int i = 0; i < kGnStages; ++i) mbar_init(&full[i], 1);
    fence_mbar_init();
  }
  __syncthreads();
  griddep_wait();
  griddep_trigger();
  const int p = blockIdx.x / a.S, s = blockIdx.x % a.S;
  const int v = threadIdx.x % a.vpp, pl = threadIdx.x / a.vpp;
  const bool worker = threadIdx.x < a.vpp * a.lanes;
  const int chunk = (a.HWp + a.S - 1) / a.S;
  const int beg = min(a.HWp, s * chunk);
  const int end = min(a.HWp, beg + chunk);
  GnRing<T> rg{ring, full, x + (static_cast<size_t>(p) * a.HWp + beg) * a.C, end - beg, a.piece, a.C};
  const int np = rg.pieces();
  if (threadIdx.x == 0)
    for (int k = 0; k < min(np, kGnStages); ++k) rg.issue(k);

  float sum[V], sq[V];
#pragma unroll
  for (int j = 0; j < V; ++j) sum[j] = sq[j] = 0.f;
  VecAcc<T> vacc;
  for (int k = 0; k < np; ++k) {
    rg.wait(k, status);
    const T* st = rg.stage(k) + v * V;
    const int cnt = rg.count(k);
    if (worker) {
      for (int q = pl; q < cnt; q += a.lanes) {
        vacc.add(st + static_cast<size_t>(q) * a.C);
      }
    }
    __syncthreads();   // the stage is free again
    if (threadIdx.x == 0 && k + kGnStages < np) rg.issue(k + kGnStages);
  }
  vacc.get(sum, sq);
  // 16-byte stores: scalar ones at this stride would conflict 8-way
  if (worker) {
#pragma unroll
    for (int j = 0; j < V; j += 4) {
      *reinterpret_cast<float4*>(ssum + pl * a.C + v * V + j) =
          make_float4(sum[j], sum[j + 1], sum[j + 2], sum[j + 3]);
      *reinterpret_cast<float4*>(ssq + pl * a.C + v * V + j) =
          make_float4(sq[j], sq[j + 1], sq[j + 2], sq[j + 3]);
    }
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
    atomicAdd(acc + (p * a.G + g) * kAccStride, ds);
    atomicAdd(acc + (p * a.G + g) * kAccStride + 1, dq);
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
    double* cell = acc + (i >> 1) * kAccStride + (i & 1);
    const double m = __ldcg(cell) / n;
    *cell = 0.0;                                     // ready for the next call
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
                                                        GnArgs a, int* __restrict__ status) {
  constexpr int V = Vec<T>::N;
  extern __shared__ __align__(128) unsigned char gn_smem[];
  T* ring = reinterpret_cast<T*>(gn_smem);                     // [kGnStages][piece][C]
  float* sscale = reinterpret_cast<float*>(gn_smem + static_cast<size_t>(kGnStages) * a.piece * a.C * sizeof(T));
  float* sshift = sscale + a.C;
  __shared__ __align__(8) uint64_t full[kGnStages];
  if (threadIdx.x == 0) {
    for (int i = 0; i < kGnStages; ++i) mbar_init(&full[i], 1);
    fence_mbar_init();
  }
  __syncthreads();
  const int b = gridDim.x - 1 - blockIdx.x;   // reverse walk: L2-hot tail first
  const int p = b / a.S, s = b % a.S;
  const int chunk = (a.HWp + a.S - 1) / a.S;
  const int beg = min(a.HWp, s * chunk);
  const int end = min(a.HWp, beg + chunk);
  const size_t off = (static_cast<size_t>(p) * a.HWp + beg) * a.C;
  GnRing<T> rg{ring, full, x + off, end - beg, a.piece, a.C};
  const int np = rg.pieces();
  // The first pieces of x are fetched before the wait: this kernel always
  // follows the statistics kernel on the stream, which lets it start only
  // after every one of its blocks has passed its own wait, so the kernel that
  // wrote x has completed.  Only the moments (written by the statistics
  // kernel) and y need the wait.
  if (threadIdx.x == 0)
    for (int k = 0; k < min(np, kGnStages); ++k) rg.issue(k);
  griddep_wait();
  griddep_trigger();
  const int cg = a.C / a.G;
  for (int c = threadIdx.x; c < a.C; c += blockDim.x) {
    const int g = c / cg;
    gn_scale_shift(used[2 * (p * a.G + g)], used[2 * (p * a.G + g) + 1], a.eps, gamma[c], beta[c],
                   &sscale[c], &sshift[c]);
  }
  __syncthreads();
  const int v = threadIdx.x % a.vpp, pl = threadIdx.x / a.vpp;
  const bool worker = threadIdx.x < a.vpp * a.lanes;
  float sc[V], sh[V];
#pragma unroll
  for (int j = 0; j < V; ++j) {
    sc[j] = worker ? sscale[v * V + j] : 0.f;
    sh[j] = worker ? sshift[v * V + j] : 0.f;
  }
  const VecApply<T> ap(sc, sh);
  T* yb = y + off + v * V;
  for (int k = 0; k < np; ++k) {
    rg.wait(k, status);
    const T* st = rg.stage(k) + v * V;
    const int cnt = rg.count(k);
    if (worker) {
      T* yk = yb + static_cast<size_t>(k) * a.piece * a.C;
      for (int q = pl; q < cnt; q += a.lanes) {
        ap.run(st + static_cast<size_t>(q) * a.C, yk + static_cast<size_t>(q) * a.C, a.silu);
      }
    }
    __syncthreads();   // the stage is free again
    if (threadIdx.x == 0 && k + kGnStages < np) rg.issue(k + kGnStages);
  }
}

// ---------------------------------------------------------------------------
// Single-pass variant for tensors that fit in the GPU's shared memory: one
// block per SM (cooperative launch, so all blocks are resident), each block
// pulls its contiguous chunk of x into shared memory with bulk copies and
// writes the sums of each (band segment, group) it holds to its own slot of
// a partials array (no atomics: the order of every sum is fixed, so results
// are reproducible).  After a grid barrier every block reduces the partials
// of all bands in fp64, normalises its chunk from shared memory and stores
// it straight to y.  x is read from HBM once and y written once, in one
// launch.
struct GnFusedArgs {
  int HW, HWp, C, G, P, vpp, lanes, chunk;
  float eps, w;
  int silu, mode;
};

// Moments band pp normalises with for group g, from the fresh moments f
// (f[(p*G+g)*2] = E[x], +1 = E[x^2]) of all bands; see the file comment.
__device__ __forceinline__ void gn_used_moments(const double* f, int pp, int g, int P, int G,
                                                int mode, float w, const float* stale_global,
                                                const float* stale_local, double* m_out,
                                                double* var_out, double* gm1_out,
                                                double* gm2_out) {
  const int i = pp * G + g;
  double gm1 = 0.0, gm2 = 0.0;
  for (int q = 0; q < P; ++q) {
    gm1 += f[2 * (q * G + g)];
    gm2 += f[2 * (q * G + g) + 1];
  }
  gm1 /= P;
  gm2 /= P;
  double m1, m2;
  if (mode == DP_MODE_SYNC) {
    m1 = gm1;
    m2 = gm2;
  } else if (mode == DP_MODE_DISPLACED) {
    m1 = static_cast<double>(stale_global[2 * g]) + w * (f[2 * i] - static_cast<double>(stale_local[2 * i]));
    m2 = static_cast<double>(stale_global[2 * g + 1]) +
         w * (f[2 * i + 1] - static_cast<double>(stale_local[2 * i + 1]));
  } else {
    m1 = f[2 * i];
    m2 = f[2 * i + 1];
  }
  double var = m2 - m1 * m1;
  if (var < 0.0) var = f[2 * i + 1] - f[2 * i] * f[2 * i];
  *m_out = m1;
  *var_out = var;
  *gm1_out = gm1;
  *gm2_out = gm2;
}

template <typename T>
__global__ void __launch_bounds__(1024, 1) gn_fused_kernel(
    const T* __restrict__ x, T* __restrict__ y, const float* __restrict__ gamma,
    const float* __restrict__ beta, GnFusedArgs a, float2* __restrict__ part,
    unsigned* __restrict__ bar, const float* __restrict__ stale_global,
    const float* __restrict__ stale_local, float* __restrict__ fresh_local,
    float* __restrict__ fresh_global, float* __restrict__ used, int* __restrict__ status) {
  constexpr int V = Vec<T>::N;
  extern __shared__ __align__(128) unsigned char gn_smem[];
  T* data = reinterpret_cast<T*>(gn_smem);                               // [chunk][C]
  const size_t data_bytes = ((static_cast<size_t>(a.chunk) * a.C * sizeof(T)) + 127) & ~size_t(127);
  float* ssum = reinterpret_cast<float*>(gn_smem + data_bytes);          // [lanes][C]
  float* ssq = ssum + a.lanes * a.C;                                     // [lanes][C]
  double* f = reinterpret_cast<double*>(ssq + a.lanes * a.C);            // [P][G][2]
  float* sscale = reinterpret_cast<float*>(f + a.P * a.G * 2);           // [C]
  float* sshift = sscale + a.C;                                          // [C]
  float* sgamma = sshift + a.C;                                          // [C]
  float* sbeta = sgamma + a.C;                                           // [C]
  float2* stage = reinterpret_cast<float2*>(sbeta + a.C);                // [G][slots]
  __shared__ __align__(8) uint64_t load_bar;
  __shared__ int s_ok;

  const int beg = blockIdx.x * a.chunk;
  const int end = min(a.HW, beg + a.chunk);
  const int npix = max(0, end - beg);
  const int v = threadIdx.x % a.vpp, pl = threadIdx.x / a.vpp;
  const bool worker = threadIdx.x < a.vpp * a.lanes;
  const int cg = a.C / a.G;
  const size_t row_bytes = static_cast<size_t>(a.C) * sizeof(T);

  // ---- phase 1: bulk-load the chunk; gamma and beta meanwhile
  if (threadIdx.x == 0) {
    mbar_init(&load_bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  griddep_wait();
  griddep_trigger();
  if (threadIdx.x == 0 && npix > 0) {
    const uint32_t total = static_cast<uint32_t>(npix * row_bytes);
    mbar_arrive_expect_tx(&load_bar, total);
    const char* src = reinterpret_cast<const char*>(x) + static_cast<size_t>(beg) * row_bytes;
    char* dst = reinterpret_cast<char*>(data);
    for (uint32_t off = 0; off < total; off += 16384u) {
      const uint32_t n = min(16384u, total - off);
      bulk_load(dst + off, src + off, n, &load_bar);
    }
  }
  for (int c = threadIdx.x; c < a.C; c += blockDim.x) {
    sgamma[c] = __ldg(gamma + c);
    sbeta[c] = __ldg(beta + c);
  }
  if (npix > 0) {
    // a load that never lands is recorded in *status; the block still meets
    // the others at the grid barrier so that nobody waits on it
    int no_abort = 0;
    mbar_wait(&load_bar, 0, &no_abort, status);
  }
  __syncthreads();

  // ---- per-(band segment, group) sums of the chunk into this block's slots:
  // the segment of band b in block i is slot i + b (unique, in order)
  for (int b = npix > 0 ? beg / a.HWp : a.P; b < a.P && b * a.HWp < end; ++b) {
    const int lo = max(beg, b * a.HWp) - beg, hi = min(end, (b + 1) * a.HWp) - beg;
    float sum[V], sq[V];
#pragma unroll
    for (int j = 0; j < V; ++j) sum[j] = sq[j] = 0.f;
    VecAcc<T> vacc;
    if (worker) {
      for (int pix = lo + pl; pix < hi; pix += a.lanes) {
        vacc.add(data + static_cast<size_t>(pix) * a.C + v * V);
      }
      vacc.get(sum, sq);
      // 16-byte stores: scalar ones at this stride would conflict 8-way
#pragma unroll
      for (int j = 0; j < V; j += 4) {
        *reinterpret_cast<float4*>(ssum + pl * a.C + v * V + j) =
            make_float4(sum[j], sum[j + 1], sum[j + 2], sum[j + 3]);
        *reinterpret_cast<float4*>(ssq + pl * a.C + v * V + j) =
            make_float4(sq[j], sq[j + 1], sq[j + 2], sq[j + 3]);
      }
    }
    __syncthreads();
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
    for (int g = threadIdx.x; g < a.G; g += blockDim.x) {
      float ds = 0.f, dq = 0.f;
      for (int c = g * cg; c < (g + 1) * cg; ++c) {
        ds += ssum[c];
        dq += ssq[c];
      }
      __stcg(part + static_cast<size_t>(blockIdx.x + b) * a.G + g, make_float2(ds, dq));
    }
    __syncthreads();
  }

  // ---- grid barrier (count, generation), bounded.  The arrival releases
  // this block's partials; the last block opens the barrier by bumping the
  // generation and only then clears the count (the next launch on this
  // workspace starts after this one has finished).
  if (threadIdx.x == 0) {
    s_ok = 1;
    const unsigned my_gen = ld_acquire_gpu(bar + 1);
    if (atom_add_release_gpu(bar, 1u) == gridDim.x - 1) {
      st_release_gpu(bar + 1, my_gen + 1u);
      bar[0] = 0u;
    } else {
      if (!flag_wait_change(bar + 1, my_gen, status, kWaitLimitNs)) s_ok = 0;
    }
  }
  __syncthreads();
  if (!s_ok) return;

  // ---- fresh moments of every band: the partials are staged in shared
  // memory with independent coalesced loads (transposed to [group][slot]),
  // then one thread per (band, group) sums its segments in fp64 in order
  {
    const int nslots = gridDim.x + a.P - 1;
    const int total = nslots * a.G;
#pragma unroll 4
    for (int k = threadIdx.x; k < total; k += blockDim.x) {
      const int slot = k / a.G, g = k - slot * a.G;
      stage[g * nslots + slot] = __ldcg(part + k);
    }
    __syncthreads();
    const double n = static_cast<double>(a.HWp) * cg;
    for (int pg = threadIdx.x; pg < a.P * a.G; pg += blockDim.x) {
      const int b = pg / a.G, g = pg - b * a.G;
      const int i_lo = (b * a.HWp) / a.chunk, i_hi = ((b + 1) * a.HWp - 1) / a.chunk;
      const float2* row = stage + g * nslots + b;
      double s1 = 0.0, s2 = 0.0;
      for (int i = i_lo; i <= i_hi; ++i) {
        const float2 pv = row[i];
        s1 += pv.x;
        s2 += pv.y;
      }
      f[2 * pg] = s1 / n;
      f[2 * pg + 1] = s2 / n;
    }
  }
  __syncthreads();
  if (blockIdx.x == 0) {
    for (int i = threadIdx.x; i < a.P * a.G; i += blockDim.x) {
      double m1, var, gm1, gm2;
      gn_used_moments(f, i / a.G, i % a.G, a.P, a.G, a.mode, a.w, stale_global, stale_local, &m1,
                      &var, &gm1, &gm2);
      used[2 * i] = static_cast<float>(m1);
      used[2 * i + 1] = static_cast<float>(var);
      fresh_local[2 * i] = static_cast<float>(f[2 * i]);
      fresh_local[2 * i + 1] = static_cast<float>(f[2 * i + 1]);
      if (fresh_global && i < a.G) {
        fresh_global[2 * i] = static_cast<float>(gm1);
        fresh_global[2 * i + 1] = static_cast<float>(gm2);
      }
    }
  }

  // ---- apply: normalise from shared memory, store straight to y with
  // coalesced 16-byte stores (consecutive threads, consecutive vectors)
  for (int b = npix > 0 ? beg / a.HWp : a.P; b < a.P && b * a.HWp < end; ++b) {
    const int lo = max(beg, b * a.HWp) - beg, hi = min(end, (b + 1) * a.HWp) - beg;
    for (int c = threadIdx.x; c < a.C; c += blockDim.x) {
      double m1, var, gm1, gm2;
      gn_used_moments(f, b, c / cg, a.P, a.G, a.mode, a.w, stale_global, stale_local, &m1, &var,
                      &gm1, &gm2);
      const float sc = rsqrtf(static_cast<float>(var) + a.eps) * sgamma[c];
      sscale[c] = sc;
      sshift[c] = sbeta[c] - static_cast<float>(m1) * sc;
    }
    __syncthreads();
    if (worker) {
      float sc[V], sh[V];
#pragma unroll
      for (int j = 0; j < V; ++j) {
        sc[j] = sscale[v * V + j];
        sh[j] = sshift[v * V + j];
      }
      const VecApply<T> ap(sc, sh);
      T* yb = y + static_cast<size_t>(beg) * a.C + v * V;
      for (int pix = lo + pl; pix < hi; pix += a.lanes) {
        ap.run(data + static_cast<size_t>(pix) * a.C + v * V, yb + static_cast<size_t>(pix) * a.C, a.silu);
      }
    }
    __syncthreads();   // sscale/sshift are rewritten for the next segment
  }
}

// ---------------------------------------------------------------------------
// Cluster variant for DISPLACED and NAIVE steps, whose bands need only their
// own fresh moments: one thread-block cluster per band (up to 16 CTAs, one
// per SM) holds the band in shared memory.  Each CTA bulk-copies its chunk,
// leaves its (group) sums in shared memory, and after a cluster barrier every
// CTA adds all the cluster's sums through distributed shared memory (in rank
// order, so every CTA gets the same bits).  It normalises its chunk from
// shared memory and stores it.  No grid-wide barrier; the whole-image
// moments (fresh_global) are formed by whichever band finishes last.
struct GnClusterArgs {
  int HWp, C, G, P, vpp, lanes, chunk, cpb;
  int slanes;   // pixel lanes of the statistics pass (lanes: of the apply pass)
  float eps, w;
  int silu, mode;
};

__device__ __forceinline__ float ld_dsmem_f32(uint32_t cluster_addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(cluster_addr) : "memory");
  return v;
}

template <typename T>
__global__ void __launch_bounds__(1024, 1) gn_cluster_kernel(
    const T* __restrict__ x, T* __restrict__ y, const float* __restrict__ gamma,
    const float* __restrict__ beta, GnClusterArgs a, unsigned* __restrict__ ticket,
    const float* __restrict__ stale_global, const float* __restrict__ stale_local,
    float* __restrict__ fresh_local, float* __restrict__ fresh_global, float* __restrict__ used,
    int* __restrict__ status) {
  constexpr int V = Vec<T>::N;
  extern __shared__ __align__(128) unsigned char gn_smem[];
  T* data = reinterpret_cast<T*>(gn_smem);                               // [chunk][C]
  const size_t data_bytes = ((static_cast<size_t>(a.chunk) * a.C * sizeof(T)) + 127) & ~size_t(127);
  float* ssum = reinterpret_cast<float*>(gn_smem + data_bytes);          // [slanes][C]
  float* ssq = ssum + a.slanes * a.C;                                    // [slanes][C]
  float* gpart = ssq + a.slanes * a.C;                                   // [G][2], read by the cluster
  double* f = reinterpret_cast<double*>(gpart + 2 * a.G + (a.G & 1) * 2);  // [G][2]
  float* sscale = reinterpret_cast<float*>(f + 2 * a.G);                 // [C]: gamma, then the scale
  float* sshift = sscale + a.C;                                          // [C]: beta, then the shift
  float* sstale = sshift + a.C;                                          // [G][2] global, [G][2] band
  float* gremote = sstale + 4 * a.G;                                     // [cpb][G][2]: the cluster's sums
  float* gbands = gremote + 2 * a.cpb * a.G;                             // [P][G][2]: every band's moments
  __shared__ __align__(8) uint64_t load_bar;
  __shared__ int s_last;

  const int p = blockIdx.x / a.cpb;
  const int rank = static_cast<int>(cluster_ctarank());
  const int beg = min(a.HWp, rank * a.chunk);
  const int end = min(a.HWp, beg + a.chunk);
  const int npix = end - beg;
  const int v = threadIdx.x % a.vpp, pl = threadIdx.x / a.vpp;
  const bool worker = threadIdx.x < a.vpp * a.lanes;          // apply pass
  const bool sworker = threadIdx.x < a.vpp * a.slanes;        // statistics pass
  const int cg = a.C / a.G;
  const size_t row_bytes = static_cast<size_t>(a.C) * sizeof(T);

  if (threadIdx.x == 0) {
    mbar_init(&load_bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  griddep_wait();
  griddep_trigger();
  if (threadIdx.x == 0 && npix > 0) {
    const uint32_t total = static_cast<uint32_t>(npix * row_bytes);
    mbar_arrive_expect_tx(&load_bar, total);
    const char* src = reinterpret_cast<const char*>(x) + (static_cast<size_t>(p) * a.HWp + beg) * row_bytes;
    char* dst = reinterpret_cast<char*>(data);
    for (uint32_t off = 0; off < total; off += 16384u)
      bulk_load(dst + off, src + off, min(16384u, total - off), &load_bar);
  }
  // while the band arrives: the affine parameters and the stale moments
  for (int c = threadIdx.x; c < a.C; c += blockDim.x) {
    sscale[c] = gamma[c];
    sshift[c] = beta[c];
  }
  if (a.mode == DP_MODE_DISPLACED) {
    for (int i = threadIdx.x; i < 2 * a.G; i += blockDim.x) {
      sstale[i] = stale_global[i];
      sstale[2 * a.G + i] = stale_local[static_cast<size_t>(p) * a.G * 2 + i];
    }
  }
  if (npix > 0) {
    int no_abort = 0;
    mbar_wait(&load_bar, 0, &no_abort, status);
  }
  __syncthreads();

  // ---- this CTA's (group) sums: per-thread channel-vector sums over the
  // thread's pixels (two interleaved accumulators), then lanes -> channels
  // -> groups
  {
    float sum[V], sq[V];
    if (sworker) {
      VecAcc<T> acc0, acc1;
      int pix = pl;
      for (; pix + a.slanes < npix; pix += 2 * a.slanes) {
        acc0.add(data + static_cast<size_t>(pix) * a.C + v * V);
        acc1.add(data + static_cast<size_t>(pix + a.slanes) * a.C + v * V);
      }
      if (pix < npix) acc0.add(data + static_cast<size_t>(pix) * a.C + v * V);
      float s1[V], q1[V];
      acc0.get(sum, sq);
      acc1.get(s1, q1);
#pragma unroll
      for (int j = 0; j < V; ++j) {
        sum[j] += s1[j];
        sq[j] += q1[j];
      }
#pragma unroll
      for (int j = 0; j < V; j += 4) {
        *reinterpret_cast<float4*>(ssum + pl * a.C + v * V + j) =
            make_float4(sum[j], sum[j + 1], sum[j + 2], sum[j + 3]);
        *reinterpret_cast<float4*>(ssq + pl * a.C + v * V + j) =
            make_float4(sq[j], sq[j + 1], sq[j + 2], sq[j + 3]);
      }
    }
  }
  __syncthreads();
  for (int c = threadIdx.x; c < a.C; c += blockDim.x) {
    float cs = 0.f, cq = 0.f;
    for (int l = 0; l < a.slanes; ++l) {
      cs += ssum[l * a.C + c];
      cq += ssq[l * a.C + c];
    }
    ssum[c] = cs;
    ssq[c] = cq;
  }
  __syncthreads();
  for (int g = threadIdx.x; g < a.G; g += blockDim.x) {
    float ds = 0.f, dq = 0.f;
    for (int c = g * cg; c < (g + 1) * cg; ++c) {
      ds += ssum[c];
      dq += ssq[c];
    }
    gpart[2 * g] = ds;
    gpart[2 * g + 1] = dq;
  }
  cluster_sync_all();   // every CTA of the band has its sums in shared memory

  // ---- the band's fresh moments, added over the cluster in rank order: each
  // (rank, moment) is read by its own thread, so the remote reads overlap
  const double n = static_cast<double>(a.HWp) * cg;
  for (int t = threadIdx.x; t < 2 * a.G * a.cpb; t += blockDim.x) {
    const int k = t / (2 * a.G), i = t - k * 2 * a.G;
    gremote[t] = ld_dsmem_f32(mapa_shared(smem_u32(gpart + i), static_cast<uint32_t>(k)));
  }
  __syncthreads();
  // no more reads of other CTAs' shared memory: arrive now, wait at exit
  cluster_arrive();
  for (int i = threadIdx.x; i < 2 * a.G; i += blockDim.x) {
    double s = 0.0;
    for (int k = 0; k < a.cpb; ++k) s += gremote[k * 2 * a.G + i];
    f[i] = s / n;
  }
  __syncthreads();
  for (int c = threadIdx.x; c < a.C; c += blockDim.x) {
    const int g = c / cg;
    double m1 = f[2 * g], m2 = f[2 * g + 1];
    if (a.mode == DP_MODE_DISPLACED) {
      m1 = static_cast<double>(sstale[2 * g]) + a.w * (m1 - static_cast<double>(sstale[2 * a.G + 2 * g]));
      m2 = static_cast<double>(sstale[2 * g + 1]) +
           a.w * (m2 - static_cast<double>(sstale[2 * a.G + 2 * g + 1]));
    }
    double var = m2 - m1 * m1;
    if (var < 0.0) var = f[2 * g + 1] - f[2 * g] * f[2 * g];
    const float sc = rsqrtf(static_cast<float>(var) + a.eps) * sscale[c];
    sshift[c] = sshift[c] - static_cast<float>(m1) * sc;
    sscale[c] = sc;
    if (rank == 0 && c % cg == 0) {
      used[(p * a.G + g) * 2] = static_cast<float>(m1);
      used[(p * a.G + g) * 2 + 1] = static_cast<float>(var);
      fresh_local[(p * a.G + g) * 2] = static_cast<float>(f[2 * g]);
      fresh_local[(p * a.G + g) * 2 + 1] = static_cast<float>(f[2 * g + 1]);
    }
  }
  __syncthreads();

  // ---- apply from shared memory, coalesced 16-byte stores, two pixels per
  // iteration
  if (worker) {
    float sc[V], sh[V];
#pragma unroll
    for (int j = 0; j < V; ++j) {
      sc[j] = sscale[v * V + j];
      sh[j] = sshift[v * V + j];
    }
    const VecApply<T> ap(sc, sh);
    T* yb = y + (static_cast<size_t>(p) * a.HWp + beg) * a.C + v * V;
    int pix = pl;
    for (; pix + a.lanes < npix; pix += 2 * a.lanes) {
      ap.run(data + static_cast<size_t>(pix) * a.C + v * V, yb + static_cast<size_t>(pix) * a.C, a.silu);
      ap.run(data + static_cast<size_t>(pix + a.lanes) * a.C + v * V,
             yb + static_cast<size_t>(pix + a.lanes) * a.C, a.silu);
    }
    if (pix < npix)
      ap.run(data + static_cast<size_t>(pix) * a.C + v * V, yb + static_cast<size_t>(pix) * a.C, a.silu);
  }
  // the cluster's other CTAs are done reading gpart before this CTA leaves
  cluster_wait();

  // ---- the band that finishes last forms the whole-image moments
  if (rank == 0 && fresh_global) {
    if (threadIdx.x == 0) {
      __threadfence();
      s_last = atomicAdd(ticket, 1u) == static_cast<unsigned>(a.P - 1);
    }
    __syncthreads();
    if (s_last) {
      __threadfence();
      // every band's moments read by their own threads, then added in band order
      for (int t = threadIdx.x; t < 2 * a.G * a.P; t += blockDim.x) gbands[t] = __ldcg(fresh_local + t);
      __syncthreads();
      for (int i = threadIdx.x; i < 2 * a.G; i += blockDim.x) {
        double s = 0.0;
        for (int q = 0; q < a.P; ++q) s += gbands[q * a.G * 2 + i];
        fresh_global[i] = static_cast<float>(s / a.P);
      }
      if (threadIdx.x == 0) *ticket = 0u;
    }
  }
}

static int gn_plan(int H, int W, int C, int G, int P, int dtype, GnArgs* a) {
  const int V = dtype == DP_BF16 ? 8 : 4;
  const int row_bytes = C * (dtype == DP_BF16 ? 2 : 4);
  a->HWp = (H / P) * W;
  a->C = C;
  a->G = G;
  a->P = P;
  a->vpp = C / V;
  a->lanes = a->vpp >= 1024 ? 1 : 1024 / a->vpp;
  // one block per SM, the SMs shared out among the bands
  int s = num_sms() / P;
  if (s > kGnMaxSplits) s = kGnMaxSplits;
  a->S = s < 1 ? 1 : s;
  const int chunk = (a->HWp + a->S - 1) / a->S;
  int piece = kGnPieceBytes / row_bytes;
  if (piece > chunk) piece = chunk;
  a->piece = piece < 1 ? 1 : piece;
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

// Workspace: [0, 256) completion ticket and grid-barrier words, then the
// fp64 accumulator of the two-kernel path (its size is gn_acc_bytes; both
// are left zero by every call that completes), then the fp32 partial sums
// of the single-pass path (one (sum, sum of squares) pair per group for each
// of at most kGnFusedMaxBlocks + P band segments; no initialisation needed).
constexpr int kGnFusedMaxBlocks = 160;

size_t gn_acc_bytes(int P, int G) {
  return 256 + static_cast<size_t>(P) * G * kAccStride * sizeof(double);
}

static size_t gn_partial_bytes(int P, int G) {
  return static_cast<size_t>(kGnFusedMaxBlocks + P) * G * sizeof(float2);
}

size_t gn_workspace_bytes(int P, int G) { return gn_acc_bytes(P, G) + gn_partial_bytes(P, G); }

// Plan of the single-pass variant: blocks, chunk and shared memory; false if
// the tensor does not fit.  Shared with the launch counter of the block step.
bool gn_fused_plan(int H, int W, int C, int G, int P, int dtype, int* blocks, int* chunk,
                   int* threads, size_t* smem) {
  const int e = dtype == DP_BF16 ? 2 : 4;
  const int V = 16 / e;
  const int vpp = C / V;
  if (vpp > 1024) return false;
  const int lanes = 1024 / vpp;
  const long HW = static_cast<long>(H) * W;
  const int nb = std::min(num_sms(), kGnFusedMaxBlocks);
  const long ch = (HW + nb - 1) / nb;
  const size_t data = ((static_cast<size_t>(ch) * C * e) + 127) & ~size_t(127);
  const size_t need = data + static_cast<size_t>(lanes) * C * 8 + static_cast<size_t>(P) * G * 16 +
                      static_cast<size_t>(C) * 16 + static_cast<size_t>(nb + P) * G * 8;
  if (need > 200 * 1024) return false;
  *blocks = static_cast<int>((HW + ch - 1) / ch);
  *chunk = static_cast<int>(ch);
  *threads = ((vpp * lanes + 31) / 32) * 32;
  *smem = need;
  return true;
}

// Plan of the cluster variant: CTAs per band (the cluster size), pixels per
// CTA and shared memory; false for SYNC steps (they need every band's
// moments) and when a band does not fit in 16 CTAs' shared memory.
bool gn_cluster_plan(int H, int W, int C, int G, int P, int dtype, int mode, int* cpb, int* chunk,
                     int* threads, size_t* smem) {
  if (mode == DP_MODE_SYNC) return false;
  const int e = dtype == DP_BF16 ? 2 : 4;
  const int vpp = C / (16 / e);
  if (vpp > 512) return false;
  const int lanes = 1024 / vpp;          // apply pass: up to 1024 threads
  const int slanes = 512 / vpp;          // statistics pass: its lane sums stay small
  const long HWp = static_cast<long>(H / P) * W;
  const int n = static_cast<int>(HWp < 16 ? HWp : 16);
  if (n < 1) return false;
  const long ch = (HWp + n - 1) / n;
  const size_t data = ((static_cast<size_t>(ch) * C * e) + 127) & ~size_t(127);
  const size_t need = data + static_cast<size_t>(slanes) * C * 8 + static_cast<size_t>(G) * 8 + 16 +
                      static_cast<size_t>(G) * 16 + static_cast<size_t>(C) * 8 +
                      static_cast<size_t>(G) * 16 + static_cast<size_t>(n + P) * G * 8;
  if (need > 220 * 1024) return false;
  *cpb = n;
  *chunk = static_cast<int>(ch);
  *threads = ((vpp * lanes + 31) / 32) * 32;
  *smem = need;
  return true;
}

// Launches the cluster variant when it applies; false leaves the choice to
// the other variants (*rc untouched).
static bool gn_cluster_launch(const void* x, void* y, const float* gamma, const float* beta, int H,
                              int W, int C, int G, int P, float eps, float w, int silu, int mode,
                              int dtype, const float* stale_global, const float* stale_local,
                              float* fresh_local, float* fresh_global, float* used, unsigned* ticket,
                              cudaStream_t stream, int* rc) {
  int cpb, chunk, threads;
  size_t smem;
  if (!gn_cluster_plan(H, W, C, G, P, dtype, mode, &cpb, &chunk, &threads, &smem)) return false;
  const void* fn = dtype == DP_BF16 ? reinterpret_cast<const void*>(gn_cluster_kernel<__nv_bfloat16>)
                                    : reinterpret_cast<const void*>(gn_cluster_kernel<float>);
  static size_t attr_set[2][32] = {};
  static int usable[2][32] = {};   // 0 unknown, 1 yes, -1 no
  int dev = 0;
  cudaGetDevice(&dev);
  if (usable[dtype][dev & 31] < 0) return false;
  if (smem > attr_set[dtype][dev & 31]) {
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
            cudaSuccess ||
        cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
      cudaGetLastError();
      usable[dtype][dev & 31] = -1;
      return false;
    }
    attr_set[dtype][dev & 31] = smem;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(P * cpb);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cpb;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  int na = 1;
  if (pdl_enabled()) {
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    na = 2;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  if (usable[dtype][dev & 31] == 0) {
    int clusters = 0;
    const cudaError_t e = cudaOccupancyMaxActiveClusters(&clusters, fn, &cfg);
    if (e != cudaSuccess || clusters < 1) {
      cudaGetLastError();
      usable[dtype][dev & 31] = -1;
      return false;
    }
    usable[dtype][dev & 31] = 1;
  }
  GnClusterArgs a;
  a.HWp = (H / P) * W;
  a.C = C;
  a.G = G;
  a.P = P;
  a.vpp = C / (dtype == DP_BF16 ? 8 : 4);
  a.lanes = 1024 / a.vpp;
  a.slanes = 512 / a.vpp;
  a.chunk = chunk;
  a.cpb = cpb;
  a.eps = eps;
  a.w = w;
  a.silu = silu;
  a.mode = mode;
  int* status = device_status_ptr();
  void* args[] = {const_cast<void**>(&x), &y, const_cast<float**>(&gamma), const_cast<float**>(&beta),
                  &a, &ticket, const_cast<float**>(&stale_global), const_cast<float**>(&stale_local),
                  &fresh_local, &fresh_global, &used, &status};
  mark_launch(stream);
  *rc = cuda_check(cudaLaunchKernelExC(&cfg, fn, args), "cluster groupnorm launch");
  return true;
}

// Launches the single-pass variant if the tensor fits; returns false (and
// leaves *rc untouched) when the two-kernel path must be used.
static bool gn_fused_launch(const void* x, void* y, const float* gamma, const float* beta, int H,
                            int W, int C, int G, int P, float eps, float w, int silu, int mode,
                            int dtype, const float* stale_global, const float* stale_local,
                            float* fresh_local, float* fresh_global, float* used, float2* part,
                            unsigned* bar, cudaStream_t stream, int* rc) {
  int blocks, chunk, threads;
  size_t smem;
  if (!gn_fused_plan(H, W, C, G, P, dtype, &blocks, &chunk, &threads, &smem)) return false;
  static int attr_mask[2] = {0, 0};
  int dev = 0;
  cudaGetDevice(&dev);
  const void* fn = dtype == DP_BF16 ? reinterpret_cast<const void*>(gn_fused_kernel<__nv_bfloat16>)
                                    : reinterpret_cast<const void*>(gn_fused_kernel<float>);
  if (!(attr_mask[dtype] & (1 << (dev & 31)))) {
    *rc = cuda_check(cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024),
                     "fused groupnorm smem attribute");
    if (*rc) return true;
    attr_mask[dtype] |= 1 << (dev & 31);
  }
  GnFusedArgs a;
  a.HW = H * W;
  a.HWp = (H / P) * W;
  a.C = C;
  a.G = G;
  a.P = P;
  a.vpp = C / (dtype == DP_BF16 ? 8 : 4);
  a.lanes = 1024 / a.vpp;
  a.chunk = chunk;
  a.eps = eps;
  a.w = w;
  a.silu = silu;
  a.mode = mode;
  int* status = device_status_ptr();
  void* args[] = {const_cast<void**>(&x), &y, const_cast<float**>(&gamma), const_cast<float**>(&beta),
                  &a, &part, &bar, const_cast<float**>(&stale_global), const_cast<float**>(&stale_local),
                  &fresh_local, &fresh_global, &used, &status};
  mark_launch(stream);
  // cooperative (the grid barrier needs every block resident) and, when the
  // driver takes both attributes, a dependent launch
  static int pdl_ok = -1;
  if (pdl_enabled() && pdl_ok != 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(blocks);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeCooperative;
    attr[1].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    const cudaError_t e = cudaLaunchKernelExC(&cfg, fn, args);
    if (e == cudaSuccess) {
      pdl_ok = 1;
      *rc = DP_OK;
      return true;
    }
    cudaGetLastError();
    pdl_ok = 0;
  }
  *rc = cuda_check(cudaLaunchCooperativeKernel(fn, dim3(blocks), dim3(threads), args, smem, stream),
                   "fused groupnorm launch");
  return true;
}

// Shared memory of the two-kernel path's kernels, with the opt-in above
// 48 KiB set (kept per dtype and device at the largest size so far).
static int gn_two_pass_setup(const GnArgs& a, int C, int G, int P, int dtype, size_t* smem_stats,
                             size_t* smem_apply) {
  const size_t ring = static_cast<size_t>(kGnStages) * a.piece * C * (dtype == DP_BF16 ? 2 : 4);
  size_t red = static_cast<size_t>(a.lanes) * C * 2 * sizeof(float);
  const size_t fin = static_cast<size_t>(P) * G * 2 * sizeof(double);
  if (fin > ring + red) red = fin - ring;
  *smem_stats = ring + red;
  *smem_apply = ring + static_cast<size_t>(C) * 2 * sizeof(float);
  if (*smem_stats > 220 * 1024 || *smem_apply > 220 * 1024)
    return set_error(DP_ERR_UNSUPPORTED, "groupnorm: C = %d needs too much shared memory", C);
  static size_t attr_set[2][32] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  size_t& done = attr_set[dtype][dev & 31];
  const size_t need = *smem_stats > *smem_apply ? *smem_stats : *smem_apply;
  if (need > done) {
    const int lim = static_cast<int>(need);
    int rc = 0;
    if (dtype == DP_BF16) {
      rc = cuda_check(cudaFuncSetAttribute(gn_stats_kernel<__nv_bfloat16>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, lim),
                      "groupnorm stats smem attribute");
      if (!rc)
        rc = cuda_check(cudaFuncSetAttribute(gn_apply_kernel<__nv_bfloat16>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, lim),
                        "groupnorm apply smem attribute");
    } else {
      rc = cuda_check(cudaFuncSetAttribute(gn_stats_kernel<float>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, lim),
                      "groupnorm stats smem attribute");
      if (!rc)
        rc = cuda_check(cudaFuncSetAttribute(gn_apply_kernel<float>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, lim),
                        "groupnorm apply smem attribute");
    }
    if (rc) return rc;
    done = need;
  }
  return DP_OK;
}

int gn_stats_launch(const void* x, int H, int W, int C, int G, int P, float w, int mode, int dtype,
                    const float* stale_global, const float* stale_local, float* fresh_local,
                    float* fresh_global, float* used, void* workspace, cudaStream_t stream) {
  GnArgs a;
  gn_plan(H, W, C, G, P, dtype, &a);
  a.eps = 1.0f;   // unused by the statistics pass
  a.w = w;
  a.silu = 0;
  a.mode = mode;
  size_t smem_stats = 0, smem_apply = 0;
  int rc = gn_two_pass_setup(a, C, G, P, dtype, &smem_stats, &smem_apply);
  if (rc) return rc;
  unsigned* counter = static_cast<unsigned*>(workspace);
  double* acc = reinterpret_cast<double*>(static_cast<char*>(workspace) + 256);
  int* status = device_status_ptr();
  mark_launch(stream);
  if (dtype == DP_BF16)
    return launch_kernel(gn_stats_kernel<__nv_bfloat16>, dim3(a.P * a.S), dim3(a.vpp * a.lanes),
                         smem_stats, stream, false, "groupnorm stats launch",
                         static_cast<const __nv_bfloat16*>(x), a, acc, counter, stale_global, stale_local,
                         fresh_local, fresh_global, used, status);
  return launch_kernel(gn_stats_kernel<float>, dim3(a.P * a.S), dim3(a.vpp * a.lanes), smem_stats, stream,
                       false, "groupnorm stats launch", static_cast<const float*>(x), a, acc, counter,
                       stale_global, stale_local, fresh_local, fresh_global, used, status);
}

// Internal entry shared by the ABI call and the block step.
int gn_launch(const void* x, void* y, const float* gamma, const float* beta, int H, int W, int C,
              int G, int P, float eps, float w, int silu, int mode, int dtype,
              const float* stale_global, const float* stale_local, float* fresh_local,
              float* fresh_global, float* used, void* workspace, size_t workspace_bytes,
              cudaStream_t stream) {
  GnArgs a;
  gn_plan(H, W, C, G, P, dtype, &a);
  a.eps = eps;
  a.w = w;
  a.silu = silu;
  a.mode = mode;
  unsigned* counter = static_cast<unsigned*>(workspace);
  double* acc = reinterpret_cast<double*>(static_cast<char*>(workspace) + 256);
  {
    int rc = 0;
    if (gn_cluster_launch(x, y, gamma, beta, H, W, C, G, P, eps, w, silu, mode, dtype, stale_global,
                          stale_local, fresh_local, fresh_global, used, counter, stream, &rc))
      return rc;
    float2* part = reinterpret_cast<float2*>(static_cast<char*>(workspace) + gn_acc_bytes(P, G));
    if (workspace_bytes >= gn_workspace_bytes(P, G) &&
        gn_fused_launch(x, y, gamma, beta, H, W, C, G, P, eps, w, silu, mode, dtype, stale_global,
                        stale_local, fresh_local, fresh_global, used, part, counter + 4, stream,
                        &rc))
      return rc;
  }
  size_t smem_stats = 0, smem_apply = 0;
  int rc0 = gn_two_pass_setup(a, C, G, P, dtype, &smem_stats, &smem_apply);
  if (rc0) return rc0;
  const int threads = a.vpp * a.lanes;
  const int blocks = a.P * a.S;
  int* status = device_status_ptr();
  const float* cgl = stale_global;
  const float* cll = stale_local;
  const float* cused = used;
  if (dtype == DP_BF16) {
    mark_launch(stream);
    int rc = launch_kernel(gn_stats_kernel<__nv_bfloat16>, dim3(blocks), dim3(threads), smem_stats,
                           stream, false, "groupnorm stats launch",
                           static_cast<const __nv_bfloat16*>(x), a, acc, counter, cgl, cll,
                           fresh_local, fresh_global, used, status);
    if (rc) return rc;
    mark_launch(stream);
    return launch_kernel(gn_apply_kernel<__nv_bfloat16>, dim3(blocks), dim3(threads), smem_apply,
                         stream, false, "groupnorm apply launch",
                         static_cast<const __nv_bfloat16*>(x), static_cast<__nv_bfloat16*>(y), gamma,
                         beta, cused, a, status);
  }
  mark_launch(stream);
  int rc = launch_kernel(gn_stats_kernel<float>, dim3(blocks), dim3(threads), smem_stats, stream,
                         false, "groupnorm stats launch", static_cast<const float*>(x), a, acc,
                         counter, cgl, cll, fresh_local, fresh_global, used, status);
  if (rc) return rc;
  mark_launch(stream);
  return launch_kernel(gn_apply_kernel<float>, dim3(blocks), dim3(threads), smem_apply, stream, false,
                       "groupnorm apply launch", static_cast<const float*>(x), static_cast<float*>(y),
                       gamma, beta, cused, a, status);
}

// ---------------------------------------------------------------------------
// Scratch for callers that cannot allocate device memory.  It is a fixed
// file-scope array that every GPU loading this library holds until the
// process exits.  Host code must not hand the array's name to a kernel: on
// the host that name is only a stand-in, so its device address is looked up
// once per device with cudaGetSymbolAddress and that address is passed on.
constexpr size_t kGnStaticScratchBytes = 64 * 1024;
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

int dp_groupnorm_stats(const void* x, int H, int W, int C, int G, int P, float w, int mode, int dtype,
                       const float* stale_global, const float* stale_local, float* fresh_local,
                       float* used_stats, void* workspace, size_t workspace_bytes, void* stream) {
  int rc = dp::gn_validate(x, x, H, W, C, G, P, dtype, mode);   // no output tensor: x stands in
  if (rc) return rc;
  if (!fresh_local || !used_stats || !workspace)
    return dp::set_error(DP_ERR_INVALID_ARG, "groupnorm stats: null fresh_local/used/workspace");
  if (mode == DP_MODE_DISPLACED && (!stale_global || !stale_local))
    return dp::set_error(DP_ERR_INVALID_ARG, "groupnorm stats: displaced mode needs stale statistics");
  if (workspace_bytes < dp::gn_acc_bytes(P, G))
    return dp::set_error(DP_ERR_INVALID_ARG, "groupnorm stats: workspace too small (%zu < %zu)",
                         workspace_bytes, dp::gn_acc_bytes(P, G));
  return dp::gn_stats_launch(x, H, W, C, G, P, w, mode, dtype, stale_global, stale_local, fresh_local,
                             nullptr, used_stats, workspace, static_cast<cudaStream_t>(stream));
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
  if (workspace_bytes < dp::gn_acc_bytes(P, G))
    return dp::set_error(DP_ERR_INVALID_ARG, "groupnorm: workspace too small (%zu < %zu)",
                         workspace_bytes, dp::gn_acc_bytes(P, G));
  if (!(eps > 0.f)) return dp::set_error(DP_ERR_INVALID_ARG, "groupnorm: eps must be > 0");
  return dp::gn_launch(x, y, gamma, beta, H, W, C, G, P, eps, w, silu, mode, dtype, stale_global,
                       stale_local, fresh_local, nullptr, used_stats, workspace, workspace_bytes,
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
  const size_t need = dp::gn_acc_bytes(P, G);
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
                       stale_local, fresh_local, nullptr, used_stats, scratch,
                       dp::kGnStaticScratchBytes, s);
}

}  // extern "C"
