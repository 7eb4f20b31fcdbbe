// dp_attn.cu -- self-attention over stitched fresh / stale keys and values.
//
// Semantics: DistriFusion keeps the full-spatial K and V of every attention
// layer; a band's fresh queries attend over its own fresh keys and values and
// over the other bands' keys and values from the previous step ("PipeFusion:
// Patch-level Pipeline Parallelism for Diffusion Transformers Inference",
// gist.science explainer, Problem Statement and Memory Efficiency, describing
// DistriFusion).  Sync steps use fresh keys everywhere; naive steps see only
// the band's own keys.
//
// Two kernels.  Bands of a multiple of 256 tokens take attn_pair_kernel (two
// query tiles per CTA, ping-ponged on the tensor core; described above it).
// Other bands take attn_kernel:
// B200 design (one CTA = 128 queries of one head, 320 threads, 2 CTAs/SM):
//   warp 0     TMA producer: Q once per unit, then K and V tiles of 128 keys
//              through two 2-deep rings (a K slot is free once S = Q K^T has
//              read it, long before P V frees the V slot, so the next K loads
//              early); each tile is taken whole from the fresh or the stale
//              buffer (bands are multiples of 128 tokens);
//   warp 1     MMA issuer: S = Q K^T (128x128x64) into tensor memory, then
//              O += P V (128x64x128) with P read straight from tensor memory;
//              S of tile j+1 is issued before O += P_j V_j so the tensor core
//              works while the softmax warps exponentiate;
//   warps 2-9  softmax: two warps per 32 query rows, one half-row (64
//              scores) per thread; S -> registers, online max with lazy
//              rescaling (O is only rescaled when the running maximum grows by
//              more than 2^8), exp2 (part on the FMA pipe), packed bf16 P back
//              to tensor memory; final O / l, bf16 store.
// Tensor memory per CTA (256 columns): S [0,128), P [128,192) as bf16 pairs,
// O [192,256).
#include <cstring>

#include "dp_common.cuh"
#include "dp_internal.h"

namespace dp {

struct AttnParams {
  CUtensorMap tmQ, tmKf, tmVf, tmKs, tmVs;
  int T, heads, P, tb, mode;
  // Work split: a unit is 128 queries of one head (256 in the two-tile
  // kernel; units ordered head-major, n_qt units per head); it takes n_kv key
  // tiles.  CTA b owns the iterations [b L, (b+1) L) of the W = units x n_kv
  // (unit, key tile) iterations.
  int n_qt, n_kv, W, L;
  // keys in the last key tile (128 unless the key count is ragged, as for
  // cross-attention over a text context; the rest of that tile is masked)
  int kv_last;
  float scale_log2;
  __nv_bfloat16* o;
  int ld;
  // Partials of units cut between CTAs: slot 2b + 1 holds CTA b's last
  // segment when it is a unit's start, slot 2b its first segment otherwise.
  // One-tile kernel: each slot is 8 warp slices of 32 rows x (32 O columns,
  // m, l, 2 pad); two-tile kernel: 16 lane-contiguous warp slices (see
  // kPairSliceFloats).
  float* part;
  unsigned* count;          // per CTA 8 (one-tile) or 16 (two-tile) counters: parts of the unit
                            // starting in that CTA done so far
  int* status;
};

constexpr int kAttnStages = 2;
constexpr int kTile = 16384;                     // 128 rows x 128 bytes
constexpr int kAttnThreads = 320;               // producer, MMA, 8 softmax warps
constexpr int kAttnTail = 4096;                  // barriers + max/sum exchange buffers
constexpr int kAttnSmem = kTile * (2 + 2 * kAttnStages) + 1024 + kAttnTail;
constexpr int kSliceFloats = 32 * 36;           // one warp's 32 rows x (32 O, m, l, pad)
constexpr int kSlotFloats = 8 * kSliceFloats;

// The next run of consecutive key tiles of one unit in this CTA's range.
struct AttnSeg {
  int u, k0, k1;
};
__device__ __forceinline__ bool attn_next_seg(const AttnParams& p, int& it, int end, AttnSeg& s) {
  if (it >= end) return false;
  s.u = it / p.n_kv;
  s.k0 = it - s.u * p.n_kv;
  s.k1 = min(p.n_kv, s.k0 + (end - it));
  it += s.k1 - s.k0;
  return true;
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// 2^x for two values on the FMA pipe, so that part of the softmax's
// exponentials leave the special-function unit (the bottleneck of this kernel
// at head_dim 64).  Method: round-to-nearest range reduction x = n + f,
// f in [-1/2, 1/2], by adding 1.5 * 2^23 (the sum's low mantissa bits hold n);
// 2^f by a cubic fitted here for minimax relative error on [-1/2, 1/2]
// (Remez exchange; max relative error 7.5e-5, far below the 2^-9 of the bf16
// that P is rounded to); 2^n by adding n to the exponent field (the low bits
// of t = x + 1.5 * 2^23 hold n, and the magic's own bits vanish in the shift
// by 23).  Inputs are clamped at -125 so the result stays a normal number.
__device__ __forceinline__ void exp2_poly_x2(uint64_t x2, float& e0, float& e1) {
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
  float x0, x1;
  f2_unpack(x2, x0, x1);
  x2 = f2_pack(fmaxf(x0, -125.f), fmaxf(x1, -125.f));
  const uint64_t t2 = f2_add(x2, f2_pack(kMagic, kMagic));
  const uint64_t n2 = f2_add(t2, f2_pack(-kMagic, -kMagic));
  const uint64_t f2 = f2_fma(n2, f2_pack(-1.f, -1.f), x2);
  uint64_t p2 = f2_fma(f2_pack(0.05517166905792616f, 0.05517166905792616f), f2,
                       f2_pack(0.2426111221932161f, 0.2426111221932161f));
  p2 = f2_fma(p2, f2, f2_pack(0.6932609854606553f, 0.6932609854606553f));
  p2 = f2_fma(p2, f2, f2_pack(0.9999280735394012f, 0.9999280735394012f));
  float t0, t1, p0, p1;
  f2_unpack(t2, t0, t1);
  f2_unpack(p2, p0, p1);
  e0 = __int_as_float(__float_as_int(p0) + (__float_as_int(t0) << 23));
  e1 = __int_as_float(__float_as_int(p1) + (__float_as_int(t1) << 23));
}

__device__ __forceinline__ void umma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void attn_wait_teardown(uint64_t* bar, uint32_t parity) {
  const unsigned long long t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) return;
  }
}

__global__ void __launch_bounds__(kAttnThreads, 2) attn_kernel(const __grid_constant__ AttnParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;                                           // [2] query tiles
  uint8_t* sK = smem + 2 * kTile;
  uint8_t* sV = sK + kAttnStages * kTile;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + kAttnStages * kTile);
  uint64_t* q_full = bars;                                      // [2]
  uint64_t* q_empty = q_full + 2;                               // [2]
  uint64_t* k_full = q_empty + 2;
  uint64_t* k_empty = k_full + kAttnStages;
  uint64_t* v_full = k_empty + kAttnStages;
  uint64_t* v_empty = v_full + kAttnStages;
  uint64_t* s_full = v_empty + kAttnStages;
  uint64_t* s_free = s_full + 1;
  uint64_t* p_full = s_free + 1;
  uint64_t* o_done = p_full + 1;
  uint64_t* o_free = o_done + 1;
  uint64_t* drain = o_free + 1;
  uint64_t* xbar = drain + 1;                                   // [4], one per row quarter
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(xbar + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* red = reinterpret_cast<float*>(bars + 64);             // [2 parities][2 halves][128]

  const int warp = warp_id(), lane = lane_id();
  const int band_tiles = p.tb / 128;
  const int start = blockIdx.x * p.L;
  const int end = min(p.W, start + p.L);

  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&q_full[b], 1);
      mbar_init(&q_empty[b], 1);
    }
    for (int s = 0; s < kAttnStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, 8);
    mbar_init(p_full, 8);
    mbar_init(o_done, 1);
    mbar_init(o_free, 8);
    for (int i = 0; i < 4; ++i) mbar_init(&xbar[i], 2);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // set-up done: from here on this grid reads its predecessor's outputs
  griddep_wait();
  griddep_trigger();
  const uint32_t tS = tmem, tP = tmem + 128, tO = tmem + 192;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      // loads in flight, for the teardown after an abort: bits 0-1 K slots,
      // 2-3 V slots, 4-5 Q buffers (with the parity each will complete)
      uint32_t issued = 0, issued_par = 0;
      int stage = 0, qb = 0;
      uint32_t phase = 0, qpar[2] = {0u, 0u};
      int it = start;
      AttnSeg sg;
      while (attn_next_seg(p, it, end, sg)) {
        const int h = sg.u / p.n_qt, q0 = (sg.u - h * p.n_qt) * 128;
        const int band = q0 / p.tb;
        const int first_kv = p.mode == DP_MODE_NAIVE ? band * band_tiles : 0;
        if (!mbar_wait(&q_empty[qb], qpar[qb] ^ 1u, abort_flag, p.status)) break;
        mbar_arrive_expect_tx(&q_full[qb], kTile);
        tma_load_2d(sQ + qb * kTile, &p.tmQ, &q_full[qb], h * 64, q0);
        issued |= 16u << qb;
        issued_par = (issued_par & ~(16u << qb)) | (qpar[qb] << (4 + qb));
        qpar[qb] ^= 1u;
        qb ^= 1;
        bool ok = true;
        for (int j = sg.k0; j < sg.k1; ++j) {
          const int t = first_kv + j;
          const bool own = (t * 128) / p.tb == band;
          const bool stale = !own && p.mode == DP_MODE_DISPLACED;
          if (!mbar_wait(&k_empty[stage], phase ^ 1u, abort_flag, p.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&k_full[stage], kTile);
          tma_load_2d(sK + stage * kTile, stale ? &p.tmKs : &p.tmKf, &k_full[stage], h * 64, t * 128);
          issued |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          if (!mbar_wait(&v_empty[stage], phase ^ 1u, abort_flag, p.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&v_full[stage], kTile);
          tma_load_2d(sV + stage * kTile, stale ? &p.tmVs : &p.tmVf, &v_full[stage], h * 64, t * 128);
          issued |= 4u << stage;
          issued_par = (issued_par & ~(4u << stage)) | (phase << (2 + stage));
          if (++stage == kAttnStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
      }
      if (*abort_flag) {
        for (int s = 0; s < 6; ++s)
          if (issued & (1u << s))
            attn_wait_teardown(s < 2 ? &k_full[s] : s < 4 ? &v_full[s - 2] : &q_full[s - 4],
                               (issued_par >> s) & 1u);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      constexpr uint32_t idesc_qk = idesc_dense(128, 128, 1, 0, 0);
      constexpr uint32_t idesc_pv = idesc_dense(128, 64, 1, 0, 1);
      int stage = 0, prev_stage = 0, qb = 0;
      uint32_t phase = 0, prev_phase = 0, qpar[2] = {0u, 0u};
      int t = 0, si = 0;       // key tiles and segments done by this CTA
      int it = start;
      AttnSeg sg;
      bool ok = true;
      while (ok && attn_next_seg(p, it, end, sg)) {
        const int n = sg.k1 - sg.k0;
        if (!mbar_wait(&q_full[qb], qpar[qb], abort_flag, p.status)) break;
        qpar[qb] ^= 1u;
        tc_fence_after();
        const uint64_t qd = sdesc_sw128(smem_u32(sQ + qb * kTile), 1024);
        for (int jj = 0; jj <= n; ++jj) {
          const int tt = t + jj;
          if (jj < n) {
            if (!mbar_wait(&k_full[stage], phase, abort_flag, p.status) ||
                (tt > 0 && !mbar_wait(s_free, (tt - 1) & 1, abort_flag, p.status))) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t kd = sdesc_sw128(smem_u32(sK + stage * kTile), 1024);
#pragma unroll
            for (int k = 0; k < 4; ++k) umma_f16_ss(tS, qd + 2 * k, kd + 2 * k, idesc_qk, k != 0);
            umma_commit(s_full);
            umma_commit(&k_empty[stage]);
            if (jj == n - 1) umma_commit(&q_empty[qb]);   // this segment's last read of Q
          }
          if (jj > 0) {
            // O += P V of the previous key tile; the segment's first one
            // overwrites O, so the softmax warps must have read the last O
            if (!mbar_wait(p_full, (tt - 1) & 1, abort_flag, p.status) ||
                !mbar_wait(&v_full[prev_stage], prev_phase, abort_flag, p.status) ||
                (jj == 1 && si > 0 && !mbar_wait(o_free, (si - 1) & 1, abort_flag, p.status))) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t vd = sdesc_sw128(smem_u32(sV + prev_stage * kTile), 1024);
#pragma unroll
            for (int k = 0; k < 8; ++k)
              umma_f16_ts(tO, tP + 8 * k, vd + 128 * k, idesc_pv, (jj > 1 || k != 0));
            umma_commit(&v_empty[prev_stage]);
            umma_commit(o_done);
          }
          if (jj < n) {
            prev_stage = stage;
            prev_phase = phase;
            if (++stage == kAttnStages) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
        t += n;
        ++si;
        qb ^= 1;
      }
      if (*abort_flag) {
        umma_commit(drain);
        attn_wait_teardown(drain, 0);
      }
    }
  } else {
    // -------------------------------------------------------------- softmax
    // Warps w and w+4 share TMEM lanes 32*(w%4).. (the same 32 query rows)
    // and split each row's 128 scores into halves, so 8 warps exponentiate.
    // Per tile they exchange their half-row maxima through shared memory
    // (double-buffered by use parity, bounded mbarrier waits); each half
    // keeps its own partial row sum and owns 32 of the 64 output columns.
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    const int row = q * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    const float c = p.scale_log2;
    bool aborted = false;
    uint32_t xuse = 0;
    auto exchange = [&](float mine, float* other) -> bool {
      float* buf = red + (xuse & 1) * 256;
      buf[half * 128 + row] = mine;
      __syncwarp();
      if (lane == 0) mbar_arrive(&xbar[q]);
      const bool ok = mbar_wait(&xbar[q], xuse & 1, abort_flag, p.status);
      ++xuse;
      if (!ok) return false;
      *other = buf[(half ^ 1) * 128 + row];
      return true;
    };
    int t = 0;
    int it = start;
    AttnSeg sg;
    while (!aborted && attn_next_seg(p, it, end, sg)) {
      const int n = sg.k1 - sg.k0;
      float m_used = 0.f, l = 0.f;
      for (int jj = 0; jj < n; ++jj) {
        const int tt = t + jj;
        if (!mbar_wait(s_full, tt & 1, abort_flag, p.status)) {
          aborted = true;
          break;
        }
        tc_fence_after();
        uint32_t s[2][32];
        tmem_ld32(tS + lane_off + half * 64, s[0]);
        tmem_ld32(tS + lane_off + half * 64 + 32, s[1]);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_free);
        float mx = __uint_as_float(s[0][0]);
#pragma unroll
        for (int k = 0; k < 2; ++k)
#pragma unroll
          for (int i = 0; i < 32; i += 2)
            mx = max3(mx, __uint_as_float(s[k][i]), __uint_as_float(s[k][i + 1]));
        float mo;
        if (!exchange(mx, &mo)) {
          aborted = true;
          break;
        }
        const float m_tile = fmaxf(mx, mo) * c;
        float alpha = 1.f;
        if (jj == 0) {
          m_used = m_tile;
        } else if (m_tile > m_used + 8.f) {
          alpha = ex2_approx(m_used - m_tile);
          m_used = m_tile;
        }
        // P = exp2(s * c - m_used), packed bf16 pairs.  1 of every 4 pairs takes
        // the FMA-pipe exponential, the rest the special-function unit (the
        // fastest split measured: 3/8, 3/16 and 1/8 were slower).
        uint32_t pk[32];
        const uint64_t c2 = f2_pack(c, c), negm2 = f2_pack(-m_used, -m_used);
        uint64_t sum2 = f2_pack(0.f, 0.f);
#pragma unroll
        for (int k = 0; k < 2; ++k)
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const uint64_t x2 =
                f2_fma(f2_pack(__uint_as_float(s[k][2 * i]), __uint_as_float(s[k][2 * i + 1])), c2, negm2);
            float e0, e1;
            if ((i & 7) < 2) {
              exp2_poly_x2(x2, e0, e1);
            } else {
              float x0, x1;
              f2_unpack(x2, x0, x1);
              e0 = ex2_approx(x0);
              e1 = ex2_approx(x1);
            }
            sum2 = f2_add(sum2, f2_pack(e0, e1));
            pk[k * 16 + i] = pack_bf16x2(e0, e1);
          }
        float rs0, rs1;
        f2_unpack(sum2, rs0, rs1);
        l = l * alpha + (rs0 + rs1);
        if (tt > 0) {
          // the previous P V must be done before P is overwritten (and, inside
          // a segment, before O is rescaled)
          if (!mbar_wait(o_done, (tt - 1) & 1, abort_flag, p.status)) {
            aborted = true;
            break;
          }
          tc_fence_after();
          if (jj > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
            uint32_t o[32];
            tmem_ld32(tO + lane_off + half * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(tO + lane_off + half * 32, o);
          }
        }
        tmem_st32(tP + lane_off + half * 32, pk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full);
      }
      if (aborted) break;
      // ---- end of the segment: O leaves tensor memory
      float lo = 0.f;
      if (!exchange(l, &lo) || !mbar_wait(o_done, (t + n - 1) & 1, abort_flag, p.status)) {
        aborted = true;
        break;
      }
      tc_fence_after();
      float acc[32];
      {
        uint32_t o[32];
        tmem_ld32(tO + lane_off + half * 32, o);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) acc[i] = __uint_as_float(o[i]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(o_free);
      const float lsum = l + lo;
      const int h = sg.u / p.n_qt, q0 = (sg.u - h * p.n_qt) * 128;
      float inv;
      if (sg.k0 == 0 && sg.k1 == p.n_kv) {
        inv = 1.f / lsum;
      } else {
        // A unit cut between CTAs b_lo..b_hi.  Each part stores this warp's
        // slice (unnormalised O, row max m in the log2 domain, row sum l);
        // the part that finishes last merges all parts in part order (the
        // same bits whichever finishes last) and writes O.  Nothing waits on
        // another CTA.
        const int b_lo = (sg.u * p.n_kv) / p.L, b_hi = ((sg.u + 1) * p.n_kv - 1) / p.L;
        const int me = blockIdx.x;
        const int wslice = warp - 2;
        auto slice = [&](int b) {
          return p.part + (static_cast<size_t>(2 * b + (b == b_lo ? 1 : 0)) * kSlotFloats +
                           static_cast<size_t>(wslice) * kSliceFloats + lane * 36);
        };
        float* mine = slice(me);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          reinterpret_cast<float4*>(mine)[i] = make_float4(acc[4 * i], acc[4 * i + 1], acc[4 * i + 2], acc[4 * i + 3]);
        *reinterpret_cast<float2*>(mine + 32) = make_float2(m_used, lsum);
        __syncwarp();
        unsigned last = 0;
        if (lane == 0) {
          __threadfence();
          last = atomicAdd(p.count + b_lo * 8 + wslice, 1u) == static_cast<unsigned>(b_hi - b_lo);
        }
        last = __shfl_sync(0xffffffffu, last, 0);
        if (!last) {
          t += n;
          continue;
        }
        __threadfence();
        float m = m_used, ls = lsum;   // the first part's state: this CTA's own when it is the first
        if (me != b_lo) {
          const float* p0 = slice(b_lo);
          const float2 ml = __ldcg(reinterpret_cast<const float2*>(p0 + 32));
          m = ml.x;
          ls = ml.y;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 v = __ldcg(reinterpret_cast<const float4*>(p0) + i);
            acc[4 * i] = v.x;
            acc[4 * i + 1] = v.y;
            acc[4 * i + 2] = v.z;
            acc[4 * i + 3] = v.w;
          }
        }
        for (int b = b_lo + 1; b <= b_hi; ++b) {
          const float* pc = slice(b);
          const float2 ml = __ldcg(reinterpret_cast<const float2*>(pc + 32));
          const float mn = fmaxf(m, ml.x);
          const float a0 = ex2_approx(m - mn), a1 = ex2_approx(ml.x - mn);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 v = __ldcg(reinterpret_cast<const float4*>(pc) + i);
            acc[4 * i] = fmaf(acc[4 * i], a0, v.x * a1);
            acc[4 * i + 1] = fmaf(acc[4 * i + 1], a0, v.y * a1);
            acc[4 * i + 2] = fmaf(acc[4 * i + 2], a0, v.z * a1);
            acc[4 * i + 3] = fmaf(acc[4 * i + 3], a0, v.w * a1);
          }
          ls = fmaf(ls, a0, ml.y * a1);
          m = mn;
        }
        if (lane == 0) p.count[b_lo * 8 + wslice] = 0u;   // ready for the next call
        inv = 1.f / ls;
      }
      uint4* dst = reinterpret_cast<uint4*>(p.o + static_cast<size_t>(q0 + row) * p.ld + h * 64 +
                                            half * 32);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint4 u;
        u.x = pack_bf16x2(acc[8 * i] * inv, acc[8 * i + 1] * inv);
        u.y = pack_bf16x2(acc[8 * i + 2] * inv, acc[8 * i + 3] * inv);
        u.z = pack_bf16x2(acc[8 * i + 4] * inv, acc[8 * i + 5] * inv);
        u.w = pack_bf16x2(acc[8 * i + 6] * inv, acc[8 * i + 7] * inv);
        dst[i] = u;
      }
      t += n;
    }
  }

  tc_fence_before();
  __syncthreads();
  __syncwarp();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// ---------------------------------------------------------------------------
// Two query tiles per CTA (bands whose size is a multiple of 256 tokens).
//
// A unit is 256 queries of one head: query tiles A and B (rows q0.. and
// q0+128..) of the same band, so every key tile comes from the same buffer
// for both and is loaded once for both.  One CTA per SM, 608 threads:
//   warp 0       TMA producer: both query tiles once per unit (double-
//                buffered), K and V tiles of 128 keys through 3-deep rings;
//   warps 1, 2   MMA issuers of tiles A and B.  `tcgen05.mma` returns only
//                when the pipe accepts it, and one thread issues a 128x64x16
//                P V instruction in about 56 cycles against 32 of math, so
//                each tile has its own issuer.  Per key tile j an issuer
//                computes S(j) = Q K_j^T as soon as the softmax warps have read
//                S(j-1) out of tensor memory, then O += P(j-1) V_(j-1);
//   warps 3-10   softmax of tile A, warps 11-18 of tile B: 16 query rows per
//                warp, four threads per row; online maximum with lazy
//                rescaling (O is rescaled only when the running maximum grows
//                by more than 2^8), exp2 (1 in 4 on the FMA pipe), bf16 P to
//                tensor memory; at the end of a unit O / l, stored as bf16.
// Tensor memory (512 columns): S_A [0,128), S_B [128,256), O_A [256,320),
// O_B [320,384), P_A [384,448), P_B [448,512) (P as bf16 pairs).
constexpr int kPairStages = 3;
constexpr int kPairThreads = 608;
constexpr int kPairOutBytes = 16 * 2048;                  // per softmax warp: 16 rows x 128 B
constexpr int kPairSmem = 1024 + 4 * kTile + 2 * kPairStages * kTile + kPairOutBytes + kAttnTail;
// A partial of one softmax warp: 9 float4 columns x 32 lanes (a thread's 32
// O values, then m and l of its two rows), lane-contiguous so that every
// access is coalesced.
constexpr int kPairSliceFloats = 9 * 32 * 4;
constexpr int kPairSlotFloats = 16 * kPairSliceFloats;   // the 16 softmax warps
static_assert(kPairSmem > 114 * 1024, "one CTA per SM: it allocates all of tensor memory");

__global__ void __launch_bounds__(kPairThreads, 1) attn_pair_kernel(const __grid_constant__ AttnParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;                                           // [2 buffers][tiles A, B]
  uint8_t* sK = smem + 4 * kTile;
  uint8_t* sV = sK + kPairStages * kTile;
  uint8_t* sOut = sV + kPairStages * kTile;                     // [16 softmax warps][16 rows][128 B]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sOut + kPairOutBytes);
  uint64_t* q_full = bars;                                      // [2]
  uint64_t* q_empty = q_full + 2;                               // [2]
  uint64_t* k_full = q_empty + 2;                               // [stages]
  uint64_t* k_empty = k_full + kPairStages;
  uint64_t* v_full = k_empty + kPairStages;
  uint64_t* v_empty = v_full + kPairStages;
  uint64_t* s_full = v_empty + kPairStages;                     // [2], per query tile
  uint64_t* s_free = s_full + 2;                                // [2]
  uint64_t* p_full = s_free + 2;                                // [2]
  uint64_t* o_done = p_full + 2;                                // [2]
  uint64_t* o_free = o_done + 2;                                // [2]
  uint64_t* drain = o_free + 2;                                 // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = warp_id(), lane = lane_id();
  const int band_tiles = p.tb / 128;
  const int start = blockIdx.x * p.L;
  const int end = min(p.W, start + p.L);

  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&q_full[b], 1);
      mbar_init(&q_empty[b], 2);
      mbar_init(&s_full[b], 1);
      mbar_init(&s_free[b], 8);
      mbar_init(&p_full[b], 8);
      mbar_init(&o_done[b], 1);
      mbar_init(&o_free[b], 8);
      mbar_init(&drain[b], 1);
    }
    for (int s = 0; s < kPairStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 2);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 2);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_wait();
  griddep_trigger();

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      // loads in flight, for the teardown after an abort: bits 0-2 K slots,
      // 3-5 V slots, 6-7 Q buffers (with the parity each will complete)
      uint32_t issued = 0, issued_par = 0;
      int stage = 0, qb = 0;
      uint32_t phase = 0, qpar[2] = {0u, 0u};
      int it = start;
      AttnSeg sg;
      bool ok = true;
      while (ok && attn_next_seg(p, it, end, sg)) {
        const int h = sg.u / p.n_qt, q0 = (sg.u - h * p.n_qt) * 256;
        const int band = q0 / p.tb;
        const int first_kv = p.mode == DP_MODE_NAIVE ? band * band_tiles : 0;
        if (!mbar_wait(&q_empty[qb], qpar[qb] ^ 1u, abort_flag, p.status)) break;
        mbar_arrive_expect_tx(&q_full[qb], 2 * kTile);
        tma_load_2d(sQ + (2 * qb) * kTile, &p.tmQ, &q_full[qb], h * 64, q0);
        tma_load_2d(sQ + (2 * qb + 1) * kTile, &p.tmQ, &q_full[qb], h * 64, q0 + 128);
        issued |= 64u << qb;
        issued_par = (issued_par & ~(64u << qb)) | (qpar[qb] << (6 + qb));
        qpar[qb] ^= 1u;
        qb ^= 1;
        for (int j = sg.k0; j < sg.k1; ++j) {
          const int t = first_kv + j;
          const bool own = (t * 128) / p.tb == band;
          const bool stale = !own && p.mode == DP_MODE_DISPLACED;
          if (!mbar_wait(&k_empty[stage], phase ^ 1u, abort_flag, p.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&k_full[stage], kTile);
          tma_load_2d(sK + stage * kTile, stale ? &p.tmKs : &p.tmKf, &k_full[stage], h * 64, t * 128);
          issued |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          if (!mbar_wait(&v_empty[stage], phase ^ 1u, abort_flag, p.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&v_full[stage], kTile);
          tma_load_2d(sV + stage * kTile, stale ? &p.tmVs : &p.tmVf, &v_full[stage], h * 64, t * 128);
          issued |= 8u << stage;
          issued_par = (issued_par & ~(8u << stage)) | (phase << (3 + stage));
          if (++stage == kPairStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (*abort_flag) {
        for (int s = 0; s < 8; ++s)
          if (issued & (1u << s))
            attn_wait_teardown(s < 3 ? &k_full[s] : s < 6 ? &v_full[s - 3] : &q_full[s - 6],
                               (issued_par >> s) & 1u);
      }
    }
  } else if (warp == 1 || warp == 2) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      const int tile = warp - 1;
      constexpr uint32_t idesc_qk = idesc_dense(128, 128, 1, 0, 0);
      constexpr uint32_t idesc_pv = idesc_dense(128, 64, 1, 0, 1);
      const uint32_t tS = tmem + 128 * tile, tO = tmem + 256 + 64 * tile, tP = tmem + 384 + 64 * tile;
      int stage = 0, prev_stage = 0, qb = 0;
      uint32_t phase = 0, prev_phase = 0, qpar[2] = {0u, 0u};
      int t = 0, si = 0;       // key tiles and segments done by this CTA
      int it = start;
      AttnSeg sg;
      bool ok = true;
      while (ok && attn_next_seg(p, it, end, sg)) {
        const int n = sg.k1 - sg.k0;
        if (!mbar_wait(&q_full[qb], qpar[qb], abort_flag, p.status)) break;
        qpar[qb] ^= 1u;
        tc_fence_after();
        const uint64_t qd = sdesc_sw128(smem_u32(sQ + (2 * qb + tile) * kTile), 1024);
        for (int jj = 0; jj <= n; ++jj) {
          const int tt = t + jj;
          if (jj < n) {
            // S(j) once the softmax warps have read S(j-1)
            if (!mbar_wait(&k_full[stage], phase, abort_flag, p.status) ||
                (tt > 0 && !mbar_wait(&s_free[tile], (tt - 1) & 1, abort_flag, p.status))) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t kd = sdesc_sw128(smem_u32(sK + stage * kTile), 1024);
#pragma unroll
            for (int k = 0; k < 4; ++k) umma_f16_ss(tS, qd + 2 * k, kd + 2 * k, idesc_qk, k != 0);
            umma_commit(&s_full[tile]);
            umma_commit(&k_empty[stage]);
            if (jj == n - 1) umma_commit(&q_empty[qb]);   // this segment's last read of Q
          }
          if (jj > 0) {
            // O += P V of the previous key tile; the segment's first one
            // overwrites O, so the softmax warps must have read the last O
            if (!mbar_wait(&p_full[tile], (tt - 1) & 1, abort_flag, p.status) ||
                !mbar_wait(&v_full[prev_stage], prev_phase, abort_flag, p.status) ||
                (jj == 1 && si > 0 && !mbar_wait(&o_free[tile], (si - 1) & 1, abort_flag, p.status))) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t vd = sdesc_sw128(smem_u32(sV + prev_stage * kTile), 1024);
#pragma unroll
            for (int k = 0; k < 8; ++k) umma_f16_ts(tO, tP + 8 * k, vd + 128 * k, idesc_pv, (jj > 1 || k != 0));
            umma_commit(&v_empty[prev_stage]);
            umma_commit(&o_done[tile]);
          }
          if (jj < n) {
            prev_stage = stage;
            prev_phase = phase;
            if (++stage == kPairStages) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
        t += n;
        ++si;
        qb ^= 1;
      }
      if (*abort_flag) {
        umma_commit(&drain[tile]);
        attn_wait_teardown(&drain[tile], 0);
      }
    }
  } else {
    // -------------------------------------------------------------- softmax
    // Warp w (3..18): query tile (w-3)/8, TMEM lane quarter w%4 (the only
    // lanes a warp may access), 16-row half ((w-3)/4)%2 of that quarter.
    // With the 16x256b load shape, thread t holds rows t/4 and t/4+8 of the
    // warp's 16 and, of each group of 8 columns, columns 2(t%4) and +1: a
    // row's maximum and sum take two shuffles, and the thread's bf16 pairs
    // are exactly the P words it stores with the 16x128b shape.
    const int tile = (warp - 3) >> 3;
    const int q = warp & 3;
    const int half = ((warp - 3) >> 2) & 1;
    const int wslice = warp - 3;
    const int rbase = q * 32 + half * 16;                 // first row of the warp in the tile
    const uint32_t lane_off = static_cast<uint32_t>(rbase) << 16;
    const uint32_t tS = tmem + 128 * tile + lane_off;
    const uint32_t tO = tmem + 256 + 64 * tile + lane_off;
    const uint32_t tP = tmem + 384 + 64 * tile + lane_off;
    const int r = lane >> 2, cq = lane & 3;
    const float c = p.scale_log2;
    bool aborted = false;
    int t = 0, si = 0;
    int it = start;
    AttnSeg sg;
    while (!aborted && attn_next_seg(p, it, end, sg)) {
      const int n = sg.k1 - sg.k0;
      float mA = 0.f, mB = 0.f, lA = 0.f, lB = 0.f;   // rows r and r+8: running max (log2), partial sum
      for (int jj = 0; jj < n; ++jj) {
        const int tt = t + jj;
        if (!mbar_wait(&s_full[tile], tt & 1, abort_flag, p.status)) {
          aborted = true;
          break;
        }
        tc_fence_after();
        // Row maxima from both halves of S; columns 64-127 stay in registers,
        // columns 0-63 are read again after them (fewer live registers), and
        // only then is S released.
        uint32_t sa[32], sb[32];
        tmem_ld16x256_x8(tS, sa);
        tmem_ld16x256_x8(tS + 64, sb);
        tmem_wait_ld();
        // a ragged last key tile: its missing keys (zero rows from the
        // tensor map's bounds) get score -inf, i.e. weight 0
        const bool ragged = sg.k0 + jj == p.n_kv - 1 && p.kv_last < 128;
        if (ragged) {
#pragma unroll
          for (int k = 0; k < 8; ++k)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int col = 8 * k + 2 * cq + (e & 1);
              if (col >= p.kv_last) sa[4 * k + e] = 0xff800000u;
              if (col + 64 >= p.kv_last) sb[4 * k + e] = 0xff800000u;
            }
        }
        float xa0 = fmaxf(__uint_as_float(sa[0]), __uint_as_float(sa[1]));
        float xa1 = fmaxf(__uint_as_float(sb[0]), __uint_as_float(sb[1]));
        float xb0 = fmaxf(__uint_as_float(sa[2]), __uint_as_float(sa[3]));
        float xb1 = fmaxf(__uint_as_float(sb[2]), __uint_as_float(sb[3]));
#pragma unroll
        for (int k = 1; k < 8; ++k) {
          xa0 = max3(xa0, __uint_as_float(sa[4 * k]), __uint_as_float(sa[4 * k + 1]));
          xa1 = max3(xa1, __uint_as_float(sb[4 * k]), __uint_as_float(sb[4 * k + 1]));
          xb0 = max3(xb0, __uint_as_float(sa[4 * k + 2]), __uint_as_float(sa[4 * k + 3]));
          xb1 = max3(xb1, __uint_as_float(sb[4 * k + 2]), __uint_as_float(sb[4 * k + 3]));
        }
        float xa = fmaxf(xa0, xa1), xb = fmaxf(xb0, xb1);
        xa = fmaxf(xa, __shfl_xor_sync(0xffffffffu, xa, 1));
        xb = fmaxf(xb, __shfl_xor_sync(0xffffffffu, xb, 1));
        xa = fmaxf(xa, __shfl_xor_sync(0xffffffffu, xa, 2));
        xb = fmaxf(xb, __shfl_xor_sync(0xffffffffu, xb, 2));
        const float mtA = xa * c, mtB = xb * c;
        float alA = 1.f, alB = 1.f;
        if (jj == 0) {
          mA = mtA;
          mB = mtB;
        } else {
          if (mtA > mA + 8.f) {
            alA = ex2_approx(mA - mtA);
            mA = mtA;
          }
          if (mtB > mB + 8.f) {
            alB = ex2_approx(mB - mtB);
            mB = mtB;
          }
        }
        // P = exp2(s * c - m) as bf16 pairs; 1 pair in 4 takes the FMA-pipe
        // exponential
        const uint64_t c2 = f2_pack(c, c), nA2 = f2_pack(-mA, -mA), nB2 = f2_pack(-mB, -mB);
        uint64_t sumA2 = f2_pack(0.f, 0.f), sumB2 = f2_pack(0.f, 0.f);
        auto exps = [&](const uint32_t (&sk)[32], uint32_t (&pk)[16]) {
#pragma unroll
          for (int k = 0; k < 8; ++k) {
#pragma unroll
            for (int rw = 0; rw < 2; ++rw) {
              const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(sk[4 * k + 2 * rw]),
                                                 __uint_as_float(sk[4 * k + 2 * rw + 1])),
                                         c2, rw ? nB2 : nA2);
              float e0, e1;
              if ((k & 3) == 0) {
                exp2_poly_x2(x2, e0, e1);
              } else {
                float x0, x1;
                f2_unpack(x2, x0, x1);
                e0 = ex2_approx(x0);
                e1 = ex2_approx(x1);
              }
              if (rw)
                sumB2 = f2_add(sumB2, f2_pack(e0, e1));
              else
                sumA2 = f2_add(sumA2, f2_pack(e0, e1));
              pk[2 * k + rw] = pack_bf16x2(e0, e1);
            }
          }
        };
        // Both halves are exponentiated before P is written, so the previous
        // P V (which frees the P columns) has the whole softmax to complete.
        uint32_t pk_hi[16], pk_lo[16];
        exps(sb, pk_hi);
        tmem_ld16x256_x8(tS, sa);
        tmem_wait_ld();
        if (ragged) {
#pragma unroll
          for (int k = 0; k < 8; ++k)
#pragma unroll
            for (int e = 0; e < 4; ++e)
              if (8 * k + 2 * cq + (e & 1) >= p.kv_last) sa[4 * k + e] = 0xff800000u;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_free[tile]);   // S(j+1) may now be computed
        exps(sa, pk_lo);
        if (tt > 0) {
          // the previous P V must be done before P is overwritten (and, inside
          // a segment, before O is rescaled)
          if (!mbar_wait(&o_done[tile], (tt - 1) & 1, abort_flag, p.status)) {
            aborted = true;
            break;
          }
          tc_fence_after();
          if (jj > 0 && __any_sync(0xffffffffu, alA != 1.f || alB != 1.f)) {
            uint32_t o[32];
            tmem_ld16x256_x8(tO, o);
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              o[4 * k] = __float_as_uint(__uint_as_float(o[4 * k]) * alA);
              o[4 * k + 1] = __float_as_uint(__uint_as_float(o[4 * k + 1]) * alA);
              o[4 * k + 2] = __float_as_uint(__uint_as_float(o[4 * k + 2]) * alB);
              o[4 * k + 3] = __float_as_uint(__uint_as_float(o[4 * k + 3]) * alB);
            }
            tmem_st16x256_x8(tO, o);
          }
        }
        tmem_st16x128_x8(tP + 32, pk_hi);
        tmem_st16x128_x8(tP, pk_lo);
        float s0, s1;
        f2_unpack(sumA2, s0, s1);
        lA = lA * alA + (s0 + s1);
        f2_unpack(sumB2, s0, s1);
        lB = lB * alB + (s0 + s1);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[tile]);
      }
      if (aborted) break;
      // ---- end of the segment: O leaves tensor memory
      if (!mbar_wait(&o_done[tile], (t + n - 1) & 1, abort_flag, p.status)) {
        aborted = true;
        break;
      }
      tc_fence_after();
      uint32_t ob[32];
      tmem_ld16x256_x8(tO, ob);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&o_free[tile]);
      lA += __shfl_xor_sync(0xffffffffu, lA, 1);
      lB += __shfl_xor_sync(0xffffffffu, lB, 1);
      lA += __shfl_xor_sync(0xffffffffu, lA, 2);
      lB += __shfl_xor_sync(0xffffffffu, lB, 2);
      float acc[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) acc[i] = __uint_as_float(ob[i]);
      const int h = sg.u / p.n_qt, q0 = (sg.u - h * p.n_qt) * 256;
      float invA, invB;
      if (sg.k0 == 0 && sg.k1 == p.n_kv) {
        invA = 1.f / lA;
        invB = 1.f / lB;
      } else {
        // A unit cut between CTAs b_lo..b_hi: each part stores its rows
        // (unnormalised O, row max m in the log2 domain, row sum l); the part
        // that finishes last merges all parts in part order (the same bits
        // whichever finishes last) and writes O.  Nothing waits on another CTA.
        const int b_lo = (sg.u * p.n_kv) / p.L, b_hi = ((sg.u + 1) * p.n_kv - 1) / p.L;
        const int me = blockIdx.x;
        auto slice = [&](int b) {
          return reinterpret_cast<float4*>(p.part + static_cast<size_t>(2 * b + (b == b_lo ? 1 : 0)) * kPairSlotFloats +
                                           static_cast<size_t>(wslice) * kPairSliceFloats) + lane;
        };
        float4* mine = slice(me);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          mine[32 * i] = make_float4(acc[4 * i], acc[4 * i + 1], acc[4 * i + 2], acc[4 * i + 3]);
        mine[32 * 8] = make_float4(mA, lA, mB, lB);
        __syncwarp();
        unsigned last = 0;
        if (lane == 0) {
          __threadfence();
          last = atomicAdd(p.count + b_lo * 16 + wslice, 1u) == static_cast<unsigned>(b_hi - b_lo);
        }
        last = __shfl_sync(0xffffffffu, last, 0);
        if (!last) {
          t += n;
          ++si;
          continue;
        }
        __threadfence();
        float ma = mA, la = lA, mb = mB, lb = lB;   // the first part's state: this CTA's own when it is the first
        if (me != b_lo) {
          const float4* p0 = slice(b_lo);
          const float4 ml = __ldcg(p0 + 32 * 8);
          ma = ml.x;
          la = ml.y;
          mb = ml.z;
          lb = ml.w;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 v = __ldcg(p0 + 32 * i);
            acc[4 * i] = v.x;
            acc[4 * i + 1] = v.y;
            acc[4 * i + 2] = v.z;
            acc[4 * i + 3] = v.w;
          }
        }
        for (int b = b_lo + 1; b <= b_hi; ++b) {
          const float4* pc = slice(b);
          const float4 ml = __ldcg(pc + 32 * 8);
          float4 v[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) v[i] = __ldcg(pc + 32 * i);
          const float na = fmaxf(ma, ml.x), nb = fmaxf(mb, ml.z);
          const float a0 = ex2_approx(ma - na), a1 = ex2_approx(ml.x - na);
          const float b0 = ex2_approx(mb - nb), b1 = ex2_approx(ml.z - nb);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            acc[4 * i] = fmaf(acc[4 * i], a0, v[i].x * a1);
            acc[4 * i + 1] = fmaf(acc[4 * i + 1], a0, v[i].y * a1);
            acc[4 * i + 2] = fmaf(acc[4 * i + 2], b0, v[i].z * b1);
            acc[4 * i + 3] = fmaf(acc[4 * i + 3], b0, v[i].w * b1);
          }
          la = fmaf(la, a0, ml.y * a1);
          lb = fmaf(lb, b0, ml.w * b1);
          ma = na;
          mb = nb;
        }
        if (lane == 0) p.count[b_lo * 16 + wslice] = 0u;   // ready for the next call
        invA = 1.f / la;
        invB = 1.f / lb;
      }
      // O / l as bf16 through the warp's 16 staging rows of 128 bytes (16-byte
      // chunks rotated by the row, so a quarter-warp covers all banks), then
      // 8 lanes per row store 128 contiguous bytes
      uint8_t* stage_rows = sOut + wslice * 2048;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int off = ((k ^ r) << 4) + 4 * cq;
        *reinterpret_cast<uint32_t*>(stage_rows + r * 128 + off) =
            pack_bf16x2(acc[4 * k] * invA, acc[4 * k + 1] * invA);
        *reinterpret_cast<uint32_t*>(stage_rows + (r + 8) * 128 + off) =
            pack_bf16x2(acc[4 * k + 2] * invB, acc[4 * k + 3] * invB);
      }
      __syncwarp();
      const int row0 = q0 + 128 * tile + rbase;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int rr = 4 * k + (lane >> 3), ch = lane & 7;
        const uint4 u = *reinterpret_cast<const uint4*>(stage_rows + rr * 128 + ((ch ^ (rr & 7)) << 4));
        *reinterpret_cast<uint4*>(p.o + static_cast<size_t>(row0 + rr) * p.ld + h * 64 + ch * 8) = u;
      }
      __syncwarp();
      t += n;
      ++si;
    }
  }
  tc_fence_before();
  __syncthreads();
  __syncwarp();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Workspace of the balanced launch: per-CTA part counters (zero before first
// use; every call leaves them zero), then two partial slots per CTA.
static size_t attn_count_bytes(size_t slots) { return (slots * 8 * sizeof(unsigned) + 255) & ~size_t(255); }

size_t attn_workspace_bytes() {
  // counters for up to two CTAs per SM; two partial slots per CTA of either kernel
  const size_t sms = static_cast<size_t>(num_sms());
  const size_t one = 2 * (2 * sms) * kSlotFloats, pair = 2 * sms * kPairSlotFloats;
  return attn_count_bytes(2 * sms) + (one > pair ? one : pair) * sizeof(float);
}

// Self-attention (Tk = T) or, with Tk != T, attention of T queries over Tk
// keys that are all visible (mode SYNC, P = 1: cross-attention).
int attn_launch_tk(const void* q, const void* kf, const void* vf, const void* ks, const void* vs,
                   void* o, int T, int Tk, int heads, int P, float scale, int mode,
                   void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  AttnParams a;
  memset(&a, 0, sizeof(a));
  const int ld = heads * 64;
  uint64_t str[1] = {static_cast<uint64_t>(ld) * 2};
  uint32_t box[2] = {64, 128};
  const void* ptrs[5] = {q, kf, vf, ks ? ks : kf, vs ? vs : vf};
  CUtensorMap* maps[5] = {&a.tmQ, &a.tmKf, &a.tmVf, &a.tmKs, &a.tmVs};
  for (int i = 0; i < 5; ++i) {
    uint64_t dims[2] = {static_cast<uint64_t>(ld), static_cast<uint64_t>(i == 0 ? T : Tk)};
    int rc = encode_tmap(maps[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptrs[i]),
                         dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc) return rc;
  }
  a.T = T;
  a.heads = heads;
  a.P = P;
  a.tb = T / P;
  a.mode = mode;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.ld = ld;
  a.status = device_status_ptr();
  // Bands of a multiple of 256 tokens take the two-tile kernel (one CTA per
  // SM); others the one-tile kernel (two CTAs per SM).
  const bool pair = a.tb % 256 == 0;
  static int attr_mask = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  if (!(attr_mask & (1 << (dev & 31)))) {
    int rc = cuda_check(cudaFuncSetAttribute(attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kAttnSmem),
                        "attention smem attribute");
    if (!rc)
      rc = cuda_check(cudaFuncSetAttribute(attn_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           kPairSmem),
                      "attention smem attribute");
    if (rc) return rc;
    attr_mask |= 1 << (dev & 31);
  }
  a.n_qt = T / (pair ? 256 : 128);
  a.n_kv = mode == DP_MODE_NAIVE ? a.tb / 128 : (Tk + 127) / 128;
  a.kv_last = Tk - (a.n_kv - 1) * 128;
  if (mode == DP_MODE_NAIVE) a.kv_last = 128;
  const int units = a.n_qt * heads;
  a.W = units * a.n_kv;
  // Balanced split: every CTA takes an equal run of (unit, key tile)
  // iterations; the parts of a unit cut between CTAs are merged by whichever
  // finishes last, so no CTA waits on another and any residency is correct.
  // Without a workspace each CTA takes one whole unit.  The one-tile kernel
  // fits two CTAs on an SM (shared and tensor memory), the two-tile kernel one.
  const int slots = (pair ? 1 : 2) * num_sms();
  // Cost in key-tile iterations of a CTA: its fixed cost (launch, set-up,
  // first loads, epilogue) is about 5 of them and each cut segment about 2
  // more (measured on B200 with the one-tile kernel).  Whole units take
  // ceil(units / slots) rounds; the split takes one round of L iterations.
  const int L_split = (a.W + slots - 1) / slots;
  const double t_whole = static_cast<double>((units + slots - 1) / slots) * (a.n_kv + 5);
  const double t_split = L_split + 5 + 4;
  const bool split = workspace && workspace_bytes >= attn_workspace_bytes() && units % slots != 0 &&
                     t_split < 0.85 * t_whole;
  if (split) {
    a.L = L_split;
    a.count = static_cast<unsigned*>(workspace);
    a.part = reinterpret_cast<float*>(static_cast<char*>(workspace) + attn_count_bytes(2 * num_sms()));
  } else {
    a.L = a.n_kv;
  }
  const int grid = (a.W + a.L - 1) / a.L;
  mark_launch(stream);
  if (pair)
    return launch_kernel(attn_pair_kernel, dim3(grid), dim3(kPairThreads), kPairSmem, stream, false,
                         "attention launch", a);
  return launch_kernel(attn_kernel, dim3(grid), dim3(kAttnThreads), kAttnSmem, stream, false,
                       "attention launch", a);
}

int attn_launch(const void* q, const void* kf, const void* vf, const void* ks, const void* vs,
                void* o, int T, int heads, int P, float scale, int mode, void* workspace,
                size_t workspace_bytes, cudaStream_t stream) {
  return attn_launch_tk(q, kf, vf, ks, vs, o, T, T, heads, P, scale, mode, workspace,
                        workspace_bytes, stream);
}

int attn_validate(const void* q, const void* kf, const void* vf, const void* ks, const void* vs,
                  const void* o, int T, int heads, int head_dim, int P, int mode) {
  if (!q || !kf || !vf || !o) return set_error(DP_ERR_INVALID_ARG, "attention: null pointer");
  if (T <= 0 || heads <= 0 || P <= 0) return set_error(DP_ERR_INVALID_ARG, "attention: bad size");
  if (mode < DP_MODE_SYNC || mode > DP_MODE_NAIVE)
    return set_error(DP_ERR_INVALID_ARG, "attention: bad mode %d", mode);
  if (head_dim != 64) return set_error(DP_ERR_UNSUPPORTED, "attention: head_dim must be 64");
  if (T % P || (T / P) % 128)
    return set_error(DP_ERR_UNSUPPORTED, "attention: T/P must be a multiple of 128");
  if (mode == DP_MODE_DISPLACED && (!ks || !vs))
    return set_error(DP_ERR_INVALID_ARG, "attention: displaced mode needs stale K/V");
  const void* ins[5] = {q, kf, vf, ks, vs};
  for (int i = 0; i < 5; ++i) {
    if (ins[i] && !aligned16(ins[i])) return set_error(DP_ERR_UNSUPPORTED, "attention: pointer not 16-byte aligned");
    if (ins[i] == o) return set_error(DP_ERR_INVALID_ARG, "attention: o aliases an input");
  }
  if (!aligned16(o)) return set_error(DP_ERR_UNSUPPORTED, "attention: o not 16-byte aligned");
  return DP_OK;
}

}  // namespace dp

extern "C" size_t dp_attn_workspace_size(void) { return dp::attn_workspace_bytes(); }

extern "C" int dp_attn_cross(const void* q, const void* k, const void* v, void* o, int Tq, int Tk,
                             int heads, int head_dim, float scale, void* workspace,
                             size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !o) return dp::set_error(DP_ERR_INVALID_ARG, "cross-attention: null pointer");
  if (Tq <= 0 || Tk <= 0 || heads <= 0) return dp::set_error(DP_ERR_INVALID_ARG, "cross-attention: bad size");
  if (head_dim != 64) return dp::set_error(DP_ERR_UNSUPPORTED, "cross-attention: head_dim must be 64");
  if (Tq % 256) return dp::set_error(DP_ERR_UNSUPPORTED, "cross-attention: Tq must be a multiple of 256");
  const void* ins[3] = {q, k, v};
  for (int i = 0; i < 3; ++i) {
    if (!dp::aligned16(ins[i])) return dp::set_error(DP_ERR_UNSUPPORTED, "cross-attention: pointer not 16-byte aligned");
    if (ins[i] == o) return dp::set_error(DP_ERR_INVALID_ARG, "cross-attention: o aliases an input");
  }
  if (!dp::aligned16(o)) return dp::set_error(DP_ERR_UNSUPPORTED, "cross-attention: o not 16-byte aligned");
  if (workspace && !dp::aligned16(workspace))
    return dp::set_error(DP_ERR_UNSUPPORTED, "cross-attention: workspace not 16-byte aligned");
  return dp::attn_launch_tk(q, k, v, nullptr, nullptr, o, Tq, Tk, heads, 1, scale, DP_MODE_SYNC,
                            workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
}

extern "C" int dp_attn_stale_kv(const void* q, const void* k_fresh, const void* v_fresh,
                                const void* k_stale, const void* v_stale, void* o, int T,
                                int heads, int head_dim, int P, float scale, int mode,
                                void* workspace, size_t workspace_bytes, void* stream) {
  int rc = dp::attn_validate(q, k_fresh, v_fresh, k_stale, v_stale, o, T, heads, head_dim, P, mode);
  if (rc) return rc;
  if (workspace && !dp::aligned16(workspace))
    return dp::set_error(DP_ERR_UNSUPPORTED, "attention: workspace not 16-byte aligned");
  return dp::attn_launch(q, k_fresh, v_fresh, k_stale, v_stale, o, T, heads, P, scale, mode,
                         workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
}
