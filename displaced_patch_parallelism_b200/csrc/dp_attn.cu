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
// B200 design (one CTA = 128 queries of one head, 320 threads, 2 CTAs/SM):
//   warp 0     TMA producer: Q once, then K/V tiles of 128 keys through a
//              2-deep ring; each tile is taken whole from the fresh or the
//              stale buffer (bands are multiples of 128 tokens);
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
  float scale_log2;
  __nv_bfloat16* o;
  int ld;
  int* status;
};

constexpr int kAttnStages = 2;
constexpr int kTile = 16384;                     // 128 rows x 128 bytes
constexpr int kAttnThreads = 320;               // producer, MMA, 8 softmax warps
constexpr int kAttnTail = 4096;                  // barriers + max/sum exchange buffers
constexpr int kAttnSmem = kTile * (1 + 2 * kAttnStages) + 1024 + kAttnTail;

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ---- packed fp32x2 arithmetic (two lanes of work per FMA-pipe instruction)
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
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
// that P is rounded to); 2^n by adding n to the exponent field.  Inputs are
// clamped at -125 so the result stays a normal number.
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
  e0 = __int_as_float(__float_as_int(p0) + ((__float_as_int(t0) - 0x4B400000) << 23));
  e1 = __int_as_float(__float_as_int(p1) + ((__float_as_int(t1) - 0x4B400000) << 23));
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
  uint8_t* sQ = smem;
  uint8_t* sK = smem + kTile;
  uint8_t* sV = sK + kAttnStages * kTile;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + kAttnStages * kTile);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = kv_full + kAttnStages;
  uint64_t* s_full = kv_empty + kAttnStages;
  uint64_t* s_free = s_full + 1;
  uint64_t* p_full = s_free + 1;
  uint64_t* o_done = p_full + 1;
  uint64_t* drain = o_done + 1;
  uint64_t* xbar = drain + 1;                                   // [4], one per row quarter
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(xbar + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* red = reinterpret_cast<float*>(bars + 64);             // [2 parities][2 halves][128]

  const int warp = warp_id(), lane = lane_id();
  const int qtile = blockIdx.x, h = blockIdx.y;
  const int q0 = qtile * 128;
  const int band = q0 / p.tb;
  const int band_tiles = p.tb / 128;
  const int n_kv = p.mode == DP_MODE_NAIVE ? band_tiles : p.T / 128;
  const int first_kv = p.mode == DP_MODE_NAIVE ? band * band_tiles : 0;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kAttnStages; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, 8);
    mbar_init(p_full, 8);
    for (int i = 0; i < 4; ++i) mbar_init(&xbar[i], 2);
    mbar_init(o_done, 1);
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
  const uint32_t tS = tmem, tP = tmem + 128, tO = tmem + 192;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      uint32_t issued = 0, issued_par = 0;
      bool q_issued = false;
      int stage = 0;
      uint32_t phase = 0;
      mbar_arrive_expect_tx(q_full, kTile);
      tma_load_2d(sQ, &p.tmQ, q_full, h * 64, q0);
      q_issued = true;
      for (int j = 0; j < n_kv; ++j) {
        const int t = first_kv + j;
        const bool own = (t * 128) / p.tb == band;
        const bool stale = !own && p.mode == DP_MODE_DISPLACED;
        if (!mbar_wait(&kv_empty[stage], phase ^ 1u, abort_flag, p.status)) break;
        mbar_arrive_expect_tx(&kv_full[stage], 2 * kTile);
        tma_load_2d(sK + stage * kTile, stale ? &p.tmKs : &p.tmKf, &kv_full[stage], h * 64, t * 128);
        tma_load_2d(sV + stage * kTile, stale ? &p.tmVs : &p.tmVf, &kv_full[stage], h * 64, t * 128);
        issued |= 1u << stage;
        issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
        if (++stage == kAttnStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (*abort_flag) {
        if (q_issued) attn_wait_teardown(q_full, 0);
        for (int s = 0; s < kAttnStages; ++s)
          if (issued & (1u << s)) attn_wait_teardown(&kv_full[s], (issued_par >> s) & 1u);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      constexpr uint32_t idesc_qk = idesc_dense(128, 128, 1, 0, 0);
      constexpr uint32_t idesc_pv = idesc_dense(128, 64, 1, 0, 1);
      const uint64_t qd = sdesc_sw128(smem_u32(sQ), 1024);
      int stage = 0, prev_stage = 0;
      uint32_t phase = 0;
      bool ok = mbar_wait(q_full, 0, abort_flag, p.status);
      for (int j = 0; ok && j <= n_kv; ++j) {
        if (j < n_kv) {
          if (!mbar_wait(&kv_full[stage], phase, abort_flag, p.status)) break;
          if (j > 0 && !mbar_wait(s_free, (j - 1) & 1, abort_flag, p.status)) break;
          tc_fence_after();
          const uint64_t kd = sdesc_sw128(smem_u32(sK + stage * kTile), 1024);
#pragma unroll
          for (int k = 0; k < 4; ++k) umma_f16_ss(tS, qd + 2 * k, kd + 2 * k, idesc_qk, k != 0);
          umma_commit(s_full);
        }
        if (j > 0) {
          // O += P_{j-1} V_{j-1}
          if (!mbar_wait(p_full, (j - 1) & 1, abort_flag, p.status)) break;
          tc_fence_after();
          const uint64_t vd = sdesc_sw128(smem_u32(sV + prev_stage * kTile), 1024);
#pragma unroll
          for (int k = 0; k < 8; ++k)
            umma_f16_ts(tO, tP + 8 * k, vd + 128 * k, idesc_pv, (j > 1 || k != 0));
          umma_commit(&kv_empty[prev_stage]);
          umma_commit(o_done);
        }
        if (j < n_kv) {
          prev_stage = stage;
          if (++stage == kAttnStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
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
    // (double-buffered by tile parity, bounded mbarrier waits); each half
    // keeps its own partial row sum and owns 32 of the 64 output columns.
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    const int row = q * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    const float c = p.scale_log2;
    float m_used = 0.f, l = 0.f;
    bool aborted = false;
    auto exchange = [&](int use, float mine, float* other) -> bool {
      float* buf = red + (use & 1) * 256;
      buf[half * 128 + row] = mine;
      __syncwarp();
      if (lane == 0) mbar_arrive(&xbar[q]);
      if (!mbar_wait(&xbar[q], use & 1, abort_flag, p.status)) return false;
      *other = buf[(half ^ 1) * 128 + row];
      return true;
    };
    for (int j = 0; j < n_kv; ++j) {
      if (!mbar_wait(s_full, j & 1, abort_flag, p.status)) {
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
      if (!exchange(j, mx, &mo)) {
        aborted = true;
        break;
      }
      const float m_tile = fmaxf(mx, mo) * c;
      float alpha = 1.f;
      if (j == 0) {
        m_used = m_tile;
      } else if (m_tile > m_used + 8.f) {
        alpha = ex2_approx(m_used - m_tile);
        m_used = m_tile;
      }
      // P_j = exp2(s * c - m_used), packed bf16 pairs.  3 of every 8 pairs take
      // the FMA-pipe exponential, the rest the special-function unit.
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
          if ((i & 7) < 3) {
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
      if (j > 0) {
        // P_{j-1} V_{j-1} must be done before O is rescaled or P overwritten
        if (!mbar_wait(o_done, (j - 1) & 1, abort_flag, p.status)) {
          aborted = true;
          break;
        }
        tc_fence_after();
        if (__any_sync(0xffffffffu, alpha != 1.f)) {
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
    float lo = 0.f;
    if (!aborted && n_kv > 0 && exchange(n_kv, l, &lo) &&
        mbar_wait(o_done, (n_kv - 1) & 1, abort_flag, p.status)) {
      tc_fence_after();
      uint32_t o[32];
      tmem_ld32(tO + lane_off + half * 32, o);
      tmem_wait_ld();
      const float inv = 1.f / (l + lo);
      uint4* dst = reinterpret_cast<uint4*>(p.o + static_cast<size_t>(q0 + row) * p.ld + h * 64 +
                                            half * 32);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint4 u;
        u.x = pack_bf16x2(__uint_as_float(o[8 * i]) * inv, __uint_as_float(o[8 * i + 1]) * inv);
        u.y = pack_bf16x2(__uint_as_float(o[8 * i + 2]) * inv, __uint_as_float(o[8 * i + 3]) * inv);
        u.z = pack_bf16x2(__uint_as_float(o[8 * i + 4]) * inv, __uint_as_float(o[8 * i + 5]) * inv);
        u.w = pack_bf16x2(__uint_as_float(o[8 * i + 6]) * inv, __uint_as_float(o[8 * i + 7]) * inv);
        dst[i] = u;
      }
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

int attn_launch(const void* q, const void* kf, const void* vf, const void* ks, const void* vs,
                void* o, int T, int heads, int P, float scale, int mode, cudaStream_t stream) {
  AttnParams a;
  memset(&a, 0, sizeof(a));
  const int ld = heads * 64;
  uint64_t dims[2] = {static_cast<uint64_t>(ld), static_cast<uint64_t>(T)};
  uint64_t str[1] = {static_cast<uint64_t>(ld) * 2};
  uint32_t box[2] = {64, 128};
  const void* ptrs[5] = {q, kf, vf, ks ? ks : kf, vs ? vs : vf};
  CUtensorMap* maps[5] = {&a.tmQ, &a.tmKf, &a.tmVf, &a.tmKs, &a.tmVs};
  for (int i = 0; i < 5; ++i) {
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
  static int attr_mask = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  if (!(attr_mask & (1 << (dev & 31)))) {
    int rc = cuda_check(cudaFuncSetAttribute(attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kAttnSmem),
                        "attention smem attribute");
    if (rc) return rc;
    attr_mask |= 1 << (dev & 31);
  }
  dim3 grid(T / 128, heads);
  mark_launch(stream);
  attn_kernel<<<grid, kAttnThreads, kAttnSmem, stream>>>(a);
  return cuda_check(cudaGetLastError(), "attention launch");
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

extern "C" int dp_attn_stale_kv(const void* q, const void* k_fresh, const void* v_fresh,
                                const void* k_stale, const void* v_stale, void* o, int T,
                                int heads, int head_dim, int P, float scale, int mode,
                                void* stream) {
  int rc = dp::attn_validate(q, k_fresh, v_fresh, k_stale, v_stale, o, T, heads, head_dim, P, mode);
  if (rc) return rc;
  return dp::attn_launch(q, k_fresh, v_fresh, k_stale, v_stale, o, T, heads, P, scale, mode,
                         static_cast<cudaStream_t>(stream));
}
