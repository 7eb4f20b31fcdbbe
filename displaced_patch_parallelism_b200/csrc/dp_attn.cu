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
// B200 design (one CTA = 128 queries of one head, 192 threads, 2 CTAs/SM):
//   warp 0     TMA producer: Q once, then K/V tiles of 128 keys through a
//              2-deep ring; each tile is taken whole from the fresh or the
//              stale buffer (bands are multiples of 128 tokens);
//   warp 1     MMA issuer: S = Q K^T (128x128x64) into tensor memory, then
//              O += P V (128x64x128) with P read straight from tensor memory;
//              S of tile j+1 is issued before O += P_j V_j so the tensor core
//              works while the softmax warps exponentiate;
//   warps 2-5  softmax: one query row per thread; S row -> registers, online
//              max with lazy rescaling (O is only rescaled when the running
//              maximum grows by more than 2^8), exp2, packed bf16 P back to
//              tensor memory; final O / l, bf16 store.
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
constexpr int kAttnSmem = kTile * (1 + 2 * kAttnStages) + 1024 + 256;

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
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

__global__ void __launch_bounds__(192, 2) attn_kernel(const __grid_constant__ AttnParams p) {
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
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

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
    mbar_init(s_free, 4);
    mbar_init(p_full, 4);
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
    const int q = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    const float c = p.scale_log2;
    float m_used = 0.f, l = 0.f;
    bool aborted = false;
    for (int j = 0; j < n_kv; ++j) {
      if (!mbar_wait(s_full, j & 1, abort_flag, p.status)) {
        aborted = true;
        break;
      }
      tc_fence_after();
      uint32_t s[4][32];
#pragma unroll
      for (int k = 0; k < 4; ++k) tmem_ld32(tS + lane_off + 32 * k, s[k]);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free);
      float mx = __uint_as_float(s[0][0]);
#pragma unroll
      for (int k = 0; k < 4; ++k)
#pragma unroll
        for (int i = 0; i < 32; ++i) mx = fmaxf(mx, __uint_as_float(s[k][i]));
      const float m_tile = mx * c;
      float alpha = 1.f;
      if (j == 0) {
        m_used = m_tile;
      } else if (m_tile > m_used + 8.f) {
        alpha = ex2_approx(m_used - m_tile);
        m_used = m_tile;
      }
      // P_j = exp2(s * c - m_used), packed bf16 pairs
      uint32_t pk[2][32];
      float rs = 0.f;
#pragma unroll
      for (int k = 0; k < 4; ++k)
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float e0 = ex2_approx(fmaf(__uint_as_float(s[k][2 * i]), c, -m_used));
          const float e1 = ex2_approx(fmaf(__uint_as_float(s[k][2 * i + 1]), c, -m_used));
          rs += e0 + e1;
          pk[k >> 1][(k & 1) * 16 + i] = pack_bf16x2(e0, e1);
        }
      l = l * alpha + rs;
      if (j > 0) {
        // P_{j-1} V_{j-1} must be done before O is rescaled or P overwritten
        if (!mbar_wait(o_done, (j - 1) & 1, abort_flag, p.status)) {
          aborted = true;
          break;
        }
        tc_fence_after();
        if (__any_sync(0xffffffffu, alpha != 1.f)) {
          uint32_t o[2][32];
          tmem_ld32(tO + lane_off, o[0]);
          tmem_ld32(tO + lane_off + 32, o[1]);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 2; ++k)
#pragma unroll
            for (int i = 0; i < 32; ++i) o[k][i] = __float_as_uint(__uint_as_float(o[k][i]) * alpha);
          tmem_st32(tO + lane_off, o[0]);
          tmem_st32(tO + lane_off + 32, o[1]);
        }
      }
      tmem_st32(tP + lane_off, pk[0]);
      tmem_st32(tP + lane_off + 32, pk[1]);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    if (!aborted && n_kv > 0 && mbar_wait(o_done, (n_kv - 1) & 1, abort_flag, p.status)) {
      tc_fence_after();
      uint32_t o[2][32];
      tmem_ld32(tO + lane_off, o[0]);
      tmem_ld32(tO + lane_off + 32, o[1]);
      tmem_wait_ld();
      const float inv = 1.f / l;
      const int row = q0 + q * 32 + lane;
      uint4* dst = reinterpret_cast<uint4*>(p.o + static_cast<size_t>(row) * p.ld + h * 64);
#pragma unroll
      for (int k = 0; k < 2; ++k)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          uint4 u;
          u.x = pack_bf16x2(__uint_as_float(o[k][8 * i]) * inv, __uint_as_float(o[k][8 * i + 1]) * inv);
          u.y = pack_bf16x2(__uint_as_float(o[k][8 * i + 2]) * inv, __uint_as_float(o[k][8 * i + 3]) * inv);
          u.z = pack_bf16x2(__uint_as_float(o[k][8 * i + 4]) * inv, __uint_as_float(o[k][8 * i + 5]) * inv);
          u.w = pack_bf16x2(__uint_as_float(o[k][8 * i + 6]) * inv, __uint_as_float(o[k][8 * i + 7]) * inv);
          dst[k * 4 + i] = u;
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
  attn_kernel<<<grid, 192, kAttnSmem, stream>>>(a);
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
