// dp_gemm.cu -- tcgen05 implicit GEMM: the stale-halo 3x3 conv and the token
// projections.
//
// Conv semantics ("DistriFusion", study.space summary, Method): a band keeps
// its interaction with the other bands by reading their rows from the
// previous step's activations.  For output row r of band p, input row
// rho = stride*r + kh - 1 comes from the fresh buffer if it lies in band p,
// otherwise from the fresh buffer (sync), the stale buffer (displaced) or
// nowhere (naive: zeros); outside the image it is zero padding.
//
// B200 design:
//  * one persistent CTA per SM, 192 threads in three roles (the 2-SM pair
//    kernel below: 320, with two epilogue warps per TMEM lane quarter):
//      warp 0     TMA producer (one lane): A and B tiles into a STAGES-deep
//                 ring of 128-byte-swizzled shared-memory stages;
//      warp 1     MMA issuer (one lane): tcgen05.mma 128 x BN x 16 into a
//                 tensor-memory accumulator, double buffered so the
//                 epilogue of tile i overlaps the main loop of tile i+1;
//      warps 2-5  epilogue: tcgen05.ld, + bias (+ residual), cast, store.
//  * implicit GEMM for the conv: M = output pixels (a tile is R rows x Wt
//    columns, R*Wt = 128), N = Cout, K = 9 taps x Cin.  Each tap's A tile is
//    R TMA boxes of one image row each, so every box has exactly one source:
//    the fresh map, the stale map, or an out-of-range row that TMA fills with
//    zeros.  Column halos use TMA's out-of-bounds zero fill too, so no
//    padded copy of the activations is ever made.
//  * stride 2 views the image as [H][W/2][2*Cin] (two neighbouring columns
//    side by side in the channel axis): the three column taps become two
//    channel halves of pairs c-1 and c, and the same TMA boxes serve.
//  * fp32 storage runs in fp32 on the CUDA cores instead (dp_conv_f32.cu).
#include <algorithm>
#include <cstring>
#include <type_traits>

#include "dp_common.cuh"
#include "dp_gn_apply.cuh"
#include "dp_internal.h"

namespace dp {

struct GemmParams {
  CUtensorMap tmA0;   // plain A, or the conv's fresh activations
  CUtensorMap tmA1;   // the conv's stale activations
  CUtensorMap tmB;    // weights, [N][K] K-major
  // Pair kernels only: output segments as 32-column boxes of one epilogue
  // warp's 32 rows (64-byte swizzle), for TMA stores.
  CUtensorMap tmO[3];
  int a_mode;         // 0: plain [M][K] rows, 1: 3x3 conv
  int M;
  int H, W, Ho, Wo, Cin, stride, hb_in, hb_out, mode, R, Wt, tiles_w, kc;
  int N, n_tiles, m_tiles, k_blocks;
  const float* bias;
  const void* residual;
  void* out0;
  void* out1;
  void* out2;
  int ld_out;   // elements per row of each output buffer
  int split;    // output columns per buffer
  int* status;
  // Split K (pair kernels): each output tile is cut into `splits` runs of
  // k-blocks; run r stores its fp32 partial, laid out like the output
  // ([M][N]), at part + r * M * N, and a finish kernel adds the runs, bias
  // and residual and stores the outputs.
  int splits;
  float* part;
  // GroupNorm-fused conv only (igemm_gn_pair_kernel): tmA0 maps the raw input
  // x, tmA1 the previous step's normalised activations; the kernel normalises
  // each staged input row in shared memory.
  const float* gn_used;    // [P][G][2]: (mean, var) band p normalises group g with
  const float* gn_gamma;   // [Cin]
  const float* gn_beta;    // [Cin]
  float gn_eps;
  int gn_cg;               // channels per group
  int gn_silu;
  void* a_next;            // [H][W][Cin]: receives the normalised band-edge rows, or null
  // Pair kernels, 3x3 conv: stores under an L2 evict-first policy (an output
  // larger than L2 is written back while the kernel runs).
  int out_evict_first;
  // Pair kernels, plain A only: the epilogue applies the gated GELU.  The N =
  // 2F accumulator columns hold value and gate interleaved in blocks of 16
  // (each 32-column chunk: 16 values, then their 16 gates); tmO[0] maps the
  // [M][F] output as 16-column boxes of 32 rows, unswizzled.
  int geglu;
};

// k-blocks [*kb0, *kb1) of run `r` of `splits` over `kb` k-blocks.
__device__ __forceinline__ void split_range(int kb, int splits, int r, int* kb0, int* kb1) {
  *kb0 = (r * kb) / splits;
  *kb1 = ((r + 1) * kb) / splits;
}

template <int BN>
struct GemmCfg {
  static constexpr int BM = 128;
  static constexpr int BK = 64;                  // bf16 elements per 128-byte row
  static constexpr int A_BYTES = BM * 128;
  static constexpr int B_BYTES = BN * 128;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES_RAW = (200 * 1024) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_RAW > 8 ? 8 : STAGES_RAW;
  static constexpr int ACC = (2 * BN <= 512) ? 2 : 1;
  static constexpr int KG = BN >= 256 ? 1 : BN >= 128 ? 2 : 4;   // k-blocks per MMA-issuer wait
  static constexpr int COLS_NEED = ACC * BN;
  static constexpr int TMEM_COLS =
      COLS_NEED <= 32 ? 32 : COLS_NEED <= 64 ? 64 : COLS_NEED <= 128 ? 128 : COLS_NEED <= 256 ? 256 : 512;
  static constexpr int SMEM = STAGES * STAGE_BYTES + 1024 + 256;
  static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256, "BN");
  static_assert(STAGES >= KG + 1, "stages per issuer wait");
  static_assert(B_BYTES % 1024 == 0, "stage alignment");
};

// Bounded wait that ignores the abort flag (teardown of an aborted block).
__device__ __forceinline__ void mbar_wait_teardown(uint64_t* bar, uint32_t parity) {
  const unsigned long long t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) return;
  }
}

template <int BN>
__global__ void __launch_bounds__(192, 1) igemm_kernel(const __grid_constant__ GemmParams p) {
  using C = GemmCfg<BN>;
  using OutT = __nv_bfloat16;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::STAGES * C::A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + C::STAGES * C::B_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* acc_full = empty + C::STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = warp_id(), lane = lane_id();
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&p.tmA0);
    if (p.a_mode == 1) prefetch_tmap(&p.tmA1);
    prefetch_tmap(&p.tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // set-up done: from here on this grid reads its predecessor's outputs
  griddep_wait();
  griddep_trigger();
  const int num_tiles = p.m_tiles * p.n_tiles;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0;          // bit s: stage s has a load in flight
      uint32_t issued_par = 0;      // bit s: parity of that load's phase
      // Per-tile address work is hoisted out of the K loop: the producer is a
      // single thread and runtime divisions per K block would starve the MMAs.
      int ry_tab[3 * 16];             // input row of (kh, box i), -1 for zeros
      uint64_t stale_mask = 0;        // bit kh*16+i: box comes from the stale map
      for (int tile = blockIdx.x; tile < num_tiles && !*abort_flag; tile += gridDim.x) {
        const int mt = tile / p.n_tiles, nt = tile - mt * p.n_tiles;
        int c0 = 0;
        if (p.a_mode == 1) {
          const int tr = mt / p.tiles_w, tc = mt - tr * p.tiles_w;
          const int r0 = tr * p.R;
          c0 = tc * p.Wt;
          stale_mask = 0;
          for (int i = 0; i < p.R; ++i) {
            const int r = r0 + i;
            const int band = r / p.hb_out;
            const int lo = band * p.hb_in, hi = lo + p.hb_in;     // input rows of this band
            for (int kh = 0; kh < 3; ++kh) {
              const int rho = p.stride * r + kh - 1;
              int ry = rho;
              if (r >= p.Ho) {
                ry = -1;                                          // ragged tile row: zeros
              } else if (rho >= 0 && rho < p.H && (rho < lo || rho >= hi)) {
                if (p.mode == DP_MODE_DISPLACED) stale_mask |= 1ull << (kh * 16 + i);
                else if (p.mode == DP_MODE_NAIVE) ry = -1;        // invisible band
              }
              ry_tab[kh * 16 + i] = ry;
            }
          }
        }
        int kh = 0, kw = 0, cb = 0;
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.status)) goto producer_done;
          mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
          uint8_t* a_dst = sA + stage * C::A_BYTES;
          if (p.a_mode == 0) {
            tma_load_2d(a_dst, &p.tmA0, &full[stage], kb * C::BK, mt * 128);
          } else {
            int kx, cx;
            if (p.stride == 1) {
              kx = cb * C::BK;
              cx = c0 + kw - 1;
            } else {
              kx = (kw == 1 ? 0 : p.Cin) + cb * C::BK;
              cx = c0 - (kw == 0 ? 1 : 0);
            }
            const int* ryk = ry_tab + kh * 16;
            const uint32_t sk = static_cast<uint32_t>(stale_mask >> (kh * 16));
            for (int i = 0; i < p.R; ++i)
              tma_load_3d(a_dst + i * p.Wt * 128, ((sk >> i) & 1u) ? &p.tmA1 : &p.tmA0,
                          &full[stage], kx, cx, ryk[i]);
            if (++cb == p.kc) {
              cb = 0;
              if (++kw == 3) {
                kw = 0;
                ++kh;
              }
            }
          }
          tma_load_2d(sB + stage * C::B_BYTES, &p.tmB, &full[stage], kb * C::BK, nt * BN);
          issued |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    producer_done:
      if (*abort_flag) {
        // Let every load in flight land before the block's shared memory goes away.
        for (int s = 0; s < C::STAGES; ++s)
          if (issued & (1u << s)) mbar_wait_teardown(&full[s], (issued_par >> s) & 1u);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      constexpr uint32_t idesc = idesc_dense(128, BN, 1, 0, 0);
      const uint64_t a_desc0 = sdesc_sw128(smem_u32(sA), 1024);
      const uint64_t b_desc0 = sdesc_sw128(smem_u32(sB), 1024);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
        const int buf = C::ACC == 2 ? (it & 1) : 0;
        const int use = C::ACC == 2 ? (it >> 1) : it;
        if (!mbar_wait(&acc_empty[buf], (use & 1) ^ 1, abort_flag, p.status)) goto mma_done;
        tc_fence_after();
        const uint32_t d = tmem + buf * BN;
        // C::KG k-blocks per wait: MMA issue blocks until the pipe takes the
        // instruction, so the waits, fences and commits between k-blocks
        // leave the pipe idle unless enough MMAs are queued behind them.
        for (int kb = 0; kb < p.k_blocks;) {
          const int g = min(C::KG, p.k_blocks - kb);
          int st = stage;
          uint32_t ph = phase;
          for (int h = 0; h < g; ++h) {
            if (!mbar_wait(&full[st], ph, abort_flag, p.status)) goto mma_done;
            if (++st == C::STAGES) {
              st = 0;
              ph ^= 1u;
            }
          }
          tc_fence_after();
          st = stage;
          for (int h = 0; h < g; ++h) {
            const uint64_t ad = a_desc0 + static_cast<uint64_t>((st * C::A_BYTES) >> 4);
            const uint64_t bd = b_desc0 + static_cast<uint64_t>((st * C::B_BYTES) >> 4);
#pragma unroll
            for (int k = 0; k < 4; ++k) umma_f16_ss(d, ad + 2 * k, bd + 2 * k, idesc, ((kb + h) | k) != 0);
            if (++st == C::STAGES) st = 0;
          }
          for (int h = 0; h < g; ++h) {
            umma_commit(&empty[stage]);
            if (++stage == C::STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
          kb += g;
        }
        umma_commit(&acc_full[buf]);
      }
    mma_done:
      if (*abort_flag) {
        umma_commit(drain);
        mbar_wait_teardown(drain, 0);
      }
    }
  } else {
    // -------------------------------------------------------------- epilogue
    const int q = warp & 3;                 // TMEM lane quarter this warp can read
    const int row = q * 32 + lane;
    int it = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
      const int buf = C::ACC == 2 ? (it & 1) : 0;
      const int use = C::ACC == 2 ? (it >> 1) : it;
      if (!mbar_wait(&acc_full[buf], use & 1, abort_flag, p.status)) break;
      tc_fence_after();
      const int mt = tile / p.n_tiles, nt = tile - mt * p.n_tiles;
      bool valid;
      size_t pix;
      if (p.a_mode == 0) {
        const int m = mt * 128 + row;
        valid = m < p.M;
        pix = static_cast<size_t>(m);
      } else {
        const int tr = mt / p.tiles_w, tc = mt - tr * p.tiles_w;
        const int r = tr * p.R + row / p.Wt, c = tc * p.Wt + row % p.Wt;
        valid = r < p.Ho && c < p.Wo;
        pix = static_cast<size_t>(r) * p.Wo + c;
      }
      const int n0 = nt * BN;
      const int seg = n0 / p.split;
      OutT* outp = static_cast<OutT*>(seg == 0 ? p.out0 : seg == 1 ? p.out1 : p.out2);
      const int ncol0 = n0 - seg * p.split;
      OutT* orow = outp + pix * p.ld_out + ncol0;
      const OutT* rrow =
          p.residual ? static_cast<const OutT*>(p.residual) + pix * p.N + n0 : nullptr;
#pragma unroll 1
      for (int ch = 0; ch < BN / 32; ++ch) {
        uint32_t r[32];
        tmem_ld32(tmem + (static_cast<uint32_t>(q * 32) << 16) + buf * BN + ch * 32, r);
        tmem_wait_ld();
        if (ch == BN / 32 - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[buf]);
        }
        if (!valid) continue;
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
        if (p.bias) {
          const float4* b4 = reinterpret_cast<const float4*>(p.bias + n0 + ch * 32);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float4 b = __ldg(b4 + j);
            v[4 * j] += b.x;
            v[4 * j + 1] += b.y;
            v[4 * j + 2] += b.z;
            v[4 * j + 3] += b.w;
          }
        }
        if (rrow) {
          const uint4* r4 = reinterpret_cast<const uint4*>(rrow + ch * 32);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            uint4 u = r4[j];
            const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f = __bfloat1622float2(h[e]);
              v[8 * j + 2 * e] += f.x;
              v[8 * j + 2 * e + 1] += f.y;
            }
          }
        }
        uint4* o4 = reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint4 u;
          u.x = pack_bf16x2(v[8 * j], v[8 * j + 1]);
          u.y = pack_bf16x2(v[8 * j + 2], v[8 * j + 3]);
          u.z = pack_bf16x2(v[8 * j + 4], v[8 * j + 5]);
          u.w = pack_bf16x2(v[8 * j + 6], v[8 * j + 7]);
          o4[j] = u;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  __syncwarp();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// Pair kernel: two CTAs of a cluster share one 256 x (NI*NJ) output tile.
// Each CTA loads its own 128 rows of A and half of every NI-wide slice of B;
// the leader CTA issues tcgen05.mma.cta_group::2 (M = 256), which reads both
// CTAs' shared memory and writes each CTA's 128 accumulator rows into that
// CTA's tensor memory.  Per SM this halves the weight bytes per flop.
template <int NI, int NJ>
struct PairCfg {
  static constexpr int BN = NI * NJ;                 // output columns per pair tile
  static constexpr int A_BYTES = 128 * 128;
  static constexpr int BSUB_BYTES = (NI / 2) * 128;  // this CTA's half of one B slice
  static constexpr int B_BYTES = NJ * BSUB_BYTES;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES_RAW = (190 * 1024) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_RAW > 8 ? 8 : STAGES_RAW;
  // two accumulators when they fit: the epilogue of a tile overlaps the
  // main loop of the next
  static constexpr int ACC = 2 * BN <= 512 ? 2 : 1;
  static constexpr int TMEM_COLS = ACC * BN <= 128 ? 128 : ACC * BN <= 256 ? 256 : 512;
  static constexpr int EPI_SLOT = 32 * 64;          // 32 rows x 32 bf16 columns
  static constexpr int EPI_BYTES = 8 * 2 * EPI_SLOT;  // 8 warps x 2 output slots
  static constexpr int BIAS_BYTES = 8 * BN * 4;     // one fp32 copy per epilogue warp
  static constexpr int SMEM = STAGES * STAGE_BYTES + EPI_BYTES + BIAS_BYTES + 1024 + 256;
  static_assert(BSUB_BYTES % 1024 == 0, "B slice alignment");
  static_assert(SMEM <= 227 * 1024, "shared memory");
  static_assert(BN <= 512 && NI % 32 == 0 && NI <= 256, "tile");
};

constexpr int kEpiSlot = 32 * 64;   // one epilogue warp's 32 rows x 32 bf16 columns

// Shared-memory state of one epilogue warp of a pair kernel: finished chunks
// leave by TMA stores from two alternating slots.
struct PairEpi {
  uint8_t* out;      // 2 output slots
  float* bias;       // the tile's BN bias values
  uint32_t oi;       // output stores issued so far
};

// Byte offset of 16-byte chunk j of row i in a slot written with the 64-byte
// swizzle (chunk index XOR address bits 7-8): conflict-free row-per-lane access.
__device__ __forceinline__ uint32_t sw64_off(int i, int j) {
  return static_cast<uint32_t>(i * 64 + ((j ^ ((i >> 1) & 3)) << 4));
}

// Box of one epilogue warp: first column of its output segment (x), first
// pixel (y) and image row (z, convs), the output segment, and whether any of
// its rows is inside the output.
struct EpiBox {
  int x, y, z, seg;
  bool ok;
};
__device__ __forceinline__ EpiBox pair_epi_box(const GemmParams& p, int mt, int q, int n0) {
  EpiBox b;
  if (p.a_mode == 0) {
    b.seg = n0 / p.split;
    b.x = n0 - b.seg * p.split;
    b.y = mt * 128 + q * 32;
    b.z = 0;
    b.ok = mt < p.m_tiles && b.y < p.M;
  } else {
    const int tr = mt / p.tiles_w, tc = mt - tr * p.tiles_w;
    b.seg = 0;
    b.x = n0;
    b.z = tr * p.R + (q * 32) / p.Wt;
    b.y = tc * p.Wt + (q * 32) % p.Wt;
    b.ok = mt < p.m_tiles && b.z < p.Ho && b.y < p.Wo;
  }
  return b;
}

// Output pixel of accumulator row `row` of M tile mt, and whether it exists.
__device__ __forceinline__ bool pair_row_pixel(const GemmParams& p, int mt, int row, size_t* pix) {
  if (p.a_mode == 0) {
    const int m = mt * 128 + row;
    *pix = static_cast<size_t>(m);
    return mt < p.m_tiles && m < p.M;
  }
  const int tr = mt / p.tiles_w, tc = mt - tr * p.tiles_w;
  const int r = tr * p.R + row / p.Wt, c = tc * p.Wt + row % p.Wt;
  *pix = static_cast<size_t>(r) * p.Wo + c;
  return mt < p.m_tiles && r < p.Ho && c < p.Wo;
}

// Epilogue of one pair tile for one epilogue warp: this CTA's 128 accumulator
// rows (TMEM lane quarter q) are drained in 32-column chunks, two warps per
// lane quarter taking alternate chunks (half = 0: chunks 0, 2, ...; 1: 1, 3,
// ...); each warp hands the accumulator back to the leader after its last
// chunk.  Bias (staged in shared memory) and residual (each lane's row loaded
// one chunk ahead into registers) are added and the bf16 chunk is stored by
// TMA, ragged edges clipped by the tensor map.  Returns false when a wait gave
// up (the caller tears down).
template <int BN>
__device__ __forceinline__ bool pair_epilogue_tile(const GemmParams& p, uint32_t tmem, int q, int half,
                                                   int lane, uint32_t rank, int item, uint32_t parity,
                                                   uint64_t* acc_full, uint32_t acc_empty_leader,
                                                   volatile int* abort_flag, PairEpi& e) {
  constexpr int NCH = BN / 32;
  static_assert(NCH >= 2, "chunks");
  const int last_ch = ((NCH - 1 - half) / 2) * 2 + half;   // this warp's last chunk
  // hands the accumulator back after this warp's last chunk has been read
  auto release = [&](int ch) {
    if (ch == last_ch) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty_leader);
    }
  };
  const int tile = item / p.splits;
  // Split K: this run's accumulator goes to its fp32 partial, rows at their
  // output pixels; bias, residual and the cast are the finish kernel's.
  if (p.splits > 1) {
    const int run = item - tile * p.splits;
    const int mp = tile / p.n_tiles, nt = tile - mp * p.n_tiles;
    const int mt = 2 * mp + static_cast<int>(rank);
    size_t pix;
    const bool valid = pair_row_pixel(p, mt, q * 32 + lane, &pix);
    const size_t M = p.a_mode == 0 ? static_cast<size_t>(p.M) : static_cast<size_t>(p.Ho) * p.Wo;
    float* dst = p.part + static_cast<size_t>(run) * M * p.N + pix * p.N + nt * BN;
    if (!mbar_wait(acc_full, parity, abort_flag, p.status)) return false;
    tc_fence_after();
#pragma unroll 1
    for (int ch = half; ch < NCH; ch += 2) {
      uint32_t r[32];
      tmem_ld32(tmem + (static_cast<uint32_t>(q * 32) << 16) + ch * 32, r);
      tmem_wait_ld();
      release(ch);
      if (!valid) continue;
      float4* d4 = reinterpret_cast<float4*>(dst + ch * 32);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        d4[j] = make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                            __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]));
    }
    return true;
  }
  const int mp = tile / p.n_tiles, nt = tile - mp * p.n_tiles;
  const int mt = 2 * mp + static_cast<int>(rank);
  const int n0 = nt * BN;
  const EpiBox b = pair_epi_box(p, mt, q, n0);
  const uint4* rrow = nullptr;
  if (p.residual && b.ok) {
    size_t pix;
    if (pair_row_pixel(p, mt, q * 32 + lane, &pix))
      rrow = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.residual) + pix * p.N + n0);
  }
  // Staged while the MMA of this tile still runs: the bias row and this
  // lane's first residual chunk.  The previous tile's reads are finished.
  for (int i = lane; i < BN; i += 32) e.bias[i] = p.bias ? __ldg(p.bias + n0 + i) : 0.f;
  uint4 rv[4];
  if (rrow) {
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) rv[jj] = __ldg(rrow + half * 4 + jj);
  }
  __syncwarp();
  if (!mbar_wait(acc_full, parity, abort_flag, p.status)) return false;
  tc_fence_after();
  const CUtensorMap* om = &p.tmO[b.seg];
#pragma unroll 1
  for (int ch = half; ch < NCH; ch += 2) {
    float v[32];
    {
      uint32_t r[32];
      tmem_ld32(tmem + (static_cast<uint32_t>(q * 32) << 16) + ch * 32, r);
      tmem_wait_ld();
      release(ch);
      if (!b.ok) continue;
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
    }
    const float* bb = e.bias + ch * 32;
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] += bb[j];
    if (p.geglu) {
      // 16 outputs a * gelu(g) of this row: 32 bytes, one 16-column box
      uint8_t* ob = e.out + (e.oi & 1u) * kEpiSlot;
      if (lane == 0) bulk_wait_read_1();   // the store that last used this slot has read it
      __syncwarp();
      uint32_t o[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        o[j] = pack_bf16x2(v[2 * j] * gelu_exact(v[16 + 2 * j]), v[2 * j + 1] * gelu_exact(v[17 + 2 * j]));
      *reinterpret_cast<uint4*>(ob + lane * 32) = make_uint4(o[0], o[1], o[2], o[3]);
      *reinterpret_cast<uint4*>(ob + lane * 32 + 16) = make_uint4(o[4], o[5], o[6], o[7]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_2d(om, ob, (b.x + ch * 32) / 2, b.y);
        bulk_commit();
      }
      ++e.oi;
      continue;
    }
    if (rrow) {
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&rv[jj]);
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const float2 f = __bfloat1622float2(h[t]);
          v[8 * jj + 2 * t] += f.x;
          v[8 * jj + 2 * t + 1] += f.y;
        }
      }
      if (ch + 2 < NCH) {
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) rv[jj] = __ldg(rrow + (ch + 2) * 4 + jj);
      }
    }
    uint8_t* ob = e.out + (e.oi & 1u) * kEpiSlot;
    if (lane == 0) bulk_wait_read_1();   // the store that last used this slot has read it
    __syncwarp();
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      uint4 u;
      u.x = pack_bf16x2(v[8 * jj], v[8 * jj + 1]);
      u.y = pack_bf16x2(v[8 * jj + 2], v[8 * jj + 3]);
      u.z = pack_bf16x2(v[8 * jj + 4], v[8 * jj + 5]);
      u.w = pack_bf16x2(v[8 * jj + 6], v[8 * jj + 7]);
      *reinterpret_cast<uint4*>(ob + sw64_off(lane, jj)) = u;
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      if (p.a_mode == 0) tma_store_2d(om, ob, b.x + ch * 32, b.y);
      else if (p.out_evict_first) tma_store_3d_evict_first(om, ob, b.x + ch * 32, b.y, b.z, l2_evict_first_policy());
      else tma_store_3d(om, ob, b.x + ch * 32, b.y, b.z);
      bulk_commit();
    }
    ++e.oi;
  }
  return true;
}

template <int NI, int NJ>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(320, 1)
    igemm_pair_kernel(const __grid_constant__ GemmParams p) {
  using C = PairCfg<NI, NJ>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::STAGES * C::A_BYTES;
  uint8_t* sEpi = sB + C::STAGES * C::B_BYTES;
  float* sBias = reinterpret_cast<float*>(sEpi + C::EPI_BYTES);
  uint64_t* full = reinterpret_cast<uint64_t*>(sEpi + C::EPI_BYTES + C::BIAS_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* acc_full = empty + C::STAGES;   // [2]
  uint64_t* acc_empty = acc_full + 2;       // [2]
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = warp_id(), lane = lane_id();
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int num_tiles = ((p.m_tiles + 1) >> 1) * p.n_tiles;
  const int num_items = num_tiles * p.splits;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 16);   // 8 epilogue warps in each CTA
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&p.tmA0);
    if (p.a_mode == 1) prefetch_tmap(&p.tmA1);
    prefetch_tmap(&p.tmB);
    prefetch_tmap(&p.tmO[0]);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // set-up done: from here on this grid reads its predecessor's outputs
  griddep_wait();
  griddep_trigger();

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer (both CTAs)
      int stage = 0;
      uint32_t phase = 0;
      int ry_tab[3 * 16];
      uint64_t stale_mask = 0;
      const uint32_t full0 = mapa_shared(smem_u32(full), 0);   // leader's full[0]
      for (int item = pair; item < num_items && !*abort_flag; item += npairs) {
        const int tile = item / p.splits;
        int kbeg, kend;
        split_range(p.k_blocks, p.splits, item - tile * p.splits, &kbeg, &kend);
        const int mp = tile / p.n_tiles, nt = tile - mp * p.n_tiles;
        const int mt = 2 * mp + static_cast<int>(rank);
        int c0 = 0;
        if (p.a_mode == 1) {
          const int tr = mt / p.tiles_w, tc = mt - tr * p.tiles_w;
          const int r0 = tr * p.R;
          c0 = tc * p.Wt;
          stale_mask = 0;
          for (int i = 0; i < p.R; ++i) {
            const int r = r0 + i;
            const int band = r / p.hb_out;
            const int lo = band * p.hb_in, hi = lo + p.hb_in;
            for (int kh = 0; kh < 3; ++kh) {
              const int rho = p.stride * r + kh - 1;
              int ry = rho;
              if (r >= p.Ho) {
                ry = -1;
              } else if (rho >= 0 && rho < p.H && (rho < lo || rho >= hi)) {
                if (p.mode == DP_MODE_DISPLACED) stale_mask |= 1ull << (kh * 16 + i);
                else if (p.mode == DP_MODE_NAIVE) ry = -1;
              }
              ry_tab[kh * 16 + i] = ry;
            }
          }
        }
        int cb = kbeg % (p.kc > 0 ? p.kc : 1), kh = 0, kw = 0;
        if (p.a_mode == 1) {
          const int tap = kbeg / p.kc;
          kh = tap / 3;
          kw = tap - kh * 3;
        }
        for (int kb = kbeg; kb < kend; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.status)) goto producer_done;
          if (leader) mbar_arrive_expect_tx(&full[stage], 2 * C::STAGE_BYTES);
          const uint32_t fb = full0 + stage * 8;
          uint8_t* a_dst = sA + stage * C::A_BYTES;
          if (p.a_mode == 0) {
            tma_load_2d_pair(a_dst, &p.tmA0, fb, kb * 64, mt * 128);
          } else {
            int kx, cx;
            if (p.stride == 1) {
              kx = cb * 64;
              cx = c0 + kw - 1;
            } else {
              kx = (kw == 1 ? 0 : p.Cin) + cb * 64;
              cx = c0 - (kw == 0 ? 1 : 0);
            }
            const int* ryk = ry_tab + kh * 16;
            const uint32_t sk = static_cast<uint32_t>(stale_mask >> (kh * 16));
            for (int i = 0; i < p.R; ++i)
              tma_load_3d_pair(a_dst + i * p.Wt * 128, ((sk >> i) & 1u) ? &p.tmA1 : &p.tmA0, fb,
                               kx, cx, ryk[i]);
            if (++cb == p.kc) {
              cb = 0;
              if (++kw == 3) {
                kw = 0;
                ++kh;
              }
            }
          }
          uint8_t* b_dst = sB + stage * C::B_BYTES;
#pragma unroll
          for (int j = 0; j < NJ; ++j)
            tma_load_2d_pair(b_dst + j * C::BSUB_BYTES, &p.tmB, fb, kb * 64,
                             nt * C::BN + j * NI + static_cast<int>(rank) * (NI / 2));
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    producer_done:
      if (*abort_flag) {
        // Loads in flight complete on the leader's barrier; give them time to land.
        const unsigned long long t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 2000000ull) {
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ------------------------------------------------------------ MMA issuer (leader CTA)
      constexpr uint32_t idesc = idesc_dense(256, NI, 1, 0, 0);
      const uint64_t a_desc0 = sdesc_sw128(smem_u32(sA), 1024);
      const uint64_t b_desc0 = sdesc_sw128(smem_u32(sB), 1024);
      const uint32_t empty_own = smem_u32(empty), empty_peer = mapa_shared(smem_u32(empty), 1);
      const uint32_t accf_own = smem_u32(acc_full), accf_peer = mapa_shared(smem_u32(acc_full), 1);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      for (int item = pair; item < num_items; item += npairs, ++it) {
        const int tile = item / p.splits;
        int kbeg, kend;
        split_range(p.k_blocks, p.splits, item - tile * p.splits, &kbeg, &kend);
        const int buf = C::ACC == 2 ? (it & 1) : 0;
        const int use = C::ACC == 2 ? (it >> 1) : it;
        if (!mbar_wait(&acc_empty[buf], (use & 1) ^ 1, abort_flag, p.status)) goto mma_done;
        tc_fence_after();
        const uint32_t dacc = tmem + buf * C::BN;
        // Two k-blocks per wait: tcgen05.mma issue blocks until the pipe
        // takes the instruction, so the wait, fence and commits between
        // k-blocks leave the pipe idle unless enough MMAs are queued behind
        // them (measured: 8 MMAs of 256x160x16 per wait run at 88 % of the
        // pipe, 16 per wait at 100 %).
        for (int kb = kbeg; kb < kend;) {
          const int nb = kend - kb >= 2 ? 2 : 1;
          int stage2 = stage + 1;
          uint32_t phase2 = phase;
          if (stage2 == C::STAGES) {
            stage2 = 0;
            phase2 ^= 1u;
          }
          if (!mbar_wait(&full[stage], phase, abort_flag, p.status) ||
              (nb == 2 && !mbar_wait(&full[stage2], phase2, abort_flag, p.status)))
            goto mma_done;
          tc_fence_after();
          const uint64_t ad = a_desc0 + static_cast<uint64_t>((stage * C::A_BYTES) >> 4);
          const uint64_t bd = b_desc0 + static_cast<uint64_t>((stage * C::B_BYTES) >> 4);
          if (nb == 2) {
            const uint64_t ad2 = a_desc0 + static_cast<uint64_t>((stage2 * C::A_BYTES) >> 4);
            const uint64_t bd2 = b_desc0 + static_cast<uint64_t>((stage2 * C::B_BYTES) >> 4);
#pragma unroll
            for (int k = 0; k < 4; ++k)
#pragma unroll
              for (int j = 0; j < NJ; ++j)
                umma_f16_ss_pair(dacc + j * NI, ad + 2 * k,
                                 bd + static_cast<uint64_t>((j * C::BSUB_BYTES) >> 4) + 2 * k, idesc,
                                 (kb != kbeg || k != 0));
#pragma unroll
            for (int k = 0; k < 4; ++k)
#pragma unroll
              for (int j = 0; j < NJ; ++j)
                umma_f16_ss_pair(dacc + j * NI, ad2 + 2 * k,
                                 bd2 + static_cast<uint64_t>((j * C::BSUB_BYTES) >> 4) + 2 * k, idesc, 1u);
            umma_commit_pair(empty_own + stage * 8);
            umma_commit_pair(empty_peer + stage * 8);
            umma_commit_pair(empty_own + stage2 * 8);
            umma_commit_pair(empty_peer + stage2 * 8);
          } else {
#pragma unroll
            for (int k = 0; k < 4; ++k)
#pragma unroll
              for (int j = 0; j < NJ; ++j)
                umma_f16_ss_pair(dacc + j * NI, ad + 2 * k,
                                 bd + static_cast<uint64_t>((j * C::BSUB_BYTES) >> 4) + 2 * k, idesc,
                                 (kb != kbeg || k != 0));
            umma_commit_pair(empty_own + stage * 8);
            umma_commit_pair(empty_peer + stage * 8);
          }
          kb += nb;
          stage = nb == 2 ? stage2 : stage;
          phase = nb == 2 ? phase2 : phase;
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        umma_commit_pair(accf_own + buf * 8);
        umma_commit_pair(accf_peer + buf * 8);
      }
    mma_done:
      if (*abort_flag) {
        umma_commit_pair(smem_u32(drain));
        mbar_wait_teardown(drain, 0);
      }
    }
  } else {
    // -------------------------------------------------------------- epilogue (both CTAs)
    const int q = warp & 3;
    const uint32_t acc_empty_leader = mapa_shared(smem_u32(acc_empty), 0);   // [2], 8 bytes apart
    const int ew = warp - 2, half = ew >> 2;
    PairEpi e;
    e.out = sEpi + ew * 2 * kEpiSlot;
    e.bias = sBias + ew * C::BN;
    e.oi = 0;
    int it = 0;
    for (int item = pair; item < num_items; item += npairs, ++it) {
      const int buf = C::ACC == 2 ? (it & 1) : 0;
      const int use = C::ACC == 2 ? (it >> 1) : it;
      if (!pair_epilogue_tile<C::BN>(p, tmem + buf * C::BN, q, half, lane, rank, item,
                                     static_cast<uint32_t>(use & 1), &acc_full[buf],
                                     acc_empty_leader + buf * 8, abort_flag, e))
        break;
    }
    if (lane == 0) bulk_wait_all();   // every store has finished reading its slot
  }

  tc_fence_before();
  cluster_sync_all();
  __syncwarp();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// GroupNorm-fused pair conv: the 3x3 conv of GroupNorm(x) (+SiLU) whose A
// operand is normalised in shared memory, so the normalised activations are
// never written to or read back from HBM ("DistriFusion", atlas.scime.ai
// summary, Approach: the corrected GroupNorm feeds the next layer; study.space
// summary, Method: other bands' rows are the previous step's activations).
//
// Tiles are one output row r x 128 columns (stride 1).  K runs channel block
// by channel block (64 channels), and for each block the three input rows
// r-1, r, r+1 are staged once by TMA, 130 pixels each (the tile plus one
// column of halo on each side), in 128-byte-swizzled rows 136 pixels apart.
// The nine taps are then nine shifted views of that one staging: tap (kh, kw)
// starts kh rows and kw pixels in, and the tensor core applies the swizzle to
// the absolute shared-memory address, so a shifted view reads the bytes the
// TMA wrote.  Each staged row comes from
//   * x, the raw input, when it lies in the tile's band (or in any band in a
//     sync step): the transform warps normalise it in place with that band's
//     scale and shift (exactly the GroupNorm apply pass's arithmetic);
//   * the stale normalised activations, when it lies in another band in a
//     displaced step (already normalised: left as loaded);
//   * nowhere (zero fill) outside the image or for another band in a naive
//     step; zero-filled columns outside the image stay zero.
// The transform warps also write the tile's own row, normalised, to a_next
// when it is the first or last row of its band: those are the only rows the
// next step's displaced conv reads from another band, so a_next serves as the
// next step's stale buffer without a full write.
//
// Cost on B200 at the SDXL shapes: every input row is normalised three times
// (once in each row window that reads it), and the in-place pass adds a read
// and a write of every staged byte to a shared memory whose bandwidth the
// tensor core's operand reads and the weight loads already nearly fill.  The
// separate GroupNorm pass plus the plain conv is faster there, so the block
// step takes this kernel only when asked to (dp_block_desc_set_gn_fusion).
//
// Roles (576 threads): warp 0 B producer, warp 1 MMA issuer (leader CTA),
// warps 2-9 epilogue (as in igemm_pair_kernel), warps 10-17 transform (warp
// 10 lane 0 also issues the A row loads).
template <int NJ>
struct GnConvCfg {
  static constexpr int NI = 160;
  static constexpr int BN = NI * NJ;
  static constexpr int ROW_PX = 130;                 // staged pixels per row
  static constexpr int ROW_PITCH = 136 * 128;        // bytes between staged rows (1 KiB multiple)
  static constexpr int A_BYTES = 3 * ROW_PITCH;      // one stage: rows r-1, r, r+1
  static constexpr int A_TX = 3 * ROW_PX * 128;      // bytes the three row loads deliver
  static constexpr int A_STAGES = 2;
  static constexpr int XF_WARPS = 8;                 // staging / transform warps per CTA
  static constexpr int BSUB_BYTES = (NI / 2) * 128;  // this CTA's half of one B slice
  static constexpr int B_BYTES = NJ * BSUB_BYTES;
  static constexpr int B_STAGES = NJ == 2 ? 4 : 6;
  static constexpr int ACC = 2 * BN <= 512 ? 2 : 1;
  static constexpr int TMEM_COLS = ACC * BN <= 256 ? 256 : 512;
  static constexpr int EPI_BYTES = 8 * 2 * kEpiSlot;
  static constexpr int BIAS_BYTES = 8 * BN * 4;
  static constexpr int THREADS = 320 + 32 * XF_WARPS;
  static constexpr int SMEM =
      A_STAGES * A_BYTES + B_STAGES * B_BYTES + EPI_BYTES + BIAS_BYTES + 1024 + 512;
  static_assert(SMEM <= 227 * 1024, "shared memory");
  static_assert(ROW_PITCH % 1024 == 0 && A_BYTES % 1024 == 0 && B_BYTES % 1024 == 0, "alignment");
};

// Where staged row kh (input row r - 1 + kh) of M tile mt comes from: 0 zero
// fill, 1 the raw input (normalised with band *band), 2 the stale normalised
// activations.  *rho is the input row.
__device__ __forceinline__ int gn_row_source(const GemmParams& p, int mt, int kh, int* rho, int* band) {
  if (mt >= p.m_tiles) return 0;
  const int r = mt / p.tiles_w;
  const int rr = r + kh - 1;
  *rho = rr;
  if (rr < 0 || rr >= p.H) return 0;
  const int own = r / p.hb_in, other = rr / p.hb_in;
  *band = other;
  if (other == own || p.mode == DP_MODE_SYNC) return 1;
  return p.mode == DP_MODE_DISPLACED ? 2 : 0;
}

// Scale and shift of the eight channels [c_base, c_base + 8) for band `band`
// (gamma and beta read as 16-byte vectors; c_base is a multiple of 8).
__device__ __forceinline__ void gn_chunk_scale_shift(const GemmParams& p, int band, int c_base,
                                                     float (&sc)[8], float (&sh)[8]) {
  const float4 g0 = __ldg(reinterpret_cast<const float4*>(p.gn_gamma + c_base));
  const float4 g1 = __ldg(reinterpret_cast<const float4*>(p.gn_gamma + c_base) + 1);
  const float4 b0 = __ldg(reinterpret_cast<const float4*>(p.gn_beta + c_base));
  const float4 b1 = __ldg(reinterpret_cast<const float4*>(p.gn_beta + c_base) + 1);
  const float gm[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
  const float bt[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
  const float* u = p.gn_used + 2 * band * (p.Cin / p.gn_cg);
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const int g = (c_base + e) / p.gn_cg;
    gn_scale_shift(__ldg(u + 2 * g), __ldg(u + 2 * g + 1), p.gn_eps, gm[e], bt[e], &sc[e], &sh[e]);
  }
}

template <int NJ>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(GnConvCfg<NJ>::THREADS, 1)
    igemm_gn_pair_kernel(const __grid_constant__ GemmParams p) {
  using C = GnConvCfg<NJ>;
  constexpr int NI = C::NI;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + C::A_STAGES * C::A_BYTES;
  uint8_t* sEpi = sB + C::B_STAGES * C::B_BYTES;
  float* sBias = reinterpret_cast<float*>(sEpi + C::EPI_BYTES);
  uint64_t* a_loaded = reinterpret_cast<uint64_t*>(sEpi + C::EPI_BYTES + C::BIAS_BYTES);  // [A_STAGES]
  uint64_t* a_ready = a_loaded + C::A_STAGES;   // [A_STAGES], the leader's count both CTAs
  uint64_t* a_empty = a_ready + C::A_STAGES;    // [A_STAGES]
  uint64_t* b_full = a_empty + C::A_STAGES;     // [B_STAGES], the leader's count both CTAs
  uint64_t* b_empty = b_full + C::B_STAGES;     // [B_STAGES]
  uint64_t* acc_full = b_empty + C::B_STAGES;   // [2]
  uint64_t* acc_empty = acc_full + 2;           // [2]
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = warp_id(), lane = lane_id();
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int num_items = ((p.m_tiles + 1) >> 1) * p.n_tiles;
  const int kc = p.kc;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::A_STAGES; ++s) {
      mbar_init(&a_loaded[s], 1);
      mbar_init(&a_ready[s], 2 * C::XF_WARPS);   // the transform warps of both CTAs
      mbar_init(&a_empty[s], 1);
    }
    for (int s = 0; s < C::B_STAGES; ++s) {
      mbar_init(&b_full[s], 1);
      mbar_init(&b_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 16);  // 8 epilogue warps in each CTA
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&p.tmA0);
    prefetch_tmap(&p.tmA1);
    prefetch_tmap(&p.tmB);
    prefetch_tmap(&p.tmO[0]);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_wait();
  griddep_trigger();

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ B producer (both CTAs)
      int stage = 0;
      uint32_t phase = 0;
      const uint32_t full0 = mapa_shared(smem_u32(b_full), 0);   // leader's b_full[0]
      for (int item = pair; item < num_items && !*abort_flag; item += npairs) {
        const int nt = item % p.n_tiles;
        for (int cb = 0; cb < kc; ++cb) {
          for (int tap = 0; tap < 9; ++tap) {
            if (!mbar_wait(&b_empty[stage], phase ^ 1u, abort_flag, p.status)) goto b_done;
            if (leader) mbar_arrive_expect_tx(&b_full[stage], 2 * C::B_BYTES);
            const uint32_t fb = full0 + stage * 8;
            uint8_t* b_dst = sB + stage * C::B_BYTES;
#pragma unroll
            for (int j = 0; j < NJ; ++j)
              tma_load_2d_pair(b_dst + j * C::BSUB_BYTES, &p.tmB, fb, tap * p.Cin + cb * 64,
                               nt * C::BN + j * NI + static_cast<int>(rank) * (NI / 2));
            if (++stage == C::B_STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
      }
    b_done:;
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ------------------------------------------------------------ MMA issuer (leader CTA)
      constexpr uint32_t idesc = idesc_dense(256, NI, 1, 0, 0);
      const uint64_t b_desc0 = sdesc_sw128(smem_u32(sB), 1024);
      const uint32_t a_base = smem_u32(sA);
      const uint32_t bempty_own = smem_u32(b_empty), bempty_peer = mapa_shared(smem_u32(b_empty), 1);
      const uint32_t aempty_own = smem_u32(a_empty), aempty_peer = mapa_shared(smem_u32(a_empty), 1);
      const uint32_t accf_own = smem_u32(acc_full), accf_peer = mapa_shared(smem_u32(acc_full), 1);
      int bs = 0, as = 0;
      uint32_t bph = 0, aph = 0;
      int it = 0;
      for (int item = pair; item < num_items; item += npairs, ++it) {
        const int buf = C::ACC == 2 ? (it & 1) : 0;
        const int use = C::ACC == 2 ? (it >> 1) : it;
        if (!mbar_wait(&acc_empty[buf], (use & 1) ^ 1, abort_flag, p.status)) goto mma_done;
        tc_fence_after();
        const uint32_t dacc = tmem + buf * C::BN;
        for (int cb = 0; cb < kc; ++cb) {
          if (!mbar_wait(&a_ready[as], aph, abort_flag, p.status)) goto mma_done;
          tc_fence_after();
          const uint32_t a_stage = a_base + as * C::A_BYTES;
          // taps in pairs (0,1) (2,3) (4,5) (6,7), then 8: one wait for two
          // B stages keeps enough MMAs queued behind the wait
          for (int tap = 0; tap < 9;) {
            const int nb = tap < 8 ? 2 : 1;
            int bs2 = bs + 1;
            uint32_t bph2 = bph;
            if (bs2 == C::B_STAGES) {
              bs2 = 0;
              bph2 ^= 1u;
            }
            if (!mbar_wait(&b_full[bs], bph, abort_flag, p.status) ||
                (nb == 2 && !mbar_wait(&b_full[bs2], bph2, abort_flag, p.status)))
              goto mma_done;
            tc_fence_after();
#pragma unroll 1
            for (int t = 0; t < nb; ++t) {
              const int tp = tap + t;
              const int kh = tp / 3, kw = tp - 3 * (tp / 3);
              const uint64_t ad = sdesc_sw128(a_stage + kh * C::ROW_PITCH + kw * 128, 1024);
              const int sb = t == 0 ? bs : bs2;
              const uint64_t bd = b_desc0 + static_cast<uint64_t>((sb * C::B_BYTES) >> 4);
#pragma unroll
              for (int k = 0; k < 4; ++k)
#pragma unroll
                for (int j = 0; j < NJ; ++j)
                  umma_f16_ss_pair(dacc + j * NI, ad + 2 * k,
                                   bd + static_cast<uint64_t>((j * C::BSUB_BYTES) >> 4) + 2 * k, idesc,
                                   (cb != 0 || tp != 0 || k != 0));
            }
            umma_commit_pair(bempty_own + bs * 8);
            umma_commit_pair(bempty_peer + bs * 8);
            if (nb == 2) {
              umma_commit_pair(bempty_own + bs2 * 8);
              umma_commit_pair(bempty_peer + bs2 * 8);
            }
            tap += nb;
            bs = nb == 2 ? bs2 : bs;
            bph = nb == 2 ? bph2 : bph;
            if (++bs == C::B_STAGES) {
              bs = 0;
              bph ^= 1u;
            }
          }
          umma_commit_pair(aempty_own + as * 8);
          umma_commit_pair(aempty_peer + as * 8);
          if (++as == C::A_STAGES) {
            as = 0;
            aph ^= 1u;
          }
        }
        umma_commit_pair(accf_own + buf * 8);
        umma_commit_pair(accf_peer + buf * 8);
      }
    mma_done:
      if (*abort_flag) {
        umma_commit_pair(smem_u32(drain));
        mbar_wait_teardown(drain, 0);
      }
    }
  } else if (warp < 10) {
    // -------------------------------------------------------------- epilogue (both CTAs)
    const int q = warp & 3;
    const uint32_t acc_empty_leader = mapa_shared(smem_u32(acc_empty), 0);
    const int ew = warp - 2, half = ew >> 2;
    PairEpi e;
    e.out = sEpi + ew * 2 * kEpiSlot;
    e.bias = sBias + ew * C::BN;
    e.oi = 0;
    int it = 0;
    for (int item = pair; item < num_items; item += npairs, ++it) {
      const int buf = C::ACC == 2 ? (it & 1) : 0;
      const int use = C::ACC == 2 ? (it >> 1) : it;
      if (!pair_epilogue_tile<C::BN>(p, tmem + buf * C::BN, q, half, lane, rank, item,
                                     static_cast<uint32_t>(use & 1), &acc_full[buf],
                                     acc_empty_leader + buf * 8, abort_flag, e))
        break;
    }
    if (lane == 0) bulk_wait_all();
  } else {
    // -------------------------------------------------------------- A staging + transform (both CTAs)
    const int t = threadIdx.x - 320;             // 0 .. 32 * XF_WARPS - 1
    constexpr int PXL = 4 * C::XF_WARPS;         // pixel lanes: 8 chunk lanes x PXL = the threads
    const int j = t & 7, pl = t >> 3;            // 16-byte channel chunk, pixel lane
    const uint32_t ready_leader = mapa_shared(smem_u32(a_ready), 0);
    constexpr int NPX = (C::ROW_PX + PXL - 1) / PXL;   // chunks of one staged row per thread
    // the three row loads of step (item, cb) into stage s (warp 10, lane 0)
    auto issue = [&](int item, int cb, int st) {
      const int mt = 2 * (item / p.n_tiles) + static_cast<int>(rank);
      const int c0 = (mt % p.tiles_w) * 128;
      uint8_t* dst = sA + st * C::A_BYTES;
      mbar_arrive_expect_tx(&a_loaded[st], C::A_TX);
      for (int kh = 0; kh < 3; ++kh) {
        int rho = -1, band = 0;
        const int src = gn_row_source(p, mt, kh, &rho, &band);
        tma_load_3d(dst + kh * C::ROW_PITCH, src == 2 ? &p.tmA1 : &p.tmA0, &a_loaded[st], cb * 64,
                    c0 - 1, src == 0 ? -1 : rho);
      }
    };
    // the first A_STAGES steps go out at once; later ones when the MMA frees
    // the stage of the step before the one being transformed
    int pre_item = pair, pre_cb = 0;
    auto advance = [&]() {
      if (++pre_cb == kc) {
        pre_cb = 0;
        pre_item += npairs;
      }
    };
    if (warp == 10 && lane == 0) {
      for (int k = 0; k < C::A_STAGES && pre_item < num_items; ++k) {
        issue(pre_item, pre_cb, k);
        advance();
      }
    }
    int s = 0;
    uint32_t ph = 0;
    int seq = 0;   // (item, cb) steps transformed so far
    for (int item = pair; item < num_items && !*abort_flag; item += npairs) {
      const int mt = 2 * (item / p.n_tiles) + static_cast<int>(rank);
      const int nt = item % p.n_tiles;
      const int r = mt / p.tiles_w, c0 = (mt % p.tiles_w) * 128;
      const bool edge = p.a_next && nt == 0 && mt < p.m_tiles &&
                        (r % p.hb_in == 0 || r % p.hb_in == p.hb_in - 1);
      const int own_band = r / p.hb_in;
      for (int cb = 0; cb < kc; ++cb) {
        const int c_base = cb * 64 + j * 8;      // first channel of this thread's chunk
        // the own band's scale and shift, fetched while the rows arrive
        VecApply<__nv_bfloat16> ap_own;
        {
          float sc[8], sh[8];
          gn_chunk_scale_shift(p, own_band, c_base, sc, sh);
          ap_own = VecApply<__nv_bfloat16>(sc, sh);
        }
        if (!mbar_wait(&a_loaded[s], ph, abort_flag, p.status)) goto xf_done;
        uint8_t* stage = sA + s * C::A_BYTES;
#pragma unroll 1
        for (int kh = 0; kh < 3; ++kh) {
          int rho = -1, band = 0;
          if (gn_row_source(p, mt, kh, &rho, &band) != 1) continue;   // stale or zero: as loaded
          VecApply<__nv_bfloat16> ap = ap_own;
          if (band != own_band) {                           // a sync step's halo row
            float osc[8], osh[8];
            gn_chunk_scale_shift(p, band, c_base, osc, osh);
            ap = VecApply<__nv_bfloat16>(osc, osh);
          }
          uint8_t* row = stage + kh * C::ROW_PITCH;
          const bool write_edge = edge && kh == 1;
          __nv_bfloat16* nrow = write_edge ? static_cast<__nv_bfloat16*>(p.a_next) +
                                                 static_cast<size_t>(r) * p.W * p.Cin + c_base
                                           : nullptr;
          // this thread's chunks of the row: all loads first, then normalise
          // in place (zero-filled padding columns stay zero)
          uint4 v[NPX];
#pragma unroll
          for (int i = 0; i < NPX; ++i) {
            const int px = pl + PXL * i;
            if (px < C::ROW_PX) v[i] = *reinterpret_cast<const uint4*>(row + px * 128 + ((j ^ (px & 7)) << 4));
          }
#pragma unroll
          for (int i = 0; i < NPX; ++i) {
            const int px = pl + PXL * i, c = c0 - 1 + px;
            if (px >= C::ROW_PX || c < 0 || c >= p.W) continue;
            const uint4 y = ap.apply(v[i], p.gn_silu);
            *reinterpret_cast<uint4*>(row + px * 128 + ((j ^ (px & 7)) << 4)) = y;
            if (write_edge && px >= 1 && px <= 128)
              *reinterpret_cast<uint4*>(nrow + static_cast<size_t>(c) * p.Cin) = y;
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(ready_leader + s * 8);
        // the next load goes into the stage of the step before this one, once
        // the MMA (running while this step was transformed) is done with it;
        // warp 10 leaves together if that wait gives up
        if (warp == 10 && seq >= 1) {
          int ok = 1;
          if (lane == 0 && pre_item < num_items) {
            const int st = (seq + 1) % C::A_STAGES;
            ok = mbar_wait(&a_empty[st], static_cast<uint32_t>(((seq + 1) / C::A_STAGES - 1) & 1),
                           abort_flag, p.status);
            if (ok) {
              issue(pre_item, pre_cb, st);
              advance();
            }
          }
          if (!__shfl_sync(0xffffffffu, ok, 0)) goto xf_done;
        }
        ++seq;
        if (++s == C::A_STAGES) {
          s = 0;
          ph ^= 1u;
        }
      }
    }
  xf_done:
    if (*abort_flag && warp == 10 && lane == 0) {
      // row loads in flight land in this CTA's stages: give them time
      const unsigned long long t0 = globaltimer_ns();
      while (globaltimer_ns() - t0 < 2000000ull) {
      }
    }
  }

  tc_fence_before();
  cluster_sync_all();
  __syncwarp();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, C::TMEM_COLS);
  }
}

// Tensor maps of a pair kernel's epilogue: each epilogue warp stores boxes of
// 32 channels x its 32 output rows with the 64-byte swizzle.  Conv outputs
// are [Ho][Wo][Cout] (a warp's rows span min(Wt, 32) pixels x 32 / min(Wt, 32)
// image rows); plain outputs are [M][ld_out] per column segment.
static int encode_conv_epilogue(GemmParams& p, void* out, int Cout) {
  const uint32_t bw = static_cast<uint32_t>(std::min(p.Wt, 32));
  uint64_t dims[3] = {static_cast<uint64_t>(Cout), static_cast<uint64_t>(p.Wo),
                      static_cast<uint64_t>(p.Ho)};
  uint64_t str[2] = {static_cast<uint64_t>(Cout) * 2, static_cast<uint64_t>(p.Wo) * Cout * 2};
  uint32_t box[3] = {32, bw, 32 / bw};
  return encode_tmap(&p.tmO[0], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, out, dims, str, box,
                     CU_TENSOR_MAP_SWIZZLE_64B);
}

static int encode_linear_epilogue(GemmParams& p, void* const outs[3]) {
  uint32_t box[2] = {32, 32};
  for (int sgi = 0; sgi < p.N / p.split; ++sgi) {
    uint64_t dims[2] = {static_cast<uint64_t>(p.split), static_cast<uint64_t>(p.M)};
    uint64_t str[1] = {static_cast<uint64_t>(p.ld_out) * 2};
    int rc = encode_tmap(&p.tmO[sgi], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, outs[sgi], dims, str, box,
                         CU_TENSOR_MAP_SWIZZLE_64B);
    if (rc) return rc;
  }
  return DP_OK;
}

template <int NI, int NJ>
static int launch_pair(const GemmParams& p, cudaStream_t s) {
  using C = PairCfg<NI, NJ>;
  static int grid_cache[32] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  int& maxg = grid_cache[dev & 31];
  if (!maxg) {
    int rc = cuda_check(cudaFuncSetAttribute(igemm_pair_kernel<NI, NJ>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM),
                        "pair gemm smem attribute");
    if (rc) return rc;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 2;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.gridDim = dim3(2 * num_sms());
    cfg.blockDim = dim3(320);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, igemm_pair_kernel<NI, NJ>, &cfg) != cudaSuccess ||
        clusters <= 0) {
      cudaGetLastError();
      clusters = num_sms() / 2;
    }
    maxg = 2 * clusters;
  }
  const int pair_tiles = ((p.m_tiles + 1) / 2) * p.n_tiles * p.splits;
  const int grid = std::min(2 * pair_tiles, maxg);
  mark_launch(s);
  return launch_kernel(igemm_pair_kernel<NI, NJ>, dim3(grid), dim3(320), C::SMEM, s, false,
                       "pair gemm launch", p);
}

template <int BN>
static int launch_t(const GemmParams& p, cudaStream_t s) {
  using C = GemmCfg<BN>;
  static int attr_dev_mask = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  if (!(attr_dev_mask & (1 << (dev & 31)))) {
    int rc = cuda_check(cudaFuncSetAttribute(igemm_kernel<BN>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM),
                        "gemm smem attribute");
    if (rc) return rc;
    attr_dev_mask |= 1 << (dev & 31);
  }
  const int tiles = p.m_tiles * p.n_tiles;
  const int grid = std::min(tiles, num_sms());
  mark_launch(s);
  return launch_kernel(igemm_kernel<BN>, dim3(grid), dim3(192), C::SMEM, s, false,
                       "gemm launch", p);
}

static int launch_gemm(const GemmParams& p, int BN, cudaStream_t s) {
  switch (BN) {
    case 32: return launch_t<32>(p, s);
    case 64: return launch_t<64>(p, s);
    case 96: return launch_t<96>(p, s);
    case 128: return launch_t<128>(p, s);
    case 160: return launch_t<160>(p, s);
    case 192: return launch_t<192>(p, s);
    case 256: return launch_t<256>(p, s);
    default: break;
  }
  return set_error(DP_ERR_UNSUPPORTED, "gemm: no kernel for BN=%d", BN);
}

// Tile width in N: the candidate that divides `split` with the fewest
// wave-quantised columns per SM (a small per-tile cost favours wider tiles).
static int pick_bn(int m_tiles, int N, int split) {
  static const int c[] = {256, 192, 160, 128, 96, 64, 32};
  const int nc = 7;
  int best = 0;
  long best_cost = 0;
  for (int i = 0; i < nc; ++i) {
    const int bn = c[i];
    if (split % bn) continue;
    const long tiles = static_cast<long>(m_tiles) * (N / bn);
    const long waves = (tiles + num_sms() - 1) / num_sms();
    const long cost = waves * (bn + 32);
    if (!best || cost < best_cost) {
      best = bn;
      best_cost = cost;
    }
  }
  return best;
}

// Tile choice for bf16 work: 256x320 or 256x160 pair tiles, or a 128-row
// single-CTA tile.  Estimated time = waves x per-SM work of one tile / the
// relative efficiency measured for that tile (pair tiles move half the
// weight bytes per flop).  Returns the pair width (320 or 160) or 0.
// Operand fill limits these kernels: per SM, TMA brings about 55 bytes per
// cycle into shared memory (measured), so a k-block of a tile with `cols`
// MMA columns per SM and `b_rows` weight rows staged per SM takes
// max(2 cols, (16 KiB of A + 128 b_rows) / 55) cycles.
static double kblock_cycles(int cols, int b_rows) {
  const double mma = 2.0 * cols, fill = (16384.0 + 128.0 * b_rows) / 55.0;
  return mma > fill ? mma : fill;
}

// Pair tile width (0 = single-CTA tiles) and the number of K runs, from a
// cycle model: waves x (k-blocks x kblock_cycles + 5000 per wave for pipeline
// fill and epilogue); split K (only with a workspace) cuts K into runs of at
// least 8 k-blocks, keeps all (tile, run) items in one wave and pays about
// 16000 cycles for the finish kernel (measured 8-10 us).
static int pick_pair(int m_tiles, int N, int split, int kb, bool can_split, int* bn_single,
                     int* splits) {
  const long sms = num_sms(), pairs = sms / 2;
  const long mp = (m_tiles + 1) / 2;
  double best = 0.0;
  int choice = 0;
  *splits = 1;
  for (int width : {320, 160}) {
    if (split % width) continue;
    const long tiles = mp * (N / width);
    const double per = kblock_cycles(width, width / 2);
    for (int S = 1; S <= 16; ++S) {
      if (S > 1 && (!can_split || kb / S < 8 || tiles * S > pairs)) break;
      const double t = static_cast<double>((tiles * S + pairs - 1) / pairs) *
                           (((kb + S - 1) / S) * per + 5000.0) + (S > 1 ? 16000.0 : 0.0);
      if (!choice || t < best) {
        best = t;
        choice = width;
        *splits = S;
      }
    }
  }
  *bn_single = pick_bn(m_tiles, N, split);
  if (*bn_single) {
    const long tiles = static_cast<long>(m_tiles) * (N / *bn_single);
    const double t = static_cast<double>((tiles + sms - 1) / sms) *
                     (kb * kblock_cycles(*bn_single, *bn_single) + 5000.0);
    if (!choice || t < best) {
      choice = 0;
      *splits = 1;
    }
  }
  return choice;
}

// Split-K workspace: the fp32 partials of all runs, each laid out like the
// output.  Runs x rows x columns never exceed one wave of 256 x 320 pair tiles.
size_t gemm_workspace_bytes() {
  const size_t pairs = static_cast<size_t>(num_sms()) / 2;
  return pairs * 2 * 128 * 320 * sizeof(float);
}

static void set_split(GemmParams& p, int splits, void* workspace) {
  p.splits = splits;
  if (splits > 1) p.part = static_cast<float*>(workspace);
}

// out[m][n] = sum over runs of part[run][m][n] + bias[n] (+ residual[m][n]),
// cast to bf16 into output segment n / split.  8 columns per thread, runs
// added in order (the result does not depend on which run finished first).
__global__ void __launch_bounds__(256) splitk_finish_kernel(
    const float* __restrict__ part, int runs, int M, int N, int split, int ld_out,
    const float* __restrict__ bias, const __nv_bfloat16* __restrict__ residual,
    __nv_bfloat16* out0, __nv_bfloat16* out1, __nv_bfloat16* out2) {
  griddep_wait();
  griddep_trigger();
  const long idx = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int nv = N / 8;
  if (idx >= static_cast<long>(M) * nv) return;
  const int m = static_cast<int>(idx / nv), n = static_cast<int>(idx - static_cast<long>(m) * nv) * 8;
  const size_t mn = static_cast<size_t>(M) * N;
  const float4* src = reinterpret_cast<const float4*>(part + static_cast<size_t>(m) * N + n);
  float v[8];
  {
    const float4 a = __ldcg(src), b = __ldcg(src + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
  for (int r = 1; r < runs; ++r) {
    const float4* s4 = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(src) + r * mn);
    const float4 a = __ldcg(s4), b = __ldcg(s4 + 1);
    v[0] += a.x; v[1] += a.y; v[2] += a.z; v[3] += a.w;
    v[4] += b.x; v[5] += b.y; v[6] += b.z; v[7] += b.w;
  }
  if (bias) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(bias + n));
    const float4 b = __ldg(reinterpret_cast<const float4*>(bias + n) + 1);
    v[0] += a.x; v[1] += a.y; v[2] += a.z; v[3] += a.w;
    v[4] += b.x; v[5] += b.y; v[6] += b.z; v[7] += b.w;
  }
  if (residual) {
    uint4 u = *reinterpret_cast<const uint4*>(residual + static_cast<size_t>(m) * N + n);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(h[e]);
      v[2 * e] += f.x;
      v[2 * e + 1] += f.y;
    }
  }
  const int seg = n / split;
  __nv_bfloat16* o = seg == 0 ? out0 : seg == 1 ? out1 : out2;
  uint4 u;
  u.x = pack_bf16x2(v[0], v[1]);
  u.y = pack_bf16x2(v[2], v[3]);
  u.z = pack_bf16x2(v[4], v[5]);
  u.w = pack_bf16x2(v[6], v[7]);
  *reinterpret_cast<uint4*>(o + static_cast<size_t>(m) * ld_out + (n - seg * split)) = u;
}

static int launch_finish(const GemmParams& p, int M, cudaStream_t s) {
  const long n = static_cast<long>(M) * (p.N / 8);
  mark_launch(s);
  return launch_kernel(splitk_finish_kernel, dim3(static_cast<unsigned>((n + 255) / 256)), dim3(256), 0,
                       s, false, "split-K finish launch", static_cast<const float*>(p.part), p.splits,
                       M, p.N, p.split, p.ld_out, p.bias, static_cast<const __nv_bfloat16*>(p.residual),
                       static_cast<__nv_bfloat16*>(p.out0), static_cast<__nv_bfloat16*>(p.out1),
                       static_cast<__nv_bfloat16*>(p.out2));
}

// Conv tile shape: Wt columns x 128/Wt rows, Wt a power of two in [8, 128]
// wasting the fewest columns; a single 128-pixel row per tile (one TMA box
// per A stage) when the ragged right edge wastes at most an eighth of it.
static int conv_tile_width(int Wo) {
  int Wt = 128, waste_best = 1 << 30;
  for (int w = 128; w >= 8; w >>= 1) {
    const int waste = ((Wo + w - 1) / w) * w - Wo;
    if (waste < waste_best) {
      waste_best = waste;
      Wt = w;
    }
  }
  if (Wo >= 128 && (((Wo + 127) / 128) * 128 - Wo) * 8 <= Wo) Wt = 128;
  return Wt;
}

int conv3x3_splits(int H, int W, int Cin, int Cout, int stride, int dtype, bool can_split) {
  if (dtype == DP_FP32 || conv3x3_is_narrow(Cout)) return 1;
  const int Ho = (H - 1) / stride + 1, Wo = (W - 1) / stride + 1;
  const int Wt = conv_tile_width(Wo), R = 128 / Wt;
  const int m_tiles = ((Wo + Wt - 1) / Wt) * ((Ho + R - 1) / R);
  int bn_single = 0, splits = 1;
  const int pw = pick_pair(m_tiles, Cout, Cout, 9 * (Cin / 64), can_split, &bn_single, &splits);
  return pw ? splits : 1;
}

int linear_splits(int M, int N, int K, int split, bool can_split) {
  const int kb = K / 64;
  if (kb < 16) return 1;
  int bn_single = 0, splits = 1;
  const int pw = pick_pair((M + 127) / 128, N, split, kb, can_split, &bn_single, &splits);
  return pw ? splits : 1;
}

int conv3x3_launch(const void* a_fresh, const void* a_stale, const void* weight,
                   const float* bias, const void* residual, void* out, int H, int W, int Cin,
                   int Cout, int stride, int P, int mode, int dtype, void* workspace,
                   size_t workspace_bytes, cudaStream_t stream) {
  // a few output channels: the CUDA-core conv (dp_conv_narrow.cu)
  if (conv3x3_is_narrow(Cout))
    return conv3x3_narrow_launch(a_fresh, a_stale, weight, bias, residual, out, H, W, Cin, Cout, stride, P, mode,
                                 dtype, stream);
  // fp32 storage: fp32 arithmetic on the CUDA cores (dp_conv_f32.cu)
  if (dtype == DP_FP32)
    return conv3x3_f32_launch(a_fresh, a_stale, weight, bias, residual, out, H, W, Cin, Cout, stride, P,
                              mode, stream);
  const int e = 2;   // bf16
  const int BK = 128 / e;
  const int Ho = (H - 1) / stride + 1, Wo = (W - 1) / stride + 1;
  GemmParams p;
  memset(&p, 0, sizeof(p));
  p.splits = 1;
  p.a_mode = 1;
  p.H = H;
  p.W = W;
  p.Ho = Ho;
  p.Wo = Wo;
  p.Cin = Cin;
  p.stride = stride;
  p.hb_in = H / P;
  p.hb_out = Ho / P;
  p.mode = mode;
  const int Wt = conv_tile_width(Wo);
  p.Wt = Wt;
  p.R = 128 / Wt;
  p.tiles_w = (Wo + Wt - 1) / Wt;
  p.m_tiles = p.tiles_w * ((Ho + p.R - 1) / p.R);
  p.kc = Cin / BK;
  p.k_blocks = 9 * p.kc;
  p.N = Cout;
  p.split = Cout;
  p.ld_out = Cout;
  p.bias = bias;
  p.residual = residual;
  p.out0 = out;
  p.status = device_status_ptr();
  // an output of more than three quarters of L2 (126 MB) leaves L2 as it is written
  p.out_evict_first = static_cast<size_t>(Ho) * Wo * Cout * e > (static_cast<size_t>(96) << 20);
  int bn_single = 0, splits = 1;
  const bool can_split = workspace && workspace_bytes >= gemm_workspace_bytes();
  const int pw = pick_pair(p.m_tiles, Cout, Cout, p.k_blocks, can_split, &bn_single, &splits);
  const bool pair = pw != 0;
  const int BN = pair ? pw : pick_bn(p.m_tiles, Cout, Cout);
  if (!BN) return set_error(DP_ERR_UNSUPPORTED, "conv: no N tile divides Cout=%d", Cout);
  p.n_tiles = Cout / BN;
  const CUtensorMapDataType dt =
      CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  uint64_t dims[3], str[2];
  uint32_t box[3] = {static_cast<uint32_t>(BK), static_cast<uint32_t>(Wt), 1};
  if (stride == 1) {
    dims[0] = Cin; dims[1] = W; dims[2] = H;
    str[0] = static_cast<uint64_t>(Cin) * e;
    str[1] = static_cast<uint64_t>(W) * Cin * e;
  } else {
    dims[0] = 2 * static_cast<uint64_t>(Cin); dims[1] = W / 2; dims[2] = H;
    str[0] = 2 * static_cast<uint64_t>(Cin) * e;
    str[1] = static_cast<uint64_t>(W) * Cin * e;
  }
  int rc = encode_tmap(&p.tmA0, dt, 3, const_cast<void*>(a_fresh), dims, str, box,
                       CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc) return rc;
  rc = encode_tmap(&p.tmA1, dt, 3, const_cast<void*>(a_stale ? a_stale : a_fresh), dims, str, box,
                   CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc) return rc;
  uint64_t bdims[2] = {9 * static_cast<uint64_t>(Cin), static_cast<uint64_t>(Cout)};
  uint64_t bstr[1] = {9 * static_cast<uint64_t>(Cin) * e};
  uint32_t bbox[2] = {static_cast<uint32_t>(BK), static_cast<uint32_t>(pair ? 80 : BN)};
  rc = encode_tmap(&p.tmB, dt, 2, const_cast<void*>(weight), bdims, bstr, bbox,
                   CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc) return rc;
  if (pair) {
    rc = encode_conv_epilogue(p, out, Cout);
    if (rc) return rc;
    set_split(p, splits, workspace);
    rc = pw == 320 ? launch_pair<160, 2>(p, stream) : launch_pair<160, 1>(p, stream);
    if (rc || splits == 1) return rc;
    return launch_finish(p, Ho * Wo, stream);
  }
  return launch_gemm(p, BN, stream);
}

bool conv3x3_gn_eligible(int H, int W, int Cin, int Cout, int G, int dtype) {
  return dtype == DP_BF16 && W >= 128 && Cin % 64 == 0 && G > 0 && Cin % G == 0 && Cout % 160 == 0 &&
         H >= 1;
}

template <int NJ>
static int launch_gn_pair(const GemmParams& p, cudaStream_t s) {
  using C = GnConvCfg<NJ>;
  static int grid_cache[32] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  int& maxg = grid_cache[dev & 31];
  if (!maxg) {
    int rc = cuda_check(cudaFuncSetAttribute(igemm_gn_pair_kernel<NJ>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM),
                        "groupnorm conv smem attribute");
    if (rc) return rc;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 2;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.gridDim = dim3(2 * num_sms());
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, igemm_gn_pair_kernel<NJ>, &cfg) != cudaSuccess ||
        clusters <= 0) {
      cudaGetLastError();
      clusters = num_sms() / 2;
    }
    maxg = 2 * clusters;
  }
  const int pair_tiles = ((p.m_tiles + 1) / 2) * p.n_tiles;
  const int grid = std::min(2 * pair_tiles, maxg);
  mark_launch(s);
  return launch_kernel(igemm_gn_pair_kernel<NJ>, dim3(grid), dim3(C::THREADS), C::SMEM, s, false,
                       "groupnorm conv launch", p);
}

int conv3x3_gn_launch(const void* x, const void* a_stale, void* a_next, const float* used,
                      const float* gamma, const float* beta, int G, float eps, int silu,
                      const void* weight, const float* bias, const void* residual, void* out, int H,
                      int W, int Cin, int Cout, int P, int mode, cudaStream_t stream) {
  if (!conv3x3_gn_eligible(H, W, Cin, Cout, G, DP_BF16))
    return set_error(DP_ERR_UNSUPPORTED, "groupnorm conv: needs bf16, W >= 128, Cin %% 64 == 0, "
                                         "Cout %% 160 == 0 (H=%d W=%d Cin=%d Cout=%d)", H, W, Cin, Cout);
  GemmParams p;
  memset(&p, 0, sizeof(p));
  p.splits = 1;
  p.a_mode = 1;
  p.H = H;
  p.W = W;
  p.Ho = H;
  p.Wo = W;
  p.Cin = Cin;
  p.stride = 1;
  p.hb_in = H / P;
  p.hb_out = H / P;
  p.mode = mode;
  p.Wt = 128;
  p.R = 1;
  p.tiles_w = (W + 127) / 128;
  p.m_tiles = p.tiles_w * H;
  p.kc = Cin / 64;
  p.k_blocks = 9 * p.kc;
  p.N = Cout;
  p.split = Cout;
  p.ld_out = Cout;
  p.bias = bias;
  p.residual = residual;
  p.out0 = out;
  p.status = device_status_ptr();
  p.gn_used = used;
  p.gn_gamma = gamma;
  p.gn_beta = beta;
  p.gn_eps = eps;
  p.gn_cg = Cin / G;
  p.gn_silu = silu;
  p.a_next = a_next;
  const int NJ = Cout % 320 == 0 ? 2 : 1;
  p.n_tiles = Cout / (160 * NJ);
  uint64_t dims[3] = {static_cast<uint64_t>(Cin), static_cast<uint64_t>(W), static_cast<uint64_t>(H)};
  uint64_t str[2] = {static_cast<uint64_t>(Cin) * 2, static_cast<uint64_t>(W) * Cin * 2};
  uint32_t box[3] = {64, static_cast<uint32_t>(GnConvCfg<1>::ROW_PX), 1};
  int rc = encode_tmap(&p.tmA0, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(x), dims, str, box,
                       CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc) return rc;
  rc = encode_tmap(&p.tmA1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(a_stale ? a_stale : x),
                   dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc) return rc;
  uint64_t bdims[2] = {9 * static_cast<uint64_t>(Cin), static_cast<uint64_t>(Cout)};
  uint64_t bstr[1] = {9 * static_cast<uint64_t>(Cin) * 2};
  uint32_t bbox[2] = {64, 80};
  rc = encode_tmap(&p.tmB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(weight), bdims, bstr,
                   bbox, CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc) return rc;
  rc = encode_conv_epilogue(p, out, Cout);
  if (rc) return rc;
  return NJ == 2 ? launch_gn_pair<2>(p, stream) : launch_gn_pair<1>(p, stream);
}

int linear_launch(const void* x, const void* weight, const float* bias, const void* residual,
                  void* out0, void* out1, void* out2, int M, int N, int K, int split,
                  void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  GemmParams p;
  memset(&p, 0, sizeof(p));
  p.splits = 1;
  p.a_mode = 0;
  p.M = M;
  p.m_tiles = (M + 127) / 128;
  p.k_blocks = K / 64;
  p.N = N;
  p.split = split;
  p.ld_out = split;
  p.bias = bias;
  p.residual = residual;
  p.out0 = out0;
  p.out1 = out1;
  p.out2 = out2;
  p.status = device_status_ptr();
  int bn_single = 0, splits = 1;
  const bool can_split = workspace && workspace_bytes >= gemm_workspace_bytes();
  // Very short K (under 8 K blocks per tile) does not amortise a pair tile's
  // pipeline fill; such projections stay on single-CTA tiles (measured: the
  // 4096x640x320 projection is 4 % slower on 256x160 pair tiles, the
  // 4096x1920x640 one 9 % faster).
  const int pw = p.k_blocks >= 8
                     ? pick_pair(p.m_tiles, N, split, p.k_blocks, can_split, &bn_single, &splits)
                     : 0;
  if (!pw) bn_single = pick_bn(p.m_tiles, N, split);
  const bool pair = pw != 0;
  const int BN = pair ? pw : bn_single;
  if (!BN) return set_error(DP_ERR_UNSUPPORTED, "linear: no N tile divides split=%d", split);
  p.n_tiles = N / BN;
  uint64_t adims[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(M)};
  uint64_t astr[1] = {static_cast<uint64_t>(K) * 2};
  uint32_t abox[2] = {64, 128};
  int rc = encode_tmap(&p.tmA0, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), adims,
                       astr, abox, CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc) return rc;
  uint64_t bdims[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(N)};
  uint32_t bbox[2] = {64, static_cast<uint32_t>(pair ? 80 : BN)};
  rc = encode_tmap(&p.tmB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(weight), bdims,
                   astr, bbox, CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc) return rc;
  if (pair) {
    void* const outs[3] = {out0, out1, out2};
    rc = encode_linear_epilogue(p, outs);
    if (rc) return rc;
    set_split(p, splits, workspace);
    rc = pw == 320 ? launch_pair<160, 2>(p, stream) : launch_pair<160, 1>(p, stream);
    if (rc || splits == 1) return rc;
    return launch_finish(p, M, stream);
  }
  return launch_gemm(p, BN, stream);
}

bool linear_geglu_fusable(int M, int F, int K) {
  return M > 0 && F > 0 && K > 0 && K % 64 == 0 && F % 16 == 0 && (2 * F) % 160 == 0;
}

// y = a * gelu(g) of the projection [a|g] = x W^T + b, in one pair-kernel launch
// whose epilogue applies the gated GELU (W's rows interleaved in blocks of 16).
int linear_geglu_launch(const void* x, const void* weight, const float* bias, void* y, int M, int F, int K,
                        cudaStream_t stream) {
  if (!linear_geglu_fusable(M, F, K)) return set_error(DP_ERR_UNSUPPORTED, "linear geglu: shape not fusable");
  GemmParams p;
  memset(&p, 0, sizeof(p));
  const int N = 2 * F;
  p.splits = 1;
  p.a_mode = 0;
  p.M = M;
  p.m_tiles = (M + 127) / 128;
  p.k_blocks = K / 64;
  p.N = N;
  p.split = N;
  p.ld_out = F;
  p.bias = bias;
  p.out0 = y;
  p.geglu = 1;
  p.status = device_status_ptr();
  int bn_single = 0, splits = 1;
  int pw = pick_pair(p.m_tiles, N, N, p.k_blocks, false, &bn_single, &splits);
  if (!pw) pw = N % 320 == 0 ? 320 : 160;   // the single-CTA kernel has no gated epilogue
  p.n_tiles = N / pw;
  uint64_t adims[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(M)};
  uint64_t astr[1] = {static_cast<uint64_t>(K) * 2};
  uint32_t abox[2] = {64, 128};
  int rc = encode_tmap(&p.tmA0, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), adims, astr, abox,
                       CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc) return rc;
  uint64_t bdims[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(N)};
  uint32_t bbox[2] = {64, 80};
  rc = encode_tmap(&p.tmB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(weight), bdims, astr, bbox,
                   CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc) return rc;
  uint64_t odims[2] = {static_cast<uint64_t>(F), static_cast<uint64_t>(M)};
  uint64_t ostr[1] = {static_cast<uint64_t>(F) * 2};
  uint32_t obox[2] = {16, 32};
  rc = encode_tmap(&p.tmO[0], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, y, odims, ostr, obox,
                   CU_TENSOR_MAP_SWIZZLE_NONE);
  if (rc) return rc;
  return pw == 320 ? launch_pair<160, 2>(p, stream) : launch_pair<160, 1>(p, stream);
}

int conv3x3_validate(const void* a_fresh, const void* a_stale, const void* weight,
                     const void* residual, const void* out, int H, int W, int Cin, int Cout,
                     int stride, int P, int mode, int dtype) {
  if (!a_fresh || !weight || !out) return set_error(DP_ERR_INVALID_ARG, "conv: null pointer");
  if (H <= 0 || W <= 0 || Cin <= 0 || Cout <= 0 || P <= 0)
    return set_error(DP_ERR_INVALID_ARG, "conv: non-positive size");
  if (mode < DP_MODE_SYNC || mode > DP_MODE_NAIVE)
    return set_error(DP_ERR_INVALID_ARG, "conv: bad mode %d", mode);
  if (dtype != DP_BF16 && dtype != DP_FP32) return set_error(DP_ERR_INVALID_ARG, "conv: bad dtype");
  if (stride != 1 && stride != 2) return set_error(DP_ERR_UNSUPPORTED, "conv: stride must be 1 or 2");
  if (mode == DP_MODE_DISPLACED && !a_stale)
    return set_error(DP_ERR_INVALID_ARG, "conv: displaced mode needs the stale buffer");
  const int BK = dtype == DP_FP32 ? 16 : 64;
  if (Cin % BK) return set_error(DP_ERR_UNSUPPORTED, "conv: Cin must be a multiple of %d", BK);
  if (Cout % 32 && !conv3x3_is_narrow(Cout))
    return set_error(DP_ERR_UNSUPPORTED, "conv: Cout must be a multiple of 32 or at most 16");
  const int Ho = (H - 1) / stride + 1;
  if (H % P || Ho % P) return set_error(DP_ERR_UNSUPPORTED, "conv: rows not divisible by P");
  if (stride == 2 && (W % 2)) return set_error(DP_ERR_UNSUPPORTED, "conv: stride 2 needs even W");
  if (!aligned16(a_fresh) || (a_stale && !aligned16(a_stale)) || !aligned16(weight) ||
      !aligned16(out) || (residual && !aligned16(residual)))
    return set_error(DP_ERR_UNSUPPORTED, "conv: pointers must be 16-byte aligned");
  if (a_stale && (a_stale == out)) return set_error(DP_ERR_INVALID_ARG, "conv: out aliases a_stale");
  if (a_fresh == out) return set_error(DP_ERR_INVALID_ARG, "conv: out aliases a_fresh");
  return DP_OK;
}

}  // namespace dp

extern "C" {

size_t dp_gemm_workspace_size(void) { return dp::gemm_workspace_bytes(); }

int dp_conv3x3_halo_gn(const void* x, const void* a_stale, void* a_next, const float* used_stats,
                       const float* gamma, const float* beta, int G, float eps, int silu,
                       const void* weight, const float* bias, const void* residual, void* out, int H,
                       int W, int Cin, int Cout, int P, int mode, void* stream) {
  int rc = dp::conv3x3_validate(x, a_stale, weight, residual, out, H, W, Cin, Cout, 1, P, mode, DP_BF16);
  if (rc) return rc;
  if (!used_stats || !gamma || !beta)
    return dp::set_error(DP_ERR_INVALID_ARG, "groupnorm conv: null used_stats/gamma/beta");
  if (!dp::aligned16(gamma) || !dp::aligned16(beta))
    return dp::set_error(DP_ERR_UNSUPPORTED, "groupnorm conv: gamma/beta not 16-byte aligned");
  if (G <= 0 || Cin % G) return dp::set_error(DP_ERR_UNSUPPORTED, "groupnorm conv: Cin %% G != 0");
  if (!(eps > 0.f)) return dp::set_error(DP_ERR_INVALID_ARG, "groupnorm conv: eps must be > 0");
  if (!dp::conv3x3_gn_eligible(H, W, Cin, Cout, G, DP_BF16))
    return dp::set_error(DP_ERR_UNSUPPORTED, "groupnorm conv: needs W >= 128, Cin %% 64 == 0 and "
                                             "Cout %% 160 == 0");
  if (a_next) {
    if (!dp::aligned16(a_next)) return dp::set_error(DP_ERR_UNSUPPORTED, "groupnorm conv: a_next not aligned");
    const size_t bytes = static_cast<size_t>(H) * W * Cin * 2;
    const char* n = static_cast<const char*>(a_next);
    auto hit = [&](const void* q, size_t qb) {
      const char* c = static_cast<const char*>(q);
      return q && n < c + qb && c < n + bytes;
    };
    const size_t ob = static_cast<size_t>(H) * W * Cout * 2;
    if (hit(x, bytes) || hit(a_stale, bytes) || hit(out, ob) || hit(residual, ob))
      return dp::set_error(DP_ERR_INVALID_ARG, "groupnorm conv: a_next overlaps an input or the output");
  }
  return dp::conv3x3_gn_launch(x, a_stale, a_next, used_stats, gamma, beta, G, eps, silu, weight, bias,
                               residual, out, H, W, Cin, Cout, P, mode, static_cast<cudaStream_t>(stream));
}

int dp_conv3x3_halo(const void* a_fresh, const void* a_stale, const void* weight,
                    const float* bias, const void* residual, void* out, int H, int W, int Cin,
                    int Cout, int stride, int P, int mode, int dtype, void* workspace,
                    size_t workspace_bytes, void* stream) {
  int rc = dp::conv3x3_validate(a_fresh, a_stale, weight, residual, out, H, W, Cin, Cout, stride,
                                P, mode, dtype);
  if (rc) return rc;
  if (bias && !dp::aligned16(bias)) return dp::set_error(DP_ERR_UNSUPPORTED, "conv: bias not 16-byte aligned");
  if (workspace && !dp::aligned16(workspace))
    return dp::set_error(DP_ERR_UNSUPPORTED, "conv: workspace not 16-byte aligned");
  return dp::conv3x3_launch(a_fresh, a_stale, weight, bias, residual, out, H, W, Cin, Cout, stride,
                            P, mode, dtype, workspace, workspace_bytes,
                            static_cast<cudaStream_t>(stream));
}

int dp_linear_geglu(const void* x, const void* weight, const float* bias, void* y, int M, int F, int K,
                    void* stream) {
  if (!x || !weight || !y) return dp::set_error(DP_ERR_INVALID_ARG, "linear geglu: null pointer");
  if (M <= 0 || F <= 0 || K <= 0) return dp::set_error(DP_ERR_INVALID_ARG, "linear geglu: bad size");
  if (!dp::linear_geglu_fusable(M, F, K))
    return dp::set_error(DP_ERR_UNSUPPORTED, "linear geglu: needs K %% 64 == 0, F %% 16 == 0 and 2F %% 160 == 0");
  if (!dp::aligned16(x) || !dp::aligned16(weight) || !dp::aligned16(y) || (bias && !dp::aligned16(bias)))
    return dp::set_error(DP_ERR_UNSUPPORTED, "linear geglu: pointers must be 16-byte aligned");
  const char* xb = static_cast<const char*>(x);
  const char* yb = static_cast<const char*>(y);
  const size_t xbytes = static_cast<size_t>(M) * K * 2, ybytes = static_cast<size_t>(M) * F * 2;
  if (xb < yb + ybytes && yb < xb + xbytes) return dp::set_error(DP_ERR_INVALID_ARG, "linear geglu: y overlaps x");
  return dp::linear_geglu_launch(x, weight, bias, y, M, F, K, static_cast<cudaStream_t>(stream));
}

int dp_linear(const void* x, const void* weight, const float* bias, const void* residual,
              void* out0, void* out1, void* out2, int M, int N, int K, int split, void* workspace,
              size_t workspace_bytes, void* stream) {
  if (!x || !weight || !out0) return dp::set_error(DP_ERR_INVALID_ARG, "linear: null pointer");
  if (M <= 0 || N <= 0 || K <= 0 || split <= 0)
    return dp::set_error(DP_ERR_INVALID_ARG, "linear: non-positive size");
  if (K % 64) return dp::set_error(DP_ERR_UNSUPPORTED, "linear: K must be a multiple of 64");
  if (split % 32 || N % split || N / split > 3)
    return dp::set_error(DP_ERR_UNSUPPORTED, "linear: need split %% 32 == 0, N = k*split, k <= 3");
  const int nseg = N / split;
  if ((nseg > 1 && !out1) || (nseg > 2 && !out2))
    return dp::set_error(DP_ERR_INVALID_ARG, "linear: missing output buffer");
  if (residual && nseg != 1)
    return dp::set_error(DP_ERR_UNSUPPORTED, "linear: residual needs a single output");
  if (!dp::aligned16(x) || !dp::aligned16(weight) || !dp::aligned16(out0) ||
      (out1 && !dp::aligned16(out1)) || (out2 && !dp::aligned16(out2)) ||
      (residual && !dp::aligned16(residual)) || (bias && !dp::aligned16(bias)))
    return dp::set_error(DP_ERR_UNSUPPORTED, "linear: pointers must be 16-byte aligned");
  if (workspace && !dp::aligned16(workspace))
    return dp::set_error(DP_ERR_UNSUPPORTED, "linear: workspace not 16-byte aligned");
  return dp::linear_launch(x, weight, bias, residual, out0, out1, out2, M, N, K, split, workspace,
                           workspace_bytes, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
