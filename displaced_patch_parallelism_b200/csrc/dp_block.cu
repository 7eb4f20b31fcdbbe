// dp_block.cu -- one U-Net block step over all P bands, with its cross-step state.
//
// The state of a displaced block is what the previous step left behind: the
// input of every 3x3 conv, the keys and values of every attention and the
// per-band statistics of every GroupNorm ("DistriFusion", study.space
// summary, Method; gist.science PipeFusion explainer, Memory Efficiency, on
// DistriFusion's full-spatial K/V buffers).  Each of these lives in a
// ping-pong pair inside the caller's workspace: a step writes the fresh half
// (GroupNorm output, fused q/k/v projection output, fresh statistics) and
// reads the stale half; the refresh that replaces the paper's AllGather is a
// flip of `cur`, so no byte moves.
#include <cstring>

#include "dp_common.cuh"
#include "dp_internal.h"

namespace dp {

namespace {

struct Bump {
  size_t off = 0;
  size_t take(size_t bytes) {
    const size_t o = off;
    off += (bytes + 255) & ~static_cast<size_t>(255);
    return o;
  }
};

struct GnSlots {
  size_t local[2], global[2], used, ws;
};

struct Layout {
  GnSlots gn1, gn2;
  size_t a1[2], a2[2], h, sc;        // conv inputs (pairs), conv1 output, shortcut output
  size_t act, q, k[2], v[2], o;      // attention buffers
  size_t total;
};

GnSlots gn_slots(Bump& b, int P, int G) {
  GnSlots s;
  for (int i = 0; i < 2; ++i) {
    s.local[i] = b.take(static_cast<size_t>(P) * G * 2 * sizeof(float));
    s.global[i] = b.take(static_cast<size_t>(G) * 2 * sizeof(float));
  }
  s.used = b.take(static_cast<size_t>(P) * G * 2 * sizeof(float));
  s.ws = b.take(gn_workspace_bytes(P, G));
  return s;
}

Layout layout_of(const dp_block_desc* d) {
  Layout L;
  memset(&L, 0, sizeof(L));
  Bump b;
  const size_t e = d->dtype == DP_FP32 ? 4 : 2;
  const size_t hw = static_cast<size_t>(d->H) * d->W;
  L.gn1 = gn_slots(b, d->P, d->G);
  if (d->kind == DP_BLOCK_GN_CONV) {
    for (int i = 0; i < 2; ++i) L.a1[i] = b.take(hw * d->C * e);
  } else if (d->kind == DP_BLOCK_RESBLOCK) {
    L.gn2 = gn_slots(b, d->P, d->G);
    for (int i = 0; i < 2; ++i) L.a1[i] = b.take(hw * d->C * e);
    for (int i = 0; i < 2; ++i) L.a2[i] = b.take(hw * d->Cout * e);
    L.h = b.take(hw * d->Cout * e);
    if (d->C != d->Cout) L.sc = b.take(hw * d->Cout * e);
  } else {
    L.act = b.take(hw * d->C * e);
    L.q = b.take(hw * d->C * e);
    for (int i = 0; i < 2; ++i) L.k[i] = b.take(hw * d->C * e);
    for (int i = 0; i < 2; ++i) L.v[i] = b.take(hw * d->C * e);
    L.o = b.take(hw * d->C * e);
  }
  L.total = b.off;
  return L;
}

int desc_check(const dp_block_desc* d) {
  if (!d) return set_error(DP_ERR_INVALID_ARG, "block: null descriptor");
  if (d->kind < DP_BLOCK_GN_CONV || d->kind > DP_BLOCK_ATTN)
    return set_error(DP_ERR_INVALID_ARG, "block: bad kind %d", d->kind);
  if (d->H <= 0 || d->W <= 0 || d->C <= 0 || d->Cout <= 0 || d->G <= 0 || d->P <= 0)
    return set_error(DP_ERR_INVALID_ARG, "block: non-positive size");
  if (d->dtype != DP_BF16 && d->dtype != DP_FP32)
    return set_error(DP_ERR_INVALID_ARG, "block: bad dtype");
  if (d->dtype == DP_FP32 && d->kind != DP_BLOCK_GN_CONV)
    return set_error(DP_ERR_UNSUPPORTED, "block: fp32 storage is only built for GN_CONV");
  if (d->H % d->P) return set_error(DP_ERR_UNSUPPORTED, "block: H %% P != 0");
  if (d->C % d->G || d->Cout % d->G) return set_error(DP_ERR_UNSUPPORTED, "block: channels %% G != 0");
  if (d->kind == DP_BLOCK_ATTN) {
    if (d->Cout != d->C) return set_error(DP_ERR_INVALID_ARG, "block: attention keeps C");
    if (d->heads <= 0 || d->C != d->heads * 64)
      return set_error(DP_ERR_UNSUPPORTED, "block: attention needs C == heads * 64");
    const int T = d->H * d->W;
    if ((T / d->P) % 128) return set_error(DP_ERR_UNSUPPORTED, "block: tokens per band %% 128 != 0");
  }
  if (!(d->eps > 0.f)) return set_error(DP_ERR_INVALID_ARG, "block: eps must be > 0");
  return DP_OK;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

}  // namespace
}  // namespace dp

extern "C" {

int dp_block_desc_init(dp_block_desc* d, int kind, int H, int W, int C, int Cout, int G, int P,
                       int heads, int dtype, int silu, float eps, float w) {
  if (!d) return dp::set_error(DP_ERR_INVALID_ARG, "block: null descriptor");
  d->kind = kind;
  d->H = H;
  d->W = W;
  d->C = C;
  d->Cout = Cout > 0 ? Cout : C;
  d->G = G;
  d->P = P;
  d->heads = heads;
  d->dtype = dtype;
  d->silu = silu;
  d->eps = eps;
  d->w = w;
  return dp::desc_check(d);
}

size_t dp_block_workspace_size(const dp_block_desc* d) {
  if (dp::desc_check(d)) return 0;
  return dp::layout_of(d).total;
}

int dp_block_state_init(const dp_block_desc* d, dp_block_state* s, void* workspace,
                        size_t workspace_bytes, void* stream) {
  int rc = dp::desc_check(d);
  if (rc) return rc;
  if (!s || !workspace) return dp::set_error(DP_ERR_INVALID_ARG, "block: null state/workspace");
  const dp::Layout L = dp::layout_of(d);
  if (workspace_bytes < L.total)
    return dp::set_error(DP_ERR_INVALID_ARG, "block: workspace too small (%zu < %zu)",
                         workspace_bytes, L.total);
  if (!dp::aligned16(workspace)) return dp::set_error(DP_ERR_UNSUPPORTED, "block: workspace not 16-byte aligned");
  rc = dp::cuda_check(cudaMemsetAsync(workspace, 0, L.total, static_cast<cudaStream_t>(stream)),
                      "block: zero workspace");
  if (rc) return rc;
  s->workspace = workspace;
  s->workspace_bytes = workspace_bytes;
  s->cur = 0;
  s->steps_done = 0;
  return DP_OK;
}

double dp_block_flops(const dp_block_desc* d) {
  if (dp::desc_check(d)) return 0.0;
  const double hw = static_cast<double>(d->H) * d->W;
  const double C = d->C, Co = d->Cout;
  if (d->kind == DP_BLOCK_GN_CONV) return 2.0 * hw * Co * 9.0 * C;
  if (d->kind == DP_BLOCK_RESBLOCK)
    return 2.0 * hw * Co * 9.0 * C + 2.0 * hw * Co * 9.0 * Co + (C != Co ? 2.0 * hw * Co * C : 0.0);
  // attention block: q/k/v and output projections + QK^T and PV over all keys
  return 2.0 * hw * 3.0 * C * C + 4.0 * hw * hw * C + 2.0 * hw * C * C;
}

int dp_block_step(const dp_block_desc* d, dp_block_state* s, const void* x, void* out,
                  const void* const* weights, int n_weights, int mode, void* stream) {
  int rc = dp::desc_check(d);
  if (rc) return rc;
  if (!s || !s->workspace || !x || !out || !weights)
    return dp::set_error(DP_ERR_INVALID_ARG, "block: null argument");
  if (mode < DP_MODE_SYNC || mode > DP_MODE_NAIVE)
    return dp::set_error(DP_ERR_INVALID_ARG, "block: bad mode %d", mode);
  if (mode == DP_MODE_DISPLACED && s->steps_done == 0)
    return dp::set_error(DP_ERR_STATE, "block: a displaced step needs a completed previous step");
  if (x == out) return dp::set_error(DP_ERR_INVALID_ARG, "block: out aliases x");
  if (!dp::aligned16(x) || !dp::aligned16(out))
    return dp::set_error(DP_ERR_UNSUPPORTED, "block: x/out not 16-byte aligned");
  const dp::Layout L = dp::layout_of(d);
  if (s->workspace_bytes < L.total) return dp::set_error(DP_ERR_INVALID_ARG, "block: workspace too small");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  void* ws = s->workspace;
  const int f = s->cur ^ 1, o = s->cur;   // fresh / stale halves
  const int H = d->H, W = d->W, C = d->C, Co = d->Cout, G = d->G, P = d->P;
  auto gn = [&](const dp::GnSlots& g, const void* in, void* y, const void* gamma, const void* beta,
                int ch, int silu) {
    return dp::gn_launch(in, y, static_cast<const float*>(gamma), static_cast<const float*>(beta), H,
                         W, ch, G, P, d->eps, d->w, silu, mode, d->dtype,
                         dp::at<float>(ws, g.global[o]), dp::at<float>(ws, g.local[o]),
                         dp::at<float>(ws, g.local[f]), dp::at<float>(ws, g.global[f]),
                         dp::at<float>(ws, g.used), dp::at<void>(ws, g.ws), st);
  };
  const void* const* w = weights;
  if (d->kind == DP_BLOCK_GN_CONV) {
    if (n_weights < 4) return dp::set_error(DP_ERR_INVALID_ARG, "block: GN_CONV needs 4 weights");
    if (!w[0] || !w[1] || !w[2]) return dp::set_error(DP_ERR_INVALID_ARG, "block: null weight");
    rc = dp::conv3x3_validate(x, x, w[2], nullptr, out, H, W, C, Co, 1, P, mode, d->dtype);
    if (rc) return rc;
    rc = gn(L.gn1, x, dp::at<void>(ws, L.a1[f]), w[0], w[1], C, d->silu);
    if (rc) return rc;
    rc = dp::conv3x3_launch(dp::at<void>(ws, L.a1[f]), dp::at<void>(ws, L.a1[o]), w[2],
                            static_cast<const float*>(w[3]), nullptr, out, H, W, C, Co, 1, P, mode,
                            d->dtype, st);
    if (rc) return rc;
  } else if (d->kind == DP_BLOCK_RESBLOCK) {
    const int need = C != Co ? 10 : 8;
    if (n_weights < need) return dp::set_error(DP_ERR_INVALID_ARG, "block: RESBLOCK needs %d weights", need);
    if (!w[0] || !w[1] || !w[2] || !w[4] || !w[5] || !w[6] || (C != Co && !w[8]))
      return dp::set_error(DP_ERR_INVALID_ARG, "block: null weight");
    rc = dp::conv3x3_validate(x, x, w[2], nullptr, out, H, W, C, Co, 1, P, mode, d->dtype);
    if (rc) return rc;
    rc = dp::conv3x3_validate(x, x, w[6], nullptr, out, H, W, Co, Co, 1, P, mode, d->dtype);
    if (rc) return rc;
    void* a1f = dp::at<void>(ws, L.a1[f]);
    void* a2f = dp::at<void>(ws, L.a2[f]);
    void* h = dp::at<void>(ws, L.h);
    rc = gn(L.gn1, x, a1f, w[0], w[1], C, 1);
    if (rc) return rc;
    rc = dp::conv3x3_launch(a1f, dp::at<void>(ws, L.a1[o]), w[2], static_cast<const float*>(w[3]),
                            nullptr, h, H, W, C, Co, 1, P, mode, d->dtype, st);
    if (rc) return rc;
    rc = gn(L.gn2, h, a2f, w[4], w[5], Co, 1);
    if (rc) return rc;
    const void* res = x;
    if (C != Co) {
      void* sc = dp::at<void>(ws, L.sc);
      rc = dp::linear_launch(x, w[8], static_cast<const float*>(w[9]), nullptr, sc, nullptr, nullptr,
                             H * W, Co, C, Co, st);
      if (rc) return rc;
      res = sc;
    }
    rc = dp::conv3x3_launch(a2f, dp::at<void>(ws, L.a2[o]), w[6], static_cast<const float*>(w[7]),
                            res, out, H, W, Co, Co, 1, P, mode, d->dtype, st);
    if (rc) return rc;
  } else {
    if (n_weights < 6) return dp::set_error(DP_ERR_INVALID_ARG, "block: ATTN needs 6 weights");
    if (!w[0] || !w[1] || !w[2] || !w[4]) return dp::set_error(DP_ERR_INVALID_ARG, "block: null weight");
    const int T = H * W;
    void* act = dp::at<void>(ws, L.act);
    void* q = dp::at<void>(ws, L.q);
    void* kf = dp::at<void>(ws, L.k[f]);
    void* vf = dp::at<void>(ws, L.v[f]);
    void* ob = dp::at<void>(ws, L.o);
    rc = gn(L.gn1, x, act, w[0], w[1], C, 0);
    if (rc) return rc;
    rc = dp::linear_launch(act, w[2], static_cast<const float*>(w[3]), nullptr, q, kf, vf, T, 3 * C,
                           C, C, st);
    if (rc) return rc;
    rc = dp::attn_launch(q, kf, vf, dp::at<void>(ws, L.k[o]), dp::at<void>(ws, L.v[o]), ob, T,
                         d->heads, P, 0.125f, mode, st);
    if (rc) return rc;
    rc = dp::linear_launch(ob, w[4], static_cast<const float*>(w[5]), x, out, nullptr, nullptr, T, C,
                           C, C, st);
    if (rc) return rc;
  }
  s->cur ^= 1;
  s->steps_done += 1;
  return DP_OK;
}

int dp_block_launch_count(const dp_block_desc* d) {
  int rc = dp::desc_check(d);
  if (rc) return rc;
  if (d->kind == DP_BLOCK_GN_CONV) return 3;
  if (d->kind == DP_BLOCK_RESBLOCK) return d->C != d->Cout ? 7 : 6;
  return 5;
}

int dp_block_step_timed(const dp_block_desc* d, dp_block_state* s, const void* x, void* out,
                        const void* const* weights, int n_weights, int mode, void* stream,
                        void* const* events, int n_events) {
  const int n = dp_block_launch_count(d);
  if (n < 0) return n;
  if (!events || n_events < n + 1)
    return dp::set_error(DP_ERR_INVALID_ARG, "block: need %d events, got %d", n + 1, n_events);
  dp::recorder_begin(events, n_events);
  int rc = dp_block_step(d, s, x, out, weights, n_weights, mode, stream);
  const int used = dp::recorder_end();
  if (rc) return rc;
  if (used != n) return dp::set_error(DP_ERR_CUDA, "block: %d launches recorded, expected %d", used, n);
  return dp::cuda_check(cudaEventRecord(static_cast<cudaEvent_t>(events[n]),
                                        static_cast<cudaStream_t>(stream)),
                        "block: final event");
}

}  // extern "C"
