// dp_block.cu -- one U-Net block step over all P bands, with its cross-step state.
//
// The state of a displaced block is what the previous step left behind: the
// input of every 3x3 conv, the keys and values of every attention and the
// per-band statistics of every GroupNorm ("DistriFusion", study.space
// summary, Method; gist.science PipeFusion explainer, Memory Efficiency, on
// DistriFusion's full-spatial K/V buffers).  Each of these lives in a
// ping-pong pair inside the caller's workspace: a step writes the fresh half
// (GroupNorm output, fused q/k/v projection output, fresh statistics, or the
// output of the layer feeding a conv) and reads the stale half; the refresh
// that replaces DistriFusion's AllGather is a flip of `cur`, so no byte moves.
//
// Kinds: GN_CONV, RESBLOCK (optionally with an SDXL time embedding added to
// conv1's output), ATTN, TRANSFORMER (SDXL-shaped: GroupNorm and
// self-attention with stale context, then per-token LayerNorms, a
// cross-attention over the text context and a gated feed-forward, none of
// which need context from other bands), and UNET_MINI, a chain of the others with
// two stride-2 downsampling convs (conv_in -> ResBlock(320) -> down ->
// ResBlock(320->640) -> Attn(640) -> down -> ResBlock(640->1280) ->
// Attn(1280)), and UNET_SDXL, a whole SDXL-shaped U-Net step (conv_in, three
// down levels of ResBlocks and transformers, a middle, three up levels whose
// ResBlocks take the running tensor concatenated with a skip connection, and
// GroupNorm -> SiLU -> conv_out).  Composite kinds run their sub-blocks with
// the parent's ping-pong parity.
#include <cstring>
#include <new>
#include <vector>

#include "dp_common.cuh"
#include "dp_internal.h"

namespace dp {

int conv3x3_small_launch(const void* af, const void* as, const void* w, const float* bias,
                         void* out, int H, int W, int Cin, int Cout, int P, int mode,
                         cudaStream_t stream);

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

// Mini U-Net level widths.
constexpr int kU1 = 320, kU2 = 640, kU3 = 1280;

struct Layout {
  size_t status;                      // the block state's device status word
  GnSlots gn1, gn2;
  size_t a1[2], a2[2], h, sc;        // conv inputs (pairs), conv1 output, shortcut output
  size_t act, q, k[2], v[2], o;      // attention buffers
  size_t ha, hb, tn, q2, k2, v2, o2, ffh, ffg;   // TRANSFORMER: residual stream, LN output, cross, FF
  size_t kv_layer;                    // TRANSFORMER: bytes between layers' k/v ping-pong pairs
  size_t kv2_layer;                   // TRANSFORMER: bytes between layers' context k/v
  size_t attn_ws;                     // balanced attention split: counters + partials
  size_t tbias;                       // RESBLOCK with a time embedding: conv1's step bias
  size_t gemm_ws;                     // split-K partials of the convs and projections
  // UNET_MINI: sub-block workspaces and the buffers between them
  size_t xin[2], h0, rb1, d1[2], h1, rb2, h2, at2, d2[2], h3, rb3, h4, at3;
  size_t total;
};

dp_block_desc sub_desc(const dp_block_desc* d, int kind, int H, int W, int C, int Cout,
                       int heads, int silu) {
  dp_block_desc s = *d;
  s.kind = kind;
  s.H = H;
  s.W = W;
  s.C = C;
  s.Cout = Cout;
  s.heads = heads;
  s.silu = silu;
  // kind-specific settings start from their defaults
  s.ctx_len = s.ctx_dim = s.ff_inner = s.temb_dim = s.ctx_fixed = 0;
  s.depth = 1;
  s.unet_base = 0;
  s.unet_depth[0] = s.unet_depth[1] = s.unet_depth[2] = 0;
  return s;
}

// UNET_SDXL: the stages of one step in execution order.
enum { US_CONV_IN, US_RES, US_TF, US_DOWN, US_UP, US_OUT };
struct UStage {
  int kind;
  int H, W;            // the stage's input rows and columns (UP: before upsampling)
  int ci, co;          // input / output channels (RES in the up path: ci includes the skip)
  bool cat;            // RES: input = [h, latest unused skip]
  bool skip;           // the stage's output is a skip connection of the up path
  dp_block_desc sub;   // RES, TF, OUT: the sub-block
};

std::vector<UStage> unet_stages(const dp_block_desc* d) {
  std::vector<UStage> s;
  const int base = d->unet_base;
  const int ch[3] = {base, 2 * base, 4 * base};
  int H = d->H, W = d->W, c = base;
  std::vector<int> skips;
  auto add = [&](int kind, int ci, int co, bool cat) -> UStage& {
    UStage u;
    memset(&u, 0, sizeof(u));
    u.kind = kind;
    u.H = H;
    u.W = W;
    u.ci = ci;
    u.co = co;
    u.cat = cat;
    if (kind == US_RES) {
      u.sub = sub_desc(d, DP_BLOCK_RESBLOCK, H, W, ci, co, 0, 1);
      u.sub.temb_dim = d->temb_dim;
    } else if (kind == US_TF) {
      u.sub = sub_desc(d, DP_BLOCK_TRANSFORMER, H, W, ci, ci, ci / 64, 0);
      u.sub.ctx_len = d->ctx_len;
      u.sub.ctx_dim = d->ctx_dim;
      u.sub.ctx_fixed = d->ctx_fixed;
      u.sub.ff_inner = 4 * ci;
    } else if (kind == US_OUT) {
      u.sub = sub_desc(d, DP_BLOCK_GN_CONV, H, W, ci, co, 0, 1);
    }
    s.push_back(u);
    return s.back();
  };
  add(US_CONV_IN, d->C, base, false).skip = true;
  skips.push_back(base);
  for (int lvl = 0; lvl < 3; ++lvl) {
    for (int i = 0; i < 2; ++i) {
      add(US_RES, c, ch[lvl], false);
      c = ch[lvl];
      if (d->unet_depth[lvl] > 0) add(US_TF, c, c, false).sub.depth = d->unet_depth[lvl];
      s.back().skip = true;
      skips.push_back(c);
    }
    if (lvl < 2) {
      add(US_DOWN, c, c, false).skip = true;
      skips.push_back(c);
      H /= 2;
      W /= 2;
    }
  }
  add(US_RES, c, c, false);
  if (d->unet_depth[2] > 0) add(US_TF, c, c, false).sub.depth = d->unet_depth[2];
  add(US_RES, c, c, false);
  for (int lvl = 2; lvl >= 0; --lvl) {
    for (int i = 0; i < 3; ++i) {
      add(US_RES, c + skips.back(), ch[lvl], true);
      skips.pop_back();
      c = ch[lvl];
      if (d->unet_depth[lvl] > 0) add(US_TF, c, c, false).sub.depth = d->unet_depth[lvl];
    }
    if (lvl > 0) {
      add(US_UP, c, c, false);
      H *= 2;
      W *= 2;
    }
  }
  add(US_OUT, c, d->C, false);
  return s;
}

// Weight pointers of a stage in the composite's list (a ResBlock's temb vector
// and a transformer's context are the composite's last two pointers).
int stage_weight_count(const UStage& u);

struct MiniDescs {
  dp_block_desc rb1, rb2, at2, rb3, at3;
};

MiniDescs mini_descs(const dp_block_desc* d) {
  MiniDescs m;
  const int H = d->H, W = d->W;
  m.rb1 = sub_desc(d, DP_BLOCK_RESBLOCK, H, W, kU1, kU1, 0, 1);
  m.rb2 = sub_desc(d, DP_BLOCK_RESBLOCK, H / 2, W / 2, kU1, kU2, 0, 1);
  m.at2 = sub_desc(d, DP_BLOCK_ATTN, H / 2, W / 2, kU2, kU2, kU2 / 64, 0);
  m.rb3 = sub_desc(d, DP_BLOCK_RESBLOCK, H / 4, W / 4, kU2, kU3, 0, 1);
  m.at3 = sub_desc(d, DP_BLOCK_ATTN, H / 4, W / 4, kU3, kU3, kU3 / 64, 0);
  return m;
}

// UNET_SDXL workspace: per stage its sub-block's workspace (RES, TF, OUT),
// the ping-pong pair of its conv's input (CONV_IN: a copy of x; DOWN: written
// by the stage before; UP: the upsampled tensor) and its output buffer; one
// buffer for the concatenated input of the up path's ResBlocks.
struct ULayout {
  std::vector<UStage> st;
  std::vector<size_t> ws, pair0, pair1, out;
  size_t cat = 0;
};

size_t layout_total(const dp_block_desc* d);

ULayout unet_layout(const dp_block_desc* d, Bump& b) {
  ULayout U;
  U.st = unet_stages(d);
  const size_t n = U.st.size();
  U.ws.assign(n, 0);
  U.pair0.assign(n, 0);
  U.pair1.assign(n, 0);
  U.out.assign(n, 0);
  size_t cat = 0;
  for (size_t i = 0; i < n; ++i) {
    const UStage& u = U.st[i];
    const size_t hw = static_cast<size_t>(u.H) * u.W;
    if (u.kind == US_RES || u.kind == US_TF || u.kind == US_OUT) U.ws[i] = b.take(layout_total(&u.sub));
    if (u.kind == US_CONV_IN || u.kind == US_DOWN || u.kind == US_UP) {
      const size_t pb = hw * u.ci * 2 * (u.kind == US_UP ? 4 : 1);
      U.pair0[i] = b.take(pb);
      U.pair1[i] = b.take(pb);
    }
    if (u.kind == US_RES && u.cat) cat = cat > hw * u.ci * 2 ? cat : hw * u.ci * 2;
    const size_t ob = u.kind == US_DOWN ? hw / 4 * u.co * 2 : u.kind == US_UP ? 4 * hw * u.co * 2 : hw * u.co * 2;
    // the stage before a down conv writes into that conv's input pair instead
    const bool to_down = i + 1 < n && U.st[i + 1].kind == US_DOWN;
    if (u.kind != US_OUT && !to_down) U.out[i] = b.take(ob);
  }
  U.cat = b.take(cat);
  return U;
}

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

Layout layout_of(const dp_block_desc* d);

Layout layout_of(const dp_block_desc* d) {
  Layout L;
  memset(&L, 0, sizeof(L));
  Bump b;
  const size_t e = d->dtype == DP_FP32 ? 4 : 2;
  const size_t hw = static_cast<size_t>(d->H) * d->W;
  L.status = b.take(sizeof(int));
  if (d->kind == DP_BLOCK_GN_CONV) {
    L.gn1 = gn_slots(b, d->P, d->G);
    for (int i = 0; i < 2; ++i) L.a1[i] = b.take(hw * d->C * e);
  } else if (d->kind == DP_BLOCK_RESBLOCK) {
    L.gn1 = gn_slots(b, d->P, d->G);
    L.gn2 = gn_slots(b, d->P, d->G);
    for (int i = 0; i < 2; ++i) L.a1[i] = b.take(hw * d->C * e);
    for (int i = 0; i < 2; ++i) L.a2[i] = b.take(hw * d->Cout * e);
    L.h = b.take(hw * d->Cout * e);
    if (d->C != d->Cout) L.sc = b.take(hw * d->Cout * e);
    if (d->temb_dim > 0) L.tbias = b.take(static_cast<size_t>(d->Cout) * sizeof(float));
  } else if (d->kind == DP_BLOCK_TRANSFORMER) {
    const size_t C = d->C, Tk = d->ctx_len, F = d->ff_inner;
    L.gn1 = gn_slots(b, d->P, d->G);
    L.act = b.take(hw * C * e);
    L.ha = b.take(hw * C * e);
    L.hb = b.take(hw * C * e);
    L.tn = b.take(hw * C * e);
    L.q = b.take(hw * C * e);
    // each layer's self-attention keeps its own stale keys and values
    L.kv_layer = 4 * ((hw * C * e + 255) & ~static_cast<size_t>(255));
    for (int i = 0; i < 2; ++i) L.k[i] = b.take(hw * C * e);
    for (int i = 0; i < 2; ++i) L.v[i] = b.take(hw * C * e);
    for (int l = 1; l < d->depth; ++l) b.take(L.kv_layer);
    L.o = b.take(hw * C * e);
    L.q2 = b.take(hw * C * e);
    // each layer's context keys and values (kept across steps when the context is fixed)
    L.kv2_layer = 2 * ((Tk * C * e + 255) & ~static_cast<size_t>(255));
    L.k2 = b.take(Tk * C * e);
    L.v2 = b.take(Tk * C * e);
    for (int l = 1; l < d->depth; ++l) b.take(L.kv2_layer);
    L.o2 = b.take(hw * C * e);
    L.ffh = b.take(hw * 2 * F * e);
    L.ffg = b.take(hw * F * e);
    L.attn_ws = b.take(attn_workspace_bytes());
  } else if (d->kind == DP_BLOCK_ATTN) {
    L.gn1 = gn_slots(b, d->P, d->G);
    L.act = b.take(hw * d->C * e);
    L.q = b.take(hw * d->C * e);
    for (int i = 0; i < 2; ++i) L.k[i] = b.take(hw * d->C * e);
    for (int i = 0; i < 2; ++i) L.v[i] = b.take(hw * d->C * e);
    L.o = b.take(hw * d->C * e);
    L.attn_ws = b.take(attn_workspace_bytes());
  } else if (d->kind == DP_BLOCK_UNET_SDXL) {
    unet_layout(d, b);
  } else {
    const MiniDescs m = mini_descs(d);
    const size_t hw2 = hw / 4, hw3 = hw / 16;
    for (int i = 0; i < 2; ++i) L.xin[i] = b.take(hw * d->C * 2);
    L.h0 = b.take(hw * kU1 * 2);
    L.rb1 = b.take(layout_of(&m.rb1).total);
    for (int i = 0; i < 2; ++i) L.d1[i] = b.take(hw * kU1 * 2);
    L.h1 = b.take(hw2 * kU1 * 2);
    L.rb2 = b.take(layout_of(&m.rb2).total);
    L.h2 = b.take(hw2 * kU2 * 2);
    L.at2 = b.take(layout_of(&m.at2).total);
    for (int i = 0; i < 2; ++i) L.d2[i] = b.take(hw2 * kU2 * 2);
    L.h3 = b.take(hw3 * kU2 * 2);
    L.rb3 = b.take(layout_of(&m.rb3).total);
    L.h4 = b.take(hw3 * kU3 * 2);
    L.at3 = b.take(layout_of(&m.at3).total);
  }
  L.gemm_ws = b.take(gemm_workspace_bytes());
  L.total = b.off;
  return L;
}

size_t layout_total(const dp_block_desc* d) { return layout_of(d).total; }

int desc_check(const dp_block_desc* d) {
  if (d && (d->depth < 1 || d->depth > 16 || (d->depth != 1 && d->kind != DP_BLOCK_TRANSFORMER)))
    return set_error(DP_ERR_INVALID_ARG, "block: depth %d (1..16, and above 1 only for TRANSFORMER)",
                     d->depth);
  if (d && (d->ctx_fixed != 0 && d->ctx_fixed != 1))
    return set_error(DP_ERR_INVALID_ARG, "block: fixed-context flag %d is not 0 or 1", d->ctx_fixed);
  if (d && d->gn_fuse != 0 && d->gn_fuse != 1)
    return set_error(DP_ERR_INVALID_ARG, "block: gn fusion flag %d is not 0 or 1", d->gn_fuse);
  if (!d) return set_error(DP_ERR_INVALID_ARG, "block: null descriptor");
  if (d->kind < DP_BLOCK_GN_CONV || d->kind > DP_BLOCK_UNET_SDXL)
    return set_error(DP_ERR_INVALID_ARG, "block: bad kind %d", d->kind);
  if (d->H <= 0 || d->W <= 0 || d->C <= 0 || d->Cout <= 0 || d->G <= 0 || d->P <= 0)
    return set_error(DP_ERR_INVALID_ARG, "block: non-positive size");
  if (d->dtype != DP_BF16 && d->dtype != DP_FP32)
    return set_error(DP_ERR_INVALID_ARG, "block: bad dtype");
  if (d->dtype == DP_FP32 && d->kind != DP_BLOCK_GN_CONV)
    return set_error(DP_ERR_UNSUPPORTED, "block: fp32 storage is only built for GN_CONV");
  if (!(d->eps > 0.f)) return set_error(DP_ERR_INVALID_ARG, "block: eps must be > 0");
  if (d->gn_stats < DP_GN_STATS_CORRECTED || d->gn_stats > DP_GN_STATS_SYNC)
    return set_error(DP_ERR_INVALID_ARG, "block: unknown GroupNorm statistics variant %d", d->gn_stats);
  if (d->H % d->P) return set_error(DP_ERR_UNSUPPORTED, "block: H %% P != 0");
  if (d->temb_dim < 0 || d->temb_dim > 8192)
    return set_error(DP_ERR_INVALID_ARG, "block: time-embedding width %d outside [0, 8192]", d->temb_dim);
  if (d->temb_dim && d->kind != DP_BLOCK_RESBLOCK && d->kind != DP_BLOCK_UNET_SDXL)
    return set_error(DP_ERR_INVALID_ARG, "block: a time embedding is only for RESBLOCK and UNET_SDXL blocks");
  if (d->kind == DP_BLOCK_UNET_SDXL) {
    if (d->C < 2 || d->C > 8 || d->C % 2)
      return set_error(DP_ERR_UNSUPPORTED, "block: SDXL U-Net latent needs an even C <= 8");
    if (d->Cout != d->C) return set_error(DP_ERR_INVALID_ARG, "block: SDXL U-Net needs Cout == C");
    if (d->unet_base <= 0 || d->unet_base % 64 || d->unet_base > 512)
      return set_error(DP_ERR_UNSUPPORTED, "block: SDXL U-Net base width %d (a multiple of 64, <= 512)",
                       d->unet_base);
    for (int l = 0; l < 3; ++l)
      if (d->unet_depth[l] < 0 || d->unet_depth[l] > 16)
        return set_error(DP_ERR_INVALID_ARG, "block: SDXL U-Net depth %d outside [0, 16]", d->unet_depth[l]);
    if (d->H % (4 * d->P) || d->W % 4)
      return set_error(DP_ERR_UNSUPPORTED, "block: SDXL U-Net needs H %% 4P == 0 and W %% 4 == 0");
    if (d->ctx_len < 1 || d->ctx_dim <= 0 || d->ctx_dim % 64 || d->ff_inner != 0)
      return set_error(DP_ERR_INVALID_ARG, "block: SDXL U-Net needs dp_block_desc_set_context "
                                           "(ctx_len >= 1, ctx_dim a multiple of 64, ff_inner 0)");
    if (d->temb_dim <= 0)
      return set_error(DP_ERR_INVALID_ARG, "block: SDXL U-Net needs dp_block_desc_set_time_embedding");
    for (const UStage& u : unet_stages(d)) {
      if (u.kind != US_RES && u.kind != US_TF && u.kind != US_OUT) continue;
      int rc = desc_check(&u.sub);
      if (rc) return rc;
    }
    return DP_OK;
  }
  if (d->kind == DP_BLOCK_UNET_MINI) {
    if (d->C > 16 || d->C % 2)
      return set_error(DP_ERR_UNSUPPORTED, "block: mini U-Net latent needs an even C <= 16");
    if (d->H % (4 * d->P) || d->W % 4)
      return set_error(DP_ERR_UNSUPPORTED, "block: mini U-Net needs H %% 4P == 0 and W %% 4 == 0");
    const MiniDescs m = mini_descs(d);
    const dp_block_desc* subs[5] = {&m.rb1, &m.rb2, &m.at2, &m.rb3, &m.at3};
    for (const dp_block_desc* s : subs) {
      int rc = desc_check(s);
      if (rc) return rc;
    }
    return DP_OK;
  }
  // GroupNorms act on the input channels (and on Cout inside a RESBLOCK)
  if (d->C % d->G || (d->kind != DP_BLOCK_GN_CONV && d->Cout % d->G))
    return set_error(DP_ERR_UNSUPPORTED, "block: channels %% G != 0");
  if (d->kind == DP_BLOCK_TRANSFORMER) {
    if (d->Cout != d->C) return set_error(DP_ERR_INVALID_ARG, "block: transformer keeps C");
    if (d->heads <= 0 || d->C != d->heads * 64)
      return set_error(DP_ERR_UNSUPPORTED, "block: transformer needs C == heads * 64");
    // the block's LayerNorms hold a token in one warp's registers; reject wider
    // tokens here, before a step has launched anything
    if (d->C > kLnMaxC)
      return set_error(DP_ERR_UNSUPPORTED, "block: transformer needs C <= %d (LayerNorm width)", kLnMaxC);
    const int T = d->H * d->W;
    if ((T / d->P) % 128 || T % 256)
      return set_error(DP_ERR_UNSUPPORTED, "block: transformer needs (H*W/P) %% 128 == 0 and H*W %% 256 == 0");
    if (d->ctx_len < 1 || d->ctx_dim <= 0 || d->ctx_dim % 64 || d->ff_inner <= 0 || d->ff_inner % 64)
      return set_error(DP_ERR_INVALID_ARG, "block: transformer needs dp_block_desc_set_context "
                                           "(ctx_len >= 1, ctx_dim and ff_inner multiples of 64)");
  }
  if (d->kind == DP_BLOCK_ATTN) {
    if (d->Cout != d->C) return set_error(DP_ERR_INVALID_ARG, "block: attention keeps C");
    if (d->heads <= 0 || d->C != d->heads * 64)
      return set_error(DP_ERR_UNSUPPORTED, "block: attention needs C == heads * 64");
    const int T = d->H * d->W;
    if ((T / d->P) % 128) return set_error(DP_ERR_UNSUPPORTED, "block: tokens per band %% 128 != 0");
  }
  return DP_OK;
}

int weight_count(const dp_block_desc* d) {
  if (d->kind == DP_BLOCK_GN_CONV) return 4;
  if (d->kind == DP_BLOCK_RESBLOCK) return (d->C != d->Cout ? 10 : 8) + (d->temb_dim > 0 ? 3 : 0);
  if (d->kind == DP_BLOCK_ATTN) return 6;
  if (d->kind == DP_BLOCK_TRANSFORMER) return 7 + 18 * d->depth;
  if (d->kind == DP_BLOCK_UNET_SDXL) {
    int n = 2;   // context, time embedding
    for (const UStage& u : unet_stages(d)) n += stage_weight_count(u);
    return n;
  }
  const MiniDescs m = mini_descs(d);
  return 2 + weight_count(&m.rb1) + 2 + weight_count(&m.rb2) + weight_count(&m.at2) + 2 +
         weight_count(&m.rb3) + weight_count(&m.at3);
}

int stage_weight_count(const UStage& u) {
  if (u.kind == US_RES || u.kind == US_TF) return weight_count(&u.sub) - 1;
  if (u.kind == US_OUT) return weight_count(&u.sub);
  return 2;
}

double flops_of(const dp_block_desc* d) {
  const double hw = static_cast<double>(d->H) * d->W;
  const double C = d->C, Co = d->Cout;
  if (d->kind == DP_BLOCK_GN_CONV) return 2.0 * hw * Co * 9.0 * C;
  if (d->kind == DP_BLOCK_RESBLOCK)
    return 2.0 * hw * Co * 9.0 * C + 2.0 * hw * Co * 9.0 * Co + (C != Co ? 2.0 * hw * Co * C : 0.0) +
           2.0 * Co * d->temb_dim;
  if (d->kind == DP_BLOCK_ATTN)
    return 2.0 * hw * 3.0 * C * C + 4.0 * hw * hw * C + 2.0 * hw * C * C;
  if (d->kind == DP_BLOCK_TRANSFORMER) {
    const double Tk = d->ctx_len, Cc = d->ctx_dim, F = d->ff_inner;
    return 2.0 * hw * C * C * 2.0 +                        // proj_in, proj_out
           d->depth * (2.0 * hw * C * C * 3.0 +             // wo, cq, co
                       2.0 * hw * 3.0 * C * C + 4.0 * hw * hw * C +   // q/k/v, self-attention
                       (d->ctx_fixed ? 0.0 : 2.0 * Tk * 2.0 * C * Cc) +   // context k/v (kept when fixed)
                       4.0 * hw * Tk * C +                             // cross-attention
                       2.0 * hw * 2.0 * F * C + 2.0 * hw * C * F);    // ff1, ff2
  }
  if (d->kind == DP_BLOCK_UNET_SDXL) {
    double f = 0.0;
    for (const UStage& u : unet_stages(d)) {
      const double uhw = static_cast<double>(u.H) * u.W;
      if (u.kind == US_CONV_IN) f += 2.0 * uhw * u.co * 9.0 * u.ci;
      else if (u.kind == US_DOWN) f += 2.0 * (uhw / 4) * u.co * 9.0 * u.ci;
      else if (u.kind == US_UP) f += 2.0 * (4 * uhw) * u.co * 9.0 * u.ci;
      else f += flops_of(&u.sub);
    }
    return f;
  }
  const MiniDescs m = mini_descs(d);
  return 2.0 * hw * kU1 * 9.0 * C + flops_of(&m.rb1) + 2.0 * (hw / 4) * kU1 * 9.0 * kU1 +
         flops_of(&m.rb2) + flops_of(&m.at2) + 2.0 * (hw / 16) * kU2 * 9.0 * kU2 +
         flops_of(&m.rb3) + flops_of(&m.at3);
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

// When a step runs in planning mode it records every launch it would make
// (kernel kind, algorithmic flops, algorithmic bytes) instead of launching;
// the launch count and per-launch work reported by the ABI come from here,
// so they follow the step's own code path.
struct LaunchRec {
  int kind;
  double flops, bytes;
};
struct Plan {
  std::vector<LaunchRec> rec;
  int n = 0;
  void push(int kind, double flops, double bytes) {
    rec.push_back({kind, flops, bytes});
    ++n;
  }
};

// One step of the block described by `d` whose state lives at `ws`; `cur`
// selects the stale half of every ping-pong pair (the fresh half is cur ^ 1).
// Whether a GroupNorm -> 3x3 conv pair of this block runs as the statistics
// pass plus the conv that normalises its own input tiles: when the descriptor
// asks for it (dp_block_desc_set_gn_fusion) and the shapes allow it.
bool gn_conv_fused(const dp_block_desc* d, int ch, int co) {
  return d->gn_fuse == 1 && conv3x3_gn_eligible(d->H, d->W, ch, co, d->G, d->dtype);
}

int step_impl(const dp_block_desc* d, void* ws, int cur, const void* x, void* out,
              const void* const* w, int mode, int first, cudaStream_t st, Plan* plan) {
  const Layout L = layout_of(d);
  const double e = d->dtype == DP_FP32 ? 4.0 : 2.0;
  const int f = cur ^ 1, o = cur;
  const int H = d->H, W = d->W, C = d->C, Co = d->Cout, G = d->G, P = d->P;
  // statistics of this step's GroupNorms: a displaced step takes the
  // descriptor's variant (corrected, band-local, stale-only or exact)
  int gn_mode = mode;
  float gn_w = d->w;
  if (mode == DP_MODE_DISPLACED) {
    if (d->gn_stats == DP_GN_STATS_LOCAL) gn_mode = DP_MODE_NAIVE;
    if (d->gn_stats == DP_GN_STATS_STALE) gn_w = 0.0f;
    if (d->gn_stats == DP_GN_STATS_SYNC) gn_mode = DP_MODE_SYNC;
  }
  auto gn = [&](const GnSlots& g, const void* in, void* y, const void* gamma, const void* beta,
                int ch, int silu) {
    if (plan) {
      const double bytes = static_cast<double>(H) * W * ch * e;
      int nb, chunk, th;
      size_t sm;
      if (gn_cluster_plan(H, W, ch, G, P, d->dtype, gn_mode, &nb, &chunk, &th, &sm)) {
        plan->push(DP_KERNEL_GN_CLUSTER, 0.0, 2.0 * bytes);
      } else if (gn_fused_plan(H, W, ch, G, P, d->dtype, &nb, &chunk, &th, &sm)) {
        plan->push(DP_KERNEL_GN_FUSED, 0.0, 2.0 * bytes);
      } else {
        plan->push(DP_KERNEL_GN_STATS, 0.0, bytes);
        plan->push(DP_KERNEL_GN_APPLY, 0.0, 2.0 * bytes);
      }
      return DP_OK;
    }
    return gn_launch(in, y, static_cast<const float*>(gamma), static_cast<const float*>(beta), H,
                     W, ch, G, P, d->eps, gn_w, silu, gn_mode, d->dtype, at<float>(ws, g.global[o]),
                     at<float>(ws, g.local[o]), at<float>(ws, g.local[f]),
                     at<float>(ws, g.global[f]), at<float>(ws, g.used), at<void>(ws, g.ws),
                     gn_workspace_bytes(P, G), st);
  };
  // conv / linear / attention launches, or their records in planning mode
  auto conv = [&](const void* af, const void* as, const void* wt, const void* b, const void* res,
                  void* y, int h, int wd, int ci, int co, int stride) {
    if (plan) {
      const double ho = (h - 1) / stride + 1, wo = (wd - 1) / stride + 1;
      const int S = conv3x3_splits(h, wd, ci, co, stride, d->dtype, true);
      if (conv3x3_is_narrow(co)) {
        plan->push(DP_KERNEL_CONV_NARROW, 2.0 * ho * wo * co * 9.0 * ci,
                   (static_cast<double>(h) * wd * ci + ho * wo * co * (res ? 2 : 1)) * e);
      } else if (d->dtype == DP_FP32) {
        plan->push(DP_KERNEL_CONV_F32, 2.0 * ho * wo * co * 9.0 * ci,
                   (static_cast<double>(h) * wd * ci + ho * wo * co * (res ? 2 : 1)) * e);
      } else if (S == 1) {
        plan->push(DP_KERNEL_CONV, 2.0 * ho * wo * co * 9.0 * ci,
                   (static_cast<double>(h) * wd * ci + ho * wo * co * (res ? 2 : 1)) * e);
      } else {
        plan->push(DP_KERNEL_CONV, 2.0 * ho * wo * co * 9.0 * ci,
                   static_cast<double>(h) * wd * ci * e + ho * wo * co * 4.0 * S);
        plan->push(DP_KERNEL_SPLITK_FINISH, 0.0, ho * wo * co * (4.0 * S + e * (res ? 2 : 1)));
      }
      return DP_OK;
    }
    return conv3x3_launch(af, as, wt, static_cast<const float*>(b), res, y, h, wd, ci, co, stride, P,
                          mode, d->dtype, at<void>(ws, L.gemm_ws), gemm_workspace_bytes(), st);
  };
  auto lin = [&](const void* in, const void* wt, const void* b, const void* res, void* o0, void* o1,
                 void* o2, int M, int N, int K, int split) {
    if (plan) {
      const int S = linear_splits(M, N, K, split, true);
      const double mn = static_cast<double>(M) * N;
      if (S == 1) {
        plan->push(DP_KERNEL_LINEAR, 2.0 * mn * K, (static_cast<double>(M) * K + mn * (res ? 2 : 1)) * e);
      } else {
        plan->push(DP_KERNEL_LINEAR, 2.0 * mn * K, static_cast<double>(M) * K * e + mn * 4.0 * S);
        plan->push(DP_KERNEL_SPLITK_FINISH, 0.0, mn * (4.0 * S + e * (res ? 2 : 1)));
      }
      return DP_OK;
    }
    return linear_launch(in, wt, static_cast<const float*>(b), res, o0, o1, o2, M, N, K, split,
                         at<void>(ws, L.gemm_ws), gemm_workspace_bytes(), st);
  };
  // GroupNorm (+SiLU) -> 3x3 conv, in two calls: gn_part, then conv_part.
  // Where the conv can normalise its own input tiles (gn_conv_fused), the
  // GroupNorm runs as its statistics pass only and the conv reads x itself:
  // the normalised activations never go through HBM, and the ping-pong
  // buffer `a` receives only the band-edge rows, the rows the next step's
  // displaced conv reads from other bands.  Otherwise the GroupNorm writes
  // `a` whole and the conv reads it.
  auto gn_part = [&](const GnSlots& g, const void* in, const size_t a_off[2], const void* gamma,
                     const void* beta, int ch, int co, int silu) {
    if (!gn_conv_fused(d, ch, co)) return gn(g, in, at<void>(ws, a_off[f]), gamma, beta, ch, silu);
    if (plan) {
      plan->push(DP_KERNEL_GN_STATS, 0.0, static_cast<double>(H) * W * ch * e);
      return DP_OK;
    }
    return gn_stats_launch(in, H, W, ch, G, P, gn_w, gn_mode, d->dtype, at<float>(ws, g.global[o]),
                           at<float>(ws, g.local[o]), at<float>(ws, g.local[f]),
                           at<float>(ws, g.global[f]), at<float>(ws, g.used), at<void>(ws, g.ws), st);
  };
  auto conv_part = [&](const GnSlots& g, const void* in, const size_t a_off[2], const void* gamma,
                       const void* beta, int ch, int co, int silu, const void* wt, const void* b,
                       const void* res, void* y) {
    if (!gn_conv_fused(d, ch, co))
      return conv(at<void>(ws, a_off[f]), at<void>(ws, a_off[o]), wt, b, res, y, H, W, ch, co, 1);
    if (plan) {
      const double hw = static_cast<double>(H) * W;
      plan->push(DP_KERNEL_CONV_GN, 2.0 * hw * co * 9.0 * ch,
                 (hw * ch + hw * co * (res ? 2 : 1) + 2.0 * P * W * ch) * e);
      return DP_OK;
    }
    return conv3x3_gn_launch(in, at<void>(ws, a_off[o]), at<void>(ws, a_off[f]), at<float>(ws, g.used),
                             static_cast<const float*>(gamma), static_cast<const float*>(beta), G, d->eps,
                             silu, wt, static_cast<const float*>(b), res, y, H, W, ch, co, P, mode, st);
  };
  int rc;
  if (d->kind != DP_BLOCK_UNET_MINI && d->kind != DP_BLOCK_UNET_SDXL && !plan) {
    // biases (conv_b, conv1_b, conv2_b, short_b, temb_b; bqkv, bo, ...) may be NULL
    const int temb_b = weight_count(d) - 2;   // RESBLOCK with a time embedding: temb_b
    for (int i = 0; i < weight_count(d); ++i) {
      const int tl = (i - 4) % 18;   // TRANSFORMER: index within a layer's 18 pointers
      const bool bias = d->kind == DP_BLOCK_ATTN          ? (i == 3 || i == 5)
                        : d->kind == DP_BLOCK_TRANSFORMER ? (i == 3 || i == 5 + 18 * d->depth ||
                                                             (i >= 4 && i < 4 + 18 * d->depth &&
                                                              (tl == 3 || tl == 5 || tl == 11 || tl == 15 ||
                                                               tl == 17)))
                                                          : (i == 3 || i == 7 || i == 9 ||
                                                             (d->temb_dim > 0 && i == temb_b));
      if (!w[i] && !bias) return set_error(DP_ERR_INVALID_ARG, "block: weight %d is NULL", i);
    }
  }
  if (d->kind == DP_BLOCK_GN_CONV) {
    if (!plan) {
      rc = conv3x3_validate(x, x, w[2], nullptr, out, H, W, C, Co, 1, P, mode, d->dtype);
      if (rc) return rc;
    }
    const size_t a1[2] = {L.a1[0], L.a1[1]};
    rc = gn_part(L.gn1, x, a1, w[0], w[1], C, Co, d->silu);
    if (rc) return rc;
    return conv_part(L.gn1, x, a1, w[0], w[1], C, Co, d->silu, w[2], w[3], nullptr, out);
  }
  if (d->kind == DP_BLOCK_RESBLOCK) {
    if (!plan) {
      rc = conv3x3_validate(x, x, w[2], nullptr, out, H, W, C, Co, 1, P, mode, d->dtype);
      if (rc) return rc;
      rc = conv3x3_validate(x, x, w[6], nullptr, out, H, W, Co, Co, 1, P, mode, d->dtype);
      if (rc) return rc;
    }
    void* h = at<void>(ws, L.h);
    const void* b1 = w[3];
    if (d->temb_dim > 0) {
      // the step's time embedding (temb_w, temb_b, then temb), folded with
      // conv1_b into conv1's bias
      const int t0 = C != Co ? 10 : 8;
      const int Ct = d->temb_dim;
      if (plan) {
        plan->push(DP_KERNEL_TEMB, 2.0 * Co * Ct, (static_cast<double>(Co) * Ct + Ct + 3.0 * Co) * 4.0);
      } else {
        float* tb = at<float>(ws, L.tbias);
        rc = temb_bias_validate(w[t0 + 2], w[t0], w[t0 + 1], w[3], tb, Ct, Co);
        if (rc) return rc;
        rc = temb_bias_launch(static_cast<const float*>(w[t0 + 2]), static_cast<const float*>(w[t0]),
                              static_cast<const float*>(w[t0 + 1]), static_cast<const float*>(w[3]), tb,
                              Ct, Co, st);
        if (rc) return rc;
        b1 = tb;
      }
    }
    const size_t a1[2] = {L.a1[0], L.a1[1]}, a2[2] = {L.a2[0], L.a2[1]};
    rc = gn_part(L.gn1, x, a1, w[0], w[1], C, Co, 1);
    if (rc) return rc;
    rc = conv_part(L.gn1, x, a1, w[0], w[1], C, Co, 1, w[2], b1, nullptr, h);
    if (rc) return rc;
    rc = gn_part(L.gn2, h, a2, w[4], w[5], Co, Co, 1);
    if (rc) return rc;
    const void* res = x;
    if (C != Co) {
      void* sc = at<void>(ws, L.sc);
      rc = lin(x, w[8], w[9], nullptr, sc, nullptr, nullptr, H * W, Co, C, Co);
      if (rc) return rc;
      res = sc;
    }
    return conv_part(L.gn2, h, a2, w[4], w[5], Co, Co, 1, w[6], w[7], res, out);
  }
  if (d->kind == DP_BLOCK_TRANSFORMER) {
    const int T = H * W, Tk = d->ctx_len, Cc = d->ctx_dim, Fi = d->ff_inner;
    void* act = at<void>(ws, L.act);
    void* ha = at<void>(ws, L.ha);
    void* hb = at<void>(ws, L.hb);
    void* tn = at<void>(ws, L.tn);
    void* q = at<void>(ws, L.q);
    void* ob = at<void>(ws, L.o);
    void* q2 = at<void>(ws, L.q2);
    void* o2 = at<void>(ws, L.o2);
    void* ffh = at<void>(ws, L.ffh);
    void* ffg = at<void>(ws, L.ffg);
    auto ln = [&](const void* in, void* y, const void* g, const void* b) {
      if (plan) {
        plan->push(DP_KERNEL_LAYERNORM, 0.0, 2.0 * T * C * e);
        return DP_OK;
      }
      return dp_layernorm(in, y, static_cast<const float*>(g), static_cast<const float*>(b), T, C, 1e-5f, st);
    };
    rc = gn(L.gn1, x, act, w[0], w[1], C, 0);
    if (rc) return rc;
    rc = lin(act, w[2], w[3], nullptr, ha, nullptr, nullptr, T, C, C, C);   // proj_in
    if (rc) return rc;
    const void* ctx = w[6 + 18 * d->depth];
    void* cur = ha;     // the residual stream entering the layer
    void* other = hb;
    for (int l = 0; l < d->depth; ++l) {
      const void* const* lw = w + 4 + 18 * l;   // this layer's 18 pointers
      void* kf = at<void>(ws, L.k[f] + l * L.kv_layer);
      void* vf = at<void>(ws, L.v[f] + l * L.kv_layer);
      // self-attention: other bands' keys and values are the previous step's
      rc = ln(cur, tn, lw[0], lw[1]);
      if (rc) return rc;
      rc = lin(tn, lw[2], lw[3], nullptr, q, kf, vf, T, 3 * C, C, C);
      if (rc) return rc;
      if (plan) {
        const double keys = mode == DP_MODE_NAIVE ? static_cast<double>(T) / P : T;
        plan->push(DP_KERNEL_ATTN, 4.0 * T * keys * C, 4.0 * T * C * e);
      } else {
        rc = attn_launch(q, kf, vf, at<void>(ws, L.k[o] + l * L.kv_layer), at<void>(ws, L.v[o] + l * L.kv_layer),
                         ob, T, d->heads, P, 0.125f, mode, at<void>(ws, L.attn_ws), attn_workspace_bytes(), st);
        if (rc) return rc;
      }
      rc = lin(ob, lw[4], lw[5], cur, other, nullptr, nullptr, T, C, C, C);
      if (rc) return rc;
      // cross-attention over the step's text context: the same for every band
      rc = ln(other, tn, lw[6], lw[7]);
      if (rc) return rc;
      rc = lin(tn, lw[8], nullptr, nullptr, q2, nullptr, nullptr, T, C, C, C);
      if (rc) return rc;
      void* k2 = at<void>(ws, L.k2 + l * L.kv2_layer);
      void* v2 = at<void>(ws, L.v2 + l * L.kv2_layer);
      // a fixed context's keys and values are computed at the state's first step and kept
      if (!d->ctx_fixed || first) {
        rc = lin(ctx, lw[9], nullptr, nullptr, k2, v2, nullptr, Tk, 2 * C, Cc, C);
        if (rc) return rc;
      }
      if (plan) {
        plan->push(DP_KERNEL_ATTN, 4.0 * T * static_cast<double>(Tk) * C, (2.0 * T * C + 2.0 * Tk * C) * e);
      } else {
        rc = attn_launch_tk(q2, k2, v2, nullptr, nullptr, o2, T, Tk, d->heads, 1, 0.125f, DP_MODE_SYNC,
                            at<void>(ws, L.attn_ws), attn_workspace_bytes(), st);
        if (rc) return rc;
      }
      rc = lin(o2, lw[10], lw[11], other, cur, nullptr, nullptr, T, C, C, C);
      if (rc) return rc;
      // gated feed-forward
      rc = ln(cur, tn, lw[12], lw[13]);
      if (rc) return rc;
      // ff1 with the gated GELU in its epilogue when the pair kernel tiles it;
      // otherwise ff1, then the interleaved GEGLU pass
      if (linear_geglu_fusable(T, Fi, C)) {
        if (plan) {
          plan->push(DP_KERNEL_LINEAR, 2.0 * T * 2.0 * Fi * C, (static_cast<double>(T) * C + 1.0 * T * Fi) * e);
        } else {
          rc = linear_geglu_launch(tn, lw[14], static_cast<const float*>(lw[15]), ffg, T, Fi, C, st);
          if (rc) return rc;
        }
      } else {
        rc = lin(tn, lw[14], lw[15], nullptr, ffh, nullptr, nullptr, T, 2 * Fi, C, 2 * Fi);
        if (rc) return rc;
        if (plan) {
          plan->push(DP_KERNEL_GEGLU, 0.0, 3.0 * T * Fi * e);
        } else {
          rc = geglu_launch(ffh, ffg, T, Fi, true, st);
          if (rc) return rc;
        }
      }
      rc = lin(ffg, lw[16], lw[17], cur, other, nullptr, nullptr, T, C, Fi, C);
      if (rc) return rc;
      void* t = cur;   // the layer's output is the next layer's input
      cur = other;
      other = t;
    }
    return lin(cur, w[4 + 18 * d->depth], w[5 + 18 * d->depth], x, out, nullptr, nullptr, T, C, C, C);   // proj_out + x
  }
  if (d->kind == DP_BLOCK_ATTN) {
    const int T = H * W;
    void* act = at<void>(ws, L.act);
    void* q = at<void>(ws, L.q);
    void* kf = at<void>(ws, L.k[f]);
    void* vf = at<void>(ws, L.v[f]);
    void* ob = at<void>(ws, L.o);
    rc = gn(L.gn1, x, act, w[0], w[1], C, 0);
    if (rc) return rc;
    rc = lin(act, w[2], w[3], nullptr, q, kf, vf, T, 3 * C, C, C);
    if (rc) return rc;
    if (plan) {
      const double keys = mode == DP_MODE_NAIVE ? static_cast<double>(T) / P : T;
      plan->push(DP_KERNEL_ATTN, 4.0 * T * keys * C, 4.0 * T * C * e);
    } else {
      rc = attn_launch(q, kf, vf, at<void>(ws, L.k[o]), at<void>(ws, L.v[o]), ob, T, d->heads, P,
                       0.125f, mode, at<void>(ws, L.attn_ws), attn_workspace_bytes(), st);
      if (rc) return rc;
    }
    return lin(ob, w[4], w[5], x, out, nullptr, nullptr, T, C, C, C);
  }
  if (d->kind == DP_BLOCK_UNET_SDXL) {
    Bump b;
    b.take(sizeof(int));   // the status word, as layout_of
    const ULayout U = unet_layout(d, b);
    const int nw = weight_count(d);
    const void* ctx = w[nw - 2];
    const void* temb = w[nw - 1];
    std::vector<const void*> skips, sw;
    const void* h = nullptr;
    int wi = 0;
    for (size_t i = 0; i < U.st.size(); ++i) {
      const UStage& u = U.st[i];
      const void* const* uw = w + wi;
      wi += stage_weight_count(u);
      void* sub_ws = at<void>(ws, U.ws[i]);
      // the output of a stage that feeds a down conv goes into that conv's input pair
      const bool to_down = i + 1 < U.st.size() && U.st[i + 1].kind == US_DOWN;
      void* dst = to_down ? at<void>(ws, f ? U.pair1[i + 1] : U.pair0[i + 1]) : at<void>(ws, U.out[i]);
      void* pf = at<void>(ws, f ? U.pair1[i] : U.pair0[i]);
      void* po = at<void>(ws, o ? U.pair1[i] : U.pair0[i]);
      const size_t uhw = static_cast<size_t>(u.H) * u.W;
      if ((u.kind == US_CONV_IN || u.kind == US_DOWN || u.kind == US_UP) && !plan && !uw[0])
        return set_error(DP_ERR_INVALID_ARG, "block: conv weight of U-Net stage %zu is NULL", i);
      if (u.kind == US_CONV_IN) {
        const size_t xb = uhw * u.ci * 2;
        if (plan) {
          plan->push(DP_KERNEL_COPY, 0.0, 2.0 * xb);
          plan->push(DP_KERNEL_CONV_SMALL, 2.0 * uhw * u.co * 9.0 * u.ci, static_cast<double>(uhw) * (u.ci + u.co) * 2.0);
        } else {
          rc = copy_launch(x, pf, xb, st);
          if (rc) return rc;
          rc = conv3x3_small_launch(pf, po, uw[0], static_cast<const float*>(uw[1]), dst, u.H, u.W, u.ci, u.co, P,
                                    mode, st);
          if (rc) return rc;
        }
      } else if (u.kind == US_DOWN || u.kind == US_UP) {
        int hc = u.H, wc = u.W, stride = 2;
        if (u.kind == US_UP) {
          hc = 2 * u.H;
          wc = 2 * u.W;
          stride = 1;
          if (plan) {
            plan->push(DP_KERNEL_UPSAMPLE, 0.0, 5.0 * uhw * u.ci * 2.0);
          } else {
            rc = upsample2x_launch(h, pf, u.H, u.W, u.ci, DP_BF16, st);
            if (rc) return rc;
          }
        }
        if (!plan) {
          rc = conv3x3_validate(pf, po, uw[0], nullptr, dst, hc, wc, u.ci, u.co, stride, P, mode, DP_BF16);
          if (rc) return rc;
        }
        rc = conv(pf, po, uw[0], uw[1], nullptr, dst, hc, wc, u.ci, u.co, stride);
        if (rc) return rc;
      } else if (u.kind == US_RES) {
        const void* in = h;
        if (u.cat) {
          void* cat = at<void>(ws, U.cat);
          const int ch = U.st[i - 1].co;   // the running tensor's channels; the skip has the rest
          const int ck = u.ci - ch;
          if (plan) {
            plan->push(DP_KERNEL_CONCAT, 0.0, 2.0 * uhw * u.ci * 2.0);
          } else {
            rc = concat_launch(h, skips.back(), cat, uhw, ch, ck, DP_BF16, st);
            if (rc) return rc;
          }
          skips.pop_back();
          in = cat;
        }
        sw.assign(uw, uw + stage_weight_count(u));
        sw.push_back(temb);
        rc = step_impl(&u.sub, sub_ws, cur, in, dst, sw.data(), mode, first, st, plan);
        if (rc) return rc;
      } else if (u.kind == US_TF) {
        sw.assign(uw, uw + stage_weight_count(u));
        sw.push_back(ctx);
        rc = step_impl(&u.sub, sub_ws, cur, h, dst, sw.data(), mode, first, st, plan);
        if (rc) return rc;
      } else {   // US_OUT
        return step_impl(&u.sub, sub_ws, cur, h, out, uw, mode, first, st, plan);
      }
      h = dst;
      if (u.skip) skips.push_back(h);
    }
    return set_error(DP_ERR_INVALID_ARG, "block: SDXL U-Net without an output stage");
  }
  // UNET_MINI
  const MiniDescs m = mini_descs(d);
  const int H2 = H / 2, W2 = W / 2, H3 = H / 4, W3 = W / 4;
  int wi = 0;
  auto take = [&](int n) {
    const void* const* p = w + wi;
    wi += n;
    return p;
  };
  void* xin = at<void>(ws, L.xin[f]);
  const size_t xbytes = static_cast<size_t>(H) * W * C * 2;
  if (plan) {
    plan->push(DP_KERNEL_COPY, 0.0, 2.0 * xbytes);
    plan->push(DP_KERNEL_CONV_SMALL, 2.0 * H * W * kU1 * 9.0 * C,
               static_cast<double>(H) * W * (C + kU1) * 2.0);
  } else {
    rc = copy_launch(x, xin, xbytes, st);
    if (rc) return rc;
  }
  const void* const* wc = take(2);
  if (!plan) {
    if (!wc[0]) return set_error(DP_ERR_INVALID_ARG, "block: conv_in weight is NULL");
    rc = conv3x3_small_launch(xin, at<void>(ws, L.xin[o]), wc[0], static_cast<const float*>(wc[1]),
                              at<void>(ws, L.h0), H, W, C, kU1, P, mode, st);
    if (rc) return rc;
  }
  rc = step_impl(&m.rb1, at<void>(ws, L.rb1), cur, at<void>(ws, L.h0), at<void>(ws, L.d1[f]),
                 take(weight_count(&m.rb1)), mode, first, st, plan);
  if (rc) return rc;
  wc = take(2);
  if (!plan) {
    if (!wc[0]) return set_error(DP_ERR_INVALID_ARG, "block: down1 weight is NULL");
    rc = conv3x3_validate(at<void>(ws, L.d1[f]), at<void>(ws, L.d1[o]), wc[0], nullptr,
                          at<void>(ws, L.h1), H, W, kU1, kU1, 2, P, mode, DP_BF16);
    if (rc) return rc;
  }
  rc = conv(at<void>(ws, L.d1[f]), at<void>(ws, L.d1[o]), wc[0], wc[1], nullptr, at<void>(ws, L.h1),
            H, W, kU1, kU1, 2);
  if (rc) return rc;
  rc = step_impl(&m.rb2, at<void>(ws, L.rb2), cur, at<void>(ws, L.h1), at<void>(ws, L.h2),
                 take(weight_count(&m.rb2)), mode, first, st, plan);
  if (rc) return rc;
  rc = step_impl(&m.at2, at<void>(ws, L.at2), cur, at<void>(ws, L.h2), at<void>(ws, L.d2[f]),
                 take(weight_count(&m.at2)), mode, first, st, plan);
  if (rc) return rc;
  wc = take(2);
  if (!plan) {
    if (!wc[0]) return set_error(DP_ERR_INVALID_ARG, "block: down2 weight is NULL");
    rc = conv3x3_validate(at<void>(ws, L.d2[f]), at<void>(ws, L.d2[o]), wc[0], nullptr,
                          at<void>(ws, L.h3), H2, W2, kU2, kU2, 2, P, mode, DP_BF16);
    if (rc) return rc;
  }
  rc = conv(at<void>(ws, L.d2[f]), at<void>(ws, L.d2[o]), wc[0], wc[1], nullptr, at<void>(ws, L.h3),
            H2, W2, kU2, kU2, 2);
  if (rc) return rc;
  rc = step_impl(&m.rb3, at<void>(ws, L.rb3), cur, at<void>(ws, L.h3), at<void>(ws, L.h4),
                 take(weight_count(&m.rb3)), mode, first, st, plan);
  if (rc) return rc;
  (void)H3;
  (void)W3;
  return step_impl(&m.at3, at<void>(ws, L.at3), cur, at<void>(ws, L.h4), out,
                   take(weight_count(&m.at3)), mode, first, st, plan);
}

// Records the launches of one step of `d` in `mode`.
int plan_of(const dp_block_desc* d, int mode, Plan* plan) {
  const std::vector<const void*> null_w(weight_count(d) + 1, nullptr);
  return step_impl(d, nullptr, 0, nullptr, nullptr, null_w.data(), mode, 0, nullptr, plan);
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
  d->Cout = kind == DP_BLOCK_UNET_MINI ? dp::kU3 : (Cout > 0 ? Cout : C);
  d->G = G;
  d->P = P;
  d->heads = heads;
  d->dtype = dtype;
  d->silu = silu;
  d->eps = eps;
  d->w = w;
  d->gn_stats = DP_GN_STATS_CORRECTED;
  d->ctx_len = 0;
  d->ctx_dim = 0;
  d->ff_inner = 0;
  d->temb_dim = 0;
  d->gn_fuse = 0;
  d->depth = 1;
  d->ctx_fixed = 0;
  d->unet_base = kind == DP_BLOCK_UNET_SDXL ? 320 : 0;
  d->unet_depth[0] = kind == DP_BLOCK_UNET_SDXL ? 0 : 0;
  d->unet_depth[1] = kind == DP_BLOCK_UNET_SDXL ? 2 : 0;
  d->unet_depth[2] = kind == DP_BLOCK_UNET_SDXL ? 10 : 0;
  if (kind == DP_BLOCK_UNET_SDXL) d->Cout = C;
  // checked once dp_block_desc_set_context (and, for UNET_SDXL, _set_time_embedding) is called
  if (kind == DP_BLOCK_TRANSFORMER || kind == DP_BLOCK_UNET_SDXL) return DP_OK;
  return dp::desc_check(d);
}

int dp_block_desc_set_context(dp_block_desc* d, int ctx_len, int ctx_dim, int ff_inner) {
  if (!d) return dp::set_error(DP_ERR_INVALID_ARG, "block: null descriptor");
  if (d->kind != DP_BLOCK_TRANSFORMER && d->kind != DP_BLOCK_UNET_SDXL)
    return dp::set_error(DP_ERR_INVALID_ARG, "block: a context is only for TRANSFORMER and UNET_SDXL blocks");
  d->ctx_len = ctx_len;
  d->ctx_dim = ctx_dim;
  d->ff_inner = ff_inner;
  if (d->kind == DP_BLOCK_UNET_SDXL) {
    // the time embedding may still be unset: check the context alone
    if (ctx_len < 1 || ctx_dim <= 0 || ctx_dim % 64 || ff_inner != 0)
      return dp::set_error(DP_ERR_INVALID_ARG, "block: SDXL U-Net context needs ctx_len >= 1, ctx_dim a "
                                               "multiple of 64 and ff_inner 0");
    return d->temb_dim > 0 ? dp::desc_check(d) : DP_OK;
  }
  return dp::desc_check(d);
}

int dp_block_desc_set_depth(dp_block_desc* d, int depth) {
  if (!d) return dp::set_error(DP_ERR_INVALID_ARG, "block: null descriptor");
  if (d->kind != DP_BLOCK_TRANSFORMER)
    return dp::set_error(DP_ERR_INVALID_ARG, "block: a depth is only for TRANSFORMER blocks");
  if (depth < 1 || depth > 16) return dp::set_error(DP_ERR_INVALID_ARG, "block: depth %d outside [1, 16]", depth);
  d->depth = depth;
  return DP_OK;
}

int dp_block_desc_set_time_embedding(dp_block_desc* d, int temb_dim) {
  if (!d) return dp::set_error(DP_ERR_INVALID_ARG, "block: null descriptor");
  if (d->kind != DP_BLOCK_RESBLOCK && d->kind != DP_BLOCK_UNET_SDXL)
    return dp::set_error(DP_ERR_INVALID_ARG, "block: a time embedding is only for RESBLOCK and UNET_SDXL blocks");
  if (temb_dim < 0 || temb_dim > 8192)
    return dp::set_error(DP_ERR_INVALID_ARG, "block: time-embedding width %d outside [0, 8192]", temb_dim);
  d->temb_dim = temb_dim;
  if (d->kind == DP_BLOCK_UNET_SDXL && d->ctx_len == 0) return DP_OK;   // context still to come
  return dp::desc_check(d);
}

int dp_block_desc_set_unet(dp_block_desc* d, int base, int depth0, int depth1, int depth2) {
  if (!d) return dp::set_error(DP_ERR_INVALID_ARG, "block: null descriptor");
  if (d->kind != DP_BLOCK_UNET_SDXL)
    return dp::set_error(DP_ERR_INVALID_ARG, "block: U-Net widths and depths are only for UNET_SDXL blocks");
  if (base <= 0 || base % 64 || base > 512)
    return dp::set_error(DP_ERR_INVALID_ARG, "block: SDXL U-Net base width %d (a multiple of 64, <= 512)", base);
  const int dep[3] = {depth0, depth1, depth2};
  for (int l = 0; l < 3; ++l)
    if (dep[l] < 0 || dep[l] > 16)
      return dp::set_error(DP_ERR_INVALID_ARG, "block: SDXL U-Net depth %d outside [0, 16]", dep[l]);
  d->unet_base = base;
  for (int l = 0; l < 3; ++l) d->unet_depth[l] = dep[l];
  if (d->ctx_len == 0 || d->temb_dim == 0) return DP_OK;   // checked once both are set
  return dp::desc_check(d);
}

int dp_block_desc_set_context_fixed(dp_block_desc* d, int on) {
  if (!d) return dp::set_error(DP_ERR_INVALID_ARG, "block: null descriptor");
  if (d->kind != DP_BLOCK_TRANSFORMER && d->kind != DP_BLOCK_UNET_SDXL)
    return dp::set_error(DP_ERR_INVALID_ARG, "block: a fixed context is only for TRANSFORMER and UNET_SDXL blocks");
  if (on != 0 && on != 1) return dp::set_error(DP_ERR_INVALID_ARG, "block: fixed context must be 0 or 1");
  d->ctx_fixed = on;
  return DP_OK;
}

int dp_block_desc_set_gn_fusion(dp_block_desc* d, int on) {
  if (!d) return dp::set_error(DP_ERR_INVALID_ARG, "block: null descriptor");
  if (on != 0 && on != 1) return dp::set_error(DP_ERR_INVALID_ARG, "block: gn fusion must be 0 or 1");
  d->gn_fuse = on;
  return DP_OK;
}

int dp_block_desc_set_gn_stats(dp_block_desc* d, int variant) {
  if (!d) return dp::set_error(DP_ERR_INVALID_ARG, "block: null descriptor");
  if (variant < DP_GN_STATS_CORRECTED || variant > DP_GN_STATS_SYNC)
    return dp::set_error(DP_ERR_INVALID_ARG, "block: unknown GroupNorm statistics variant %d", variant);
  d->gn_stats = variant;
  return DP_OK;
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
  return dp::flops_of(d);
}

int dp_block_weight_count(const dp_block_desc* d) {
  int rc = dp::desc_check(d);
  if (rc) return rc;
  return dp::weight_count(d);
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
  if (n_weights < dp::weight_count(d))
    return dp::set_error(DP_ERR_INVALID_ARG, "block: %d weights given, %d needed", n_weights,
                         dp::weight_count(d));
  if (s->workspace_bytes < dp::layout_of(d).total)
    return dp::set_error(DP_ERR_INVALID_ARG, "block: workspace too small");
  {
    // every kernel of this step reports a timed-out wait in the state's own word
    dp::StatusScope scope(reinterpret_cast<int*>(static_cast<char*>(s->workspace) +
                                                 dp::layout_of(d).status));
    rc = dp::step_impl(d, s->workspace, s->cur, x, out, weights, mode, s->steps_done == 0 ? 1 : 0,
                       static_cast<cudaStream_t>(stream), nullptr);
  }
  if (rc) return rc;
  s->cur ^= 1;
  s->steps_done += 1;
  return DP_OK;
}

// A captured block step per ping-pong parity: exec[c] is the step whose stale
// halves are the `c` halves.
struct dp_block_graph {
  cudaGraphExec_t exec[2];
  void* workspace;   // the state the graphs were captured on
};

int dp_block_graph_create(const dp_block_desc* d, dp_block_state* s, const void* x, void* out,
                          const void* const* weights, int n_weights, int mode, void* stream,
                          dp_block_graph** graph) {
  int rc = dp::desc_check(d);
  if (rc) return rc;
  if (!graph) return dp::set_error(DP_ERR_INVALID_ARG, "block graph: null handle pointer");
  *graph = nullptr;
  if (!s || !s->workspace || !x || !out || !weights)
    return dp::set_error(DP_ERR_INVALID_ARG, "block graph: null argument");
  if (!stream) return dp::set_error(DP_ERR_INVALID_ARG, "block graph: capture needs a stream other than the default one");
  if (mode < DP_MODE_SYNC || mode > DP_MODE_NAIVE)
    return dp::set_error(DP_ERR_INVALID_ARG, "block graph: bad mode %d", mode);
  if (s->steps_done == 0)
    return dp::set_error(DP_ERR_STATE, "block graph: capture after the state's first step");
  if (x == out) return dp::set_error(DP_ERR_INVALID_ARG, "block graph: out aliases x");
  if (!dp::aligned16(x) || !dp::aligned16(out))
    return dp::set_error(DP_ERR_UNSUPPORTED, "block graph: x/out not 16-byte aligned");
  if (n_weights < dp::weight_count(d))
    return dp::set_error(DP_ERR_INVALID_ARG, "block graph: %d weights given, %d needed", n_weights,
                         dp::weight_count(d));
  const dp::Layout L = dp::layout_of(d);
  if (s->workspace_bytes < L.total) return dp::set_error(DP_ERR_INVALID_ARG, "block graph: workspace too small");
  auto* g = new (std::nothrow) dp_block_graph;
  if (!g) return dp::set_error(DP_ERR_INVALID_ARG, "block graph: out of host memory");
  g->exec[0] = g->exec[1] = nullptr;
  g->workspace = s->workspace;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  for (int par = 0; par < 2 && !rc; ++par) {
    rc = dp::cuda_check(cudaStreamBeginCapture(st, cudaStreamCaptureModeThreadLocal), "block graph: begin capture");
    if (rc) break;
    {
      dp::StatusScope scope(reinterpret_cast<int*>(static_cast<char*>(s->workspace) + L.status));
      rc = dp::step_impl(d, s->workspace, par, x, out, weights, mode, 0, st, nullptr);
    }
    cudaGraph_t cg = nullptr;
    const int rc_end = dp::cuda_check(cudaStreamEndCapture(st, &cg), "block graph: end capture");
    if (!rc) rc = rc_end;
    if (!rc) rc = dp::cuda_check(cudaGraphInstantiate(&g->exec[par], cg, 0), "block graph: instantiate");
    if (cg) cudaGraphDestroy(cg);
  }
  if (rc) {
    for (int par = 0; par < 2; ++par)
      if (g->exec[par]) cudaGraphExecDestroy(g->exec[par]);
    delete g;
    return rc;
  }
  *graph = g;
  return DP_OK;
}

int dp_block_graph_launch(dp_block_graph* graph, dp_block_state* s, void* stream) {
  if (!graph || !s) return dp::set_error(DP_ERR_INVALID_ARG, "block graph: null argument");
  if (s->workspace != graph->workspace)
    return dp::set_error(DP_ERR_INVALID_ARG, "block graph: launched on another state than it was captured on");
  int rc = dp::cuda_check(cudaGraphLaunch(graph->exec[s->cur & 1], static_cast<cudaStream_t>(stream)),
                          "block graph: launch");
  if (rc) return rc;
  s->cur ^= 1;
  s->steps_done += 1;
  return DP_OK;
}

int dp_block_graph_destroy(dp_block_graph* graph) {
  if (!graph) return DP_OK;
  int rc = DP_OK;
  for (int par = 0; par < 2; ++par)
    if (graph->exec[par] && !rc) rc = dp::cuda_check(cudaGraphExecDestroy(graph->exec[par]), "block graph: destroy");
  delete graph;
  return rc;
}

int dp_block_status(const dp_block_desc* d, const dp_block_state* s, void* stream, int* status) {
  int rc = dp::desc_check(d);
  if (rc) return rc;
  if (!s || !s->workspace || !status) return dp::set_error(DP_ERR_INVALID_ARG, "block: null argument");
  const dp::Layout L = dp::layout_of(d);
  if (s->workspace_bytes < L.total) return dp::set_error(DP_ERR_INVALID_ARG, "block: workspace too small");
  return dp::read_clear_status(reinterpret_cast<int*>(static_cast<char*>(s->workspace) + L.status),
                               static_cast<cudaStream_t>(stream), status);
}

int dp_block_launch_count(const dp_block_desc* d) {
  int rc = dp::desc_check(d);
  if (rc) return rc;
  dp::Plan plan;
  rc = dp::plan_of(d, DP_MODE_DISPLACED, &plan);
  if (rc) return rc;
  return plan.n;
}

int dp_block_launch_info(const dp_block_desc* d, int mode, int i, int* kind, double* flops,
                         double* bytes) {
  int rc = dp::desc_check(d);
  if (rc) return rc;
  if (mode < DP_MODE_SYNC || mode > DP_MODE_NAIVE)
    return dp::set_error(DP_ERR_INVALID_ARG, "block: bad mode %d", mode);
  dp::Plan plan;
  rc = dp::plan_of(d, mode, &plan);
  if (rc) return rc;
  if (i < 0 || i >= plan.n)
    return dp::set_error(DP_ERR_INVALID_ARG, "block: launch %d of %d", i, plan.n);
  if (kind) *kind = plan.rec[i].kind;
  if (flops) *flops = plan.rec[i].flops;
  if (bytes) *bytes = plan.rec[i].bytes;
  return DP_OK;
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
