"""Pins of the CPU oracle against facts fixed by the pages and by mathematics.

The pages print no worked example, so the oracle is pinned by:
  * the P = 1 reduction to the ordinary full-image block (library routines:
    torch group_norm, conv2d, scaled_dot_product_attention), which the pages
    require as "no quality degradation" of the original model when nothing is
    displaced (study.space summary, Abstract);
  * brute-force loops on tiny inputs (conv, attention, GroupNorm moments);
  * naive mode equal to independent crops (atlas.scime.ai summary, the naive
    patch baseline rows);
  * an unchanged input making displaced equal sync;
  * a uniform drift making the corrected statistics exact (reading R1, w = 1);
  * halo and attention locality;
  * zero warm-up distinguishable from sync (atlas.scime.ai summary, warm-up
    ablation rows).
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import dp_oracle as O

SYNC, DISPLACED, NAIVE = O.SYNC, O.DISPLACED, O.NAIVE


def rng(seed):
    return np.random.default_rng(seed)


def rand_gn_conv_weights(r, C, Co):
    return {
        "gn_gamma": 1 + 0.3 * r.standard_normal(C), "gn_beta": 0.3 * r.standard_normal(C),
        "conv_w": r.standard_normal((Co, C, 3, 3)) * math.sqrt(2 / (9 * C)),
        "conv_b": 0.3 * r.standard_normal(Co),
    }


def rand_res_weights(r, C, Co, prefix=""):
    w = {
        "gn1_gamma": 1 + 0.3 * r.standard_normal(C), "gn1_beta": 0.3 * r.standard_normal(C),
        "conv1_w": r.standard_normal((Co, C, 3, 3)) * math.sqrt(2 / (9 * C)),
        "conv1_b": 0.3 * r.standard_normal(Co),
        "gn2_gamma": 1 + 0.3 * r.standard_normal(Co), "gn2_beta": 0.3 * r.standard_normal(Co),
        "conv2_w": r.standard_normal((Co, Co, 3, 3)) * math.sqrt(2 / (9 * Co)),
        "conv2_b": 0.3 * r.standard_normal(Co),
    }
    if C != Co:
        w["short_w"] = r.standard_normal((Co, C, 1, 1)) * math.sqrt(2 / C)
        w["short_b"] = 0.3 * r.standard_normal(Co)
    return {prefix + k: v for k, v in w.items()}


def rand_attn_weights(r, C, prefix=""):
    w = {"gn_gamma": 1 + 0.3 * r.standard_normal(C), "gn_beta": 0.3 * r.standard_normal(C)}
    for n in ("wq", "wk", "wv", "wo"):
        w[n] = r.standard_normal((C, C)) * (1.0 / math.sqrt(C))
    for n in ("bq", "bk", "bv", "bo"):
        w[n] = 0.3 * r.standard_normal(C)
    return {prefix + k: v for k, v in w.items()}


T64 = lambda a: torch.from_numpy(np.asarray(a, dtype=np.float64))


# ---------------------------------------------------------------- library blocks
def lib_gn_conv(x, w, G, eps, silu=True):
    t = F.group_norm(T64(x)[None], G, T64(w["gn_gamma"]), T64(w["gn_beta"]), eps)
    if silu:
        t = F.silu(t)
    return F.conv2d(t, T64(w["conv_w"]), T64(w["conv_b"]), padding=1)[0].numpy()


def lib_resblock(x, w, G, eps, prefix="", temb=None):
    g = lambda n: T64(w[prefix + n])
    t = F.silu(F.group_norm(T64(x)[None], G, g("gn1_gamma"), g("gn1_beta"), eps))
    h = F.conv2d(t, g("conv1_w"), g("conv1_b"), padding=1)
    if temb is not None:
        h = h + F.linear(F.silu(T64(temb)), g("temb_w"), g("temb_b"))[None, :, None, None]
    t = F.silu(F.group_norm(h, G, g("gn2_gamma"), g("gn2_beta"), eps))
    res = T64(x)[None]
    if prefix + "short_w" in w:
        res = F.conv2d(res, g("short_w"), g("short_b"))
    return (F.conv2d(t, g("conv2_w"), g("conv2_b"), padding=1) + res)[0].numpy()


def lib_attn(x, w, G, eps, heads, prefix=""):
    g = lambda n: T64(w[prefix + n])
    C, H, W = x.shape
    t = F.group_norm(T64(x)[None], G, g("gn_gamma"), g("gn_beta"), eps)[0]
    tok = t.reshape(C, H * W).T
    q = tok @ g("wq").T + g("bq")
    k = tok @ g("wk").T + g("bk")
    v = tok @ g("wv").T + g("bv")
    d = C // heads
    sh = lambda z: z.reshape(H * W, heads, d).permute(1, 0, 2)
    o = F.scaled_dot_product_attention(sh(q), sh(k), sh(v))
    o = o.permute(1, 0, 2).reshape(H * W, C)
    out = o @ g("wo").T + g("bo") + T64(x).reshape(C, H * W).T
    return out.T.reshape(C, H, W).numpy()


def run_two_steps(kind, x0, x1, w, P, G, mode1, heads=0, wgt=1.0, silu=True):
    st = {}
    O.block_step(kind, st, x0, w, P, G, 1e-5, wgt, SYNC, "none", heads=heads, silu=silu)
    tr = {}
    y = O.block_step(kind, st, x1, w, P, G, 1e-5, wgt, mode1, "none", heads=heads, silu=silu,
                     trace=tr)
    return y, tr, st


# ---------------------------------------------------------------- P = 1 reduction
@pytest.mark.parametrize("mode", [SYNC, DISPLACED, NAIVE])
def test_p1_gn_conv_equals_library(mode):
    r = rng(1)
    C, H, W = 16, 6, 7
    w = rand_gn_conv_weights(r, C, 12)
    x0, x1 = r.standard_normal((C, H, W)), r.standard_normal((C, H, W))
    y, _, _ = run_two_steps("gn_conv", x0, x1, w, 1, 4, mode)
    np.testing.assert_allclose(y, lib_gn_conv(x1, w, 4, 1e-5), rtol=0, atol=1e-12)


@pytest.mark.parametrize("mode", [SYNC, DISPLACED])
@pytest.mark.parametrize("co", [8, 16])
def test_p1_resblock_equals_library(mode, co):
    r = rng(2)
    C, H, W = 8, 5, 6
    w = rand_res_weights(r, C, co)
    x0, x1 = r.standard_normal((C, H, W)), r.standard_normal((C, H, W))
    y, _, _ = run_two_steps("resblock", x0, x1, w, 1, 4, mode)
    np.testing.assert_allclose(y, lib_resblock(x1, w, 4, 1e-5), rtol=0, atol=1e-11)


@pytest.mark.parametrize("mode", [SYNC, DISPLACED])
def test_p1_attn_equals_library(mode):
    r = rng(3)
    C, H, W = 16, 4, 5
    w = rand_attn_weights(r, C)
    x0, x1 = r.standard_normal((C, H, W)), r.standard_normal((C, H, W))
    y, _, _ = run_two_steps("attn", x0, x1, w, 1, 4, mode, heads=4)
    np.testing.assert_allclose(y, lib_attn(x1, w, 4, 1e-5, 4), rtol=0, atol=1e-11)


@pytest.mark.parametrize("H,W", [(8, 8), (6, 10), (7, 5)])
def test_p1_stride2_conv_equals_library(H, W):
    r = rng(4)
    a = r.standard_normal((5, H, W))
    wt = r.standard_normal((3, 5, 3, 3))
    b = r.standard_normal(3)
    y = O.conv3x3_halo(a, None, wt, b, None, 1, SYNC, stride=2)
    ref = F.conv2d(T64(a)[None], T64(wt), T64(b), stride=2, padding=1)[0].numpy()
    np.testing.assert_allclose(y, ref, rtol=0, atol=1e-12)


def test_conv1x1_equals_library():
    r = rng(5)
    a = r.standard_normal((6, 4, 5))
    wt = r.standard_normal((3, 6, 1, 1))
    b = r.standard_normal(3)
    ref = F.conv2d(T64(a)[None], T64(wt), T64(b))[0].numpy()
    np.testing.assert_allclose(O.conv1x1(a, wt, b), ref, rtol=0, atol=1e-12)


def _unet_mini_weights(seed):
    """Random weights of the mini U-Net chain (the workload's own names and shapes, random
    affine parameters and biases so that no term hides behind a zero)."""
    from displaced_patch_parallelism_b200 import synth
    wl = synth.WORKLOADS["unet_mini_4x128x128"]
    r = rng(seed)
    wts = {}
    for name, shape, std in synth.unet_mini_weight_specs(4):
        wts[name] = r.standard_normal(shape) * std
    for name, c, kind in synth.affine_specs(wl):
        wts[name] = (1 + 0.2 * r.standard_normal(c)) if kind == "gamma" else 0.2 * r.standard_normal(c)
    return wts


def lib_unet_mini(x, w, G=32, eps=1e-5, heads=(10, 20)):
    """The mini U-Net chain composed from library operators only: conv2d (stride 1 and 2,
    padding 1), the library ResBlock and the library attention block with 10 and 20 heads."""
    conv = lambda t, n, s: F.conv2d(T64(t)[None], T64(w[n + "_w"]), T64(w[n + "_b"]), stride=s,
                                    padding=1)[0].numpy()
    h = conv(x, "conv_in", 1)
    h = lib_resblock(h, w, G, eps, "rb1.")
    h = conv(h, "down1", 2)
    h = lib_resblock(h, w, G, eps, "rb2.")
    h = lib_attn(h, w, G, eps, heads[0], "at2.")
    h = conv(h, "down2", 2)
    h = lib_resblock(h, w, G, eps, "rb3.")
    return lib_attn(h, w, G, eps, heads[1], "at3.")


@pytest.mark.parametrize("mode", [SYNC, DISPLACED])
def test_p1_unet_mini_equals_library(mode):
    """With one band the whole chain is the ordinary network: conv_in, ResBlock(320), a
    stride-2 downsampler, ResBlock(320->640) with its 1x1 shortcut, attention with 10 heads,
    a second downsampler, ResBlock(640->1280), attention with 20 heads -- composed here
    from library operators.  A wrong head count, stage order, stride or shortcut fails."""
    w = _unet_mini_weights(6)
    r = rng(7)
    x0, x1 = r.standard_normal((4, 8, 8)), r.standard_normal((4, 8, 8))
    st = {}
    O.unet_mini_step(st, x0, w, 1, 32, 1e-5, 1.0, SYNC, "none")
    y = O.unet_mini_step(st, x1, w, 1, 32, 1e-5, 1.0, mode, "none")
    assert y.shape == (1280, 2, 2)
    ref = lib_unet_mini(x1, w)
    tol = 1e-9 * np.abs(ref).max()
    np.testing.assert_allclose(y, ref, rtol=0, atol=tol)
    # the pin has teeth: other head counts give results far outside the tolerance
    for heads in ((20, 20), (10, 10)):
        assert np.abs(lib_unet_mini(x1, w, heads=heads) - ref).max() > 1e3 * tol


def test_unet_mini_naive_equals_independent_crops():
    """Zero warm-up's step 0 (naive) at P = 4: every band runs the whole chain as an image of
    its own -- its own GroupNorm statistics, zero rows beyond its edges in every conv (the
    stride-2 downsamplers included) and only its own tokens as keys -- so the output is the
    library chain of each band's crop, stacked."""
    w = _unet_mini_weights(8)
    x = rng(9).standard_normal((4, 16, 8))
    y = O.unet_mini_step({}, x, w, 4, 32, 1e-5, 1.0, NAIVE, "none")
    assert y.shape == (1280, 4, 2)
    ref = np.concatenate([lib_unet_mini(x[:, 4 * p:4 * (p + 1)], w) for p in range(4)], axis=1)
    np.testing.assert_allclose(y, ref, rtol=0, atol=1e-9 * np.abs(ref).max())


def test_unet_mini_unchanged_input_displaced_equals_sync():
    """P = 4, an unchanged input after a synchronous step: every stale buffer (the halo rows
    of each conv, the downsamplers' own inputs, the keys and values of both attentions, the
    GroupNorm statistics) equals the fresh one, so the displaced chain gives the synchronous
    chain.  A stage that took its stale rows or keys from another layer's buffer fails."""
    w = _unet_mini_weights(10)
    x = rng(11).standard_normal((4, 16, 16))
    st = {}
    y_sync = O.unet_mini_step(st, x, w, 4, 32, 1e-5, 1.0, SYNC, "none")
    y_disp = O.unet_mini_step(st, x, w, 4, 32, 1e-5, 1.0, DISPLACED, "none")
    np.testing.assert_allclose(y_disp, y_sync, rtol=0, atol=1e-9 * np.abs(y_sync).max())
    # and with a changed input the displaced chain differs from the synchronous one
    x2 = x + 0.3 * rng(12).standard_normal(x.shape)
    st2 = {k: dict(v) if isinstance(v, dict) else v for k, v in st.items()}
    y2_sync = O.unet_mini_step({}, x2, w, 4, 32, 1e-5, 1.0, SYNC, "none")
    y2_disp = O.unet_mini_step(st2, x2, w, 4, 32, 1e-5, 1.0, DISPLACED, "none")
    assert np.abs(y2_disp - y2_sync).max() > 1e-4 * np.abs(y2_sync).max()


def test_p1_unet_mini_displaced_equals_sync():
    """The whole chain with one band: displacement changes nothing."""
    w = _unet_mini_weights(6)
    r = rng(6)
    x0, x1 = r.standard_normal((4, 8, 8)), r.standard_normal((4, 8, 8))
    outs = {}
    for m in (SYNC, DISPLACED):
        st = {}
        O.unet_mini_step(st, x0, w, 1, 32, 1e-5, 1.0, SYNC, "none")
        outs[m] = O.unet_mini_step(st, x1, w, 1, 32, 1e-5, 1.0, m, "none")
    np.testing.assert_allclose(outs[DISPLACED], outs[SYNC], rtol=0, atol=1e-10)
    assert outs[SYNC].shape == (1280, 2, 2)


# ---------------------------------------------------------------- brute force
def brute_conv(a_fresh, a_stale, wt, b, P, mode, stride):
    Cin, H, W = a_fresh.shape
    Co = wt.shape[0]
    Ho, Wo = (H - 1) // stride + 1, (W - 1) // stride + 1
    out = np.zeros((Co, Ho, Wo))
    for co in range(Co):
        for r in range(Ho):
            band = r // (Ho // P)
            for c in range(Wo):
                s = b[co]
                for ci in range(Cin):
                    for kh in range(3):
                        for kw in range(3):
                            rr, cc = stride * r + kh - 1, stride * c + kw - 1
                            if not (0 <= rr < H and 0 <= cc < W):
                                continue
                            if rr // (H // P) == band:
                                v = a_fresh[ci, rr, cc]
                            elif mode == SYNC:
                                v = a_fresh[ci, rr, cc]
                            elif mode == DISPLACED:
                                v = a_stale[ci, rr, cc]
                            else:
                                v = 0.0
                            s += wt[co, ci, kh, kw] * v
                out[co, r, c] = s
    return out


@pytest.mark.parametrize("mode", [SYNC, DISPLACED, NAIVE])
@pytest.mark.parametrize("stride,H,P", [(1, 6, 3), (1, 8, 2), (2, 8, 2), (2, 12, 3)])
def test_conv_matches_brute_force(mode, stride, H, P):
    r = rng(10 + stride + H)
    Cin, Co, W = 3, 2, 5
    af, ast = r.standard_normal((Cin, H, W)), r.standard_normal((Cin, H, W))
    wt, b = r.standard_normal((Co, Cin, 3, 3)), r.standard_normal(Co)
    got = O.conv3x3_halo(af, ast, wt, b, None, P, mode, stride)
    np.testing.assert_allclose(got, brute_conv(af, ast, wt, b, P, mode, stride), rtol=0,
                               atol=1e-12)


def brute_attention(q, kf, vf, ks, vs, P, heads, scale, mode):
    T, C = q.shape
    d = C // heads
    o = np.zeros((T, C))
    for i in range(T):
        band = i // (T // P)
        for h in range(heads):
            logits, vals = [], []
            for j in range(T):
                own = j // (T // P) == band
                if own or mode == SYNC:
                    kk, vv = kf[j], vf[j]
                elif mode == DISPLACED:
                    kk, vv = ks[j], vs[j]
                else:
                    continue
                logits.append(sum(q[i, h * d + e] * kk[h * d + e] for e in range(d)) * scale)
                vals.append(vv[h * d:(h + 1) * d])
            z = sum(math.exp(l) for l in logits)
            for l, vv in zip(logits, vals):
                o[i, h * d:(h + 1) * d] += math.exp(l) / z * vv
    return o


@pytest.mark.parametrize("mode", [SYNC, DISPLACED, NAIVE])
def test_attention_matches_brute_force(mode):
    r = rng(20)
    T, heads, d, P = 6, 2, 3, 3
    q, kf, vf, ks, vs = (r.standard_normal((T, heads * d)) for _ in range(5))
    got = O.attention_stale_kv(q, kf, vf, ks, vs, P, heads, 0.7, mode)
    np.testing.assert_allclose(got, brute_attention(q, kf, vf, ks, vs, P, heads, 0.7, mode),
                               rtol=0, atol=1e-12)


def test_gn_moments_match_brute_force():
    r = rng(21)
    C, H, W, P, G = 6, 4, 3, 2, 3
    x = r.standard_normal((C, H, W))
    f = O.gn_fresh_local(x, P, G)
    for p in range(P):
        for g in range(G):
            vals = [x[c, rr, cc] for c in range(C) for rr in range(H) for cc in range(W)
                    if c // (C // G) == g and rr // (H // P) == p]
            assert len(vals) == (C // G) * (H // P) * W
            assert abs(f[p, g, 0] - sum(vals) / len(vals)) < 1e-14
            assert abs(f[p, g, 1] - sum(v * v for v in vals) / len(vals)) < 1e-14


# ---------------------------------------------------------------- sync / naive
@pytest.mark.parametrize("P", [2, 4])
def test_sync_groupnorm_is_exact_full_image(P):
    r = rng(30 + P)
    C, H, W, G = 8, 8, 5, 4
    x = r.standard_normal((C, H, W)) * 2 + 0.5
    gm, bt = 1 + r.standard_normal(C) * 0.3, r.standard_normal(C) * 0.3
    y, f, used, _ = O.groupnorm_async(x, gm, bt, P, G, 1e-5, 1.0, False, SYNC, None, None)
    ref = F.group_norm(T64(x)[None], G, T64(gm), T64(bt), 1e-5)[0].numpy()
    np.testing.assert_allclose(y, ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("kind", ["gn_conv", "attn"])
def test_naive_equals_independent_crops(kind):
    r = rng(40)
    C, H, W, P, G, heads = 8, 8, 4, 4, 4, 2
    w = rand_gn_conv_weights(r, C, 6) if kind == "gn_conv" else rand_attn_weights(r, C)
    x = r.standard_normal((C, H, W))
    y = O.block_step(kind, {}, x, w, P, G, 1e-5, 1.0, NAIVE, "none", heads=heads)
    hb = H // P
    for p in range(P):
        crop = x[:, p * hb:(p + 1) * hb, :]
        ref = lib_gn_conv(crop, w, G, 1e-5) if kind == "gn_conv" else lib_attn(crop, w, G, 1e-5, heads)
        np.testing.assert_allclose(y[:, p * hb:(p + 1) * hb, :], ref, rtol=0, atol=1e-11)


@pytest.mark.parametrize("kind", ["gn_conv", "resblock", "attn"])
def test_zero_warmup_distinguishable_from_sync(kind):
    """Zero warm-up (step 0 naive) must differ from an exact-sync step 0."""
    r = rng(41)
    C, H, W, P, G, heads = 8, 8, 6, 4, 4, 2
    w = {"gn_conv": lambda: rand_gn_conv_weights(r, C, C), "resblock": lambda: rand_res_weights(r, C, C),
         "attn": lambda: rand_attn_weights(r, C)}[kind]()
    x = r.standard_normal((C, H, W))
    ys = O.block_step(kind, {}, x, w, P, G, 1e-5, 1.0, SYNC, "none", heads=heads)
    yn = O.block_step(kind, {}, x, w, P, G, 1e-5, 1.0, NAIVE, "none", heads=heads)
    rel = np.linalg.norm(yn - ys) / np.linalg.norm(ys)
    assert rel > 1e-3


# ---------------------------------------------------------------- displaced invariants
@pytest.mark.parametrize("kind", ["gn_conv", "resblock", "attn"])
def test_unchanged_input_displaced_equals_sync(kind):
    r = rng(50)
    C, H, W, P, G, heads = 8, 8, 6, 4, 4, 2
    w = {"gn_conv": lambda: rand_gn_conv_weights(r, C, C), "resblock": lambda: rand_res_weights(r, C, C),
         "attn": lambda: rand_attn_weights(r, C)}[kind]()
    x = r.standard_normal((C, H, W))
    yd, trd, _ = run_two_steps(kind, x, x, w, P, G, DISPLACED, heads=heads)
    ys, trs, _ = run_two_steps(kind, x, x, w, P, G, SYNC, heads=heads)
    np.testing.assert_allclose(yd, ys, rtol=0, atol=1e-11)
    for k in trd:
        if k.endswith(".used"):
            np.testing.assert_allclose(trd[k], trs[k], rtol=0, atol=1e-13)


def _zero_band_mean(x, P, G):
    C, H, W = x.shape
    hb, cg = H // P, C // G
    x = x.copy()
    for p in range(P):
        for g in range(G):
            v = x[g * cg:(g + 1) * cg, p * hb:(p + 1) * hb, :]
            v -= v.mean()
    return x


def test_uniform_drift_makes_corrected_stats_exact():
    """Stale bands with equal per-group means, fresh = stale + delta_g: w = 1 is exact."""
    r = rng(60)
    C, H, W, P, G = 8, 8, 5, 4, 4
    stale = _zero_band_mean(r.standard_normal((C, H, W)), P, G)
    delta = np.repeat(r.standard_normal(G) * 0.3, C // G)[:, None, None]
    fresh = stale + delta
    f_stale = O.gn_fresh_local(stale, P, G)
    sg, sl = O.refresh_stats(f_stale)
    f = O.gn_fresh_local(fresh, P, G)
    exact, _ = O.gn_used_stats(f, SYNC, None, None)
    used, nneg = O.gn_used_stats(f, DISPLACED, sg, sl, 1.0)
    assert nneg == 0
    np.testing.assert_allclose(used, exact, rtol=0, atol=1e-13)
    # w = 1/P (own band fresh, other bands stale) is not exact under a uniform drift
    used_p, _ = O.gn_used_stats(f, DISPLACED, sg, sl, 1.0 / P)
    assert np.abs(used_p - exact).max() > 1e-3


def test_displaced_stats_formula_sign_and_weight():
    """One band drifts alone: the correction moves only that band's statistics, by w * drift."""
    r = rng(61)
    C, H, W, P, G = 4, 8, 4, 4, 2
    stale = r.standard_normal((C, H, W))
    fresh = stale.copy()
    fresh[:, 2:4, :] += 0.5          # band 1 drifts by +0.5
    sg, sl = O.refresh_stats(O.gn_fresh_local(stale, P, G))
    f = O.gn_fresh_local(fresh, P, G)
    for w in (1.0, 0.25):
        used, _ = O.gn_used_stats(f, DISPLACED, sg, sl, w)
        for p in range(P):
            expect_mean = sg[:, 0] + (w * 0.5 if p == 1 else 0.0)
            np.testing.assert_allclose(used[p, :, 0], expect_mean, rtol=0, atol=1e-13)


def test_negative_corrected_variance_falls_back_to_fresh():
    r = rng(62)
    C, H, W, P, G = 4, 4, 4, 2, 2
    x = r.standard_normal((C, H, W))
    f = O.gn_fresh_local(x, P, G)
    sg = np.zeros((G, 2))
    sl = f.copy()
    sl[0, 0, 1] += 10.0               # band 0 group 0: corrected E[x^2] goes very negative
    used, nneg = O.gn_used_stats(f, DISPLACED, sg, sl, 1.0)
    assert nneg == 1
    assert abs(used[0, 0, 1] - (f[0, 0, 1] - f[0, 0, 0] ** 2)) < 1e-14
    assert used[1, 1, 1] >= 0


def test_halo_locality():
    """Only the stale rows adjacent to a band edge reach the displaced conv output."""
    r = rng(70)
    C, H, W, P, G = 8, 16, 5, 4, 4
    w = rand_gn_conv_weights(r, C, 6)
    x0, x1 = r.standard_normal((C, H, W)), r.standard_normal((C, H, W))
    st = {}
    O.block_step("gn_conv", st, x0, w, P, G, 1e-5, 1.0, SYNC, "none")
    base_state = {"gn": st["gn"], "a_stale": st["a_stale"].copy()}
    y0 = O.block_step("gn_conv", {"gn": _copy_gn(st["gn"]), "a_stale": st["a_stale"].copy()},
                      x1, w, P, G, 1e-5, 1.0, DISPLACED, "none")
    hb = H // P
    # interior rows (offsets 1 and 2 in a 4-row band) are nobody's halo
    a = base_state["a_stale"].copy()
    for p in range(P):
        a[:, p * hb + 1:p * hb + 3, :] += 5.0
    y1 = O.block_step("gn_conv", {"gn": _copy_gn(st["gn"]), "a_stale": a}, x1, w, P, G, 1e-5,
                      1.0, DISPLACED, "none")
    np.testing.assert_array_equal(y1, y0)
    # the first row of band 1 is band 0's bottom halo: only output row hb-1 changes
    a = base_state["a_stale"].copy()
    a[:, hb, :] += 5.0
    y2 = O.block_step("gn_conv", {"gn": _copy_gn(st["gn"]), "a_stale": a}, x1, w, P, G, 1e-5,
                      1.0, DISPLACED, "none")
    changed = np.abs(y2 - y0).max(axis=(0, 2)) > 0
    assert changed.tolist() == [r_ == hb - 1 for r_ in range(H)]


def _copy_gn(g):
    c = O.GNState()
    c.stale_global, c.stale_local = g.stale_global.copy(), g.stale_local.copy()
    return c


def test_attention_locality():
    """A band's own stale K/V rows are never read; other bands' stale rows are."""
    r = rng(71)
    T, heads, d, P = 16, 2, 4, 4
    q, kf, vf, ks, vs = (r.standard_normal((T, heads * d)) for _ in range(5))
    base = O.attention_stale_kv(q, kf, vf, ks, vs, P, heads, 0.5, DISPLACED)
    tb = T // P
    for p in range(P):
        ks2, vs2 = ks.copy(), vs.copy()
        ks2[p * tb:(p + 1) * tb] += 3.0
        vs2[p * tb:(p + 1) * tb] -= 2.0
        o = O.attention_stale_kv(q, kf, vf, ks2, vs2, P, heads, 0.5, DISPLACED)
        own = slice(p * tb, (p + 1) * tb)
        np.testing.assert_array_equal(o[own], base[own])
        other = np.ones(T, bool)
        other[own] = False
        assert np.abs(o[other] - base[other]).min(axis=1).max() > 0


def test_refresh_makes_fresh_the_next_stale():
    r = rng(72)
    C, H, W, P, G = 8, 8, 4, 4, 4
    w = rand_gn_conv_weights(r, C, 4)
    x = r.standard_normal((C, H, W))
    st, tr = {}, {}
    O.block_step("gn_conv", st, x, w, P, G, 1e-5, 1.0, SYNC, "none", trace=tr)
    np.testing.assert_array_equal(st["a_stale"], tr["a"])
    np.testing.assert_array_equal(st["gn"].stale_local, tr["gn.fresh_local"])
    np.testing.assert_allclose(st["gn"].stale_global, tr["gn.fresh_local"].mean(axis=0),
                               rtol=0, atol=0)


def test_bf16_rounding_matches_library():
    r = rng(80)
    x = np.concatenate([r.standard_normal(100000) * 10, [0.0, -0.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8,
                                                          -(1.0 + 2 ** -8), 65504.0, 1e-40]])
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.to_bf16(x), ref)


@pytest.mark.parametrize("mode", [SYNC, DISPLACED, NAIVE])
@pytest.mark.parametrize("stride", [1, 2])
def test_conv_rows_matches_whole_image(mode, stride):
    """The per-row restatement used at full size agrees with the whole-image one."""
    r = rng(90 + stride)
    Cin, Co, H, W, P = 4, 3, 12, 10, 3
    af, ast = r.standard_normal((Cin, H, W)), r.standard_normal((Cin, H, W))
    wt, b = r.standard_normal((Co, Cin, 3, 3)), r.standard_normal(Co)
    full = O.conv3x3_halo(af, ast, wt, b, None, P, mode, stride)
    rows = list(range(full.shape[1]))
    np.testing.assert_allclose(O.conv3x3_halo_rows(af, ast, wt, b, P, mode, rows, stride), full,
                               rtol=0, atol=1e-12)


# ---------------------------------------------------------------- GroupNorm ablation variants
def _two_step_gn_used(kind, x0, x1, w, P, G, gn_stats, heads=0):
    """GroupNorm statistics of a displaced step after a sync step, per variant."""
    st = {}
    O.block_step(kind, st, x0, w, P, G, 1e-5, 1.0, SYNC, "none", heads=heads)
    tr = {}
    y = O.block_step(kind, st, x1, w, P, G, 1e-5, 1.0, DISPLACED, "none", heads=heads, trace=tr,
                     gn_stats=gn_stats)
    return y, tr


def _library_moments(x, P, G, bands):
    """(mean, var) per (band, group): over the whole image (bands=False) or each band's rows."""
    C, H, W = x.shape
    hb, cg = H // P, C // G
    out = np.empty((P, G, 2))
    for p in range(P):
        for g in range(G):
            v = T64(x[g * cg:(g + 1) * cg, p * hb:(p + 1) * hb, :] if bands else x[g * cg:(g + 1) * cg])
            out[p, g] = (v.mean().item(), v.var(unbiased=False).item())
    return out


def test_gn_variant_sync_uses_exact_whole_image_moments():
    """The synchronous variant normalises a displaced step with this step's exact moments: its
    GroupNorm output is the library's full-image GroupNorm, while the halos stay stale."""
    r = rng(70)
    C, H, W, P, G = 8, 8, 5, 4, 4
    w = rand_gn_conv_weights(r, C, C)
    x0 = r.standard_normal((C, H, W))
    x1 = x0 + 0.3 * r.standard_normal((C, H, W))
    _, tr = _two_step_gn_used("gn_conv", x0, x1, w, P, G, O.GN_STATS_SYNC)
    np.testing.assert_allclose(tr["gn.used"], _library_moments(x1, P, G, bands=False), rtol=0, atol=1e-12)
    a = F.silu(F.group_norm(T64(x1)[None], G, T64(w["gn_gamma"]), T64(w["gn_beta"]), 1e-5))[0].numpy()
    np.testing.assert_allclose(tr["a"], a, rtol=0, atol=1e-12)


def test_gn_variant_local_uses_each_bands_own_moments():
    """The band-local variant normalises each band with its own rows' moments (the library's
    GroupNorm of the band crop)."""
    r = rng(71)
    C, H, W, P, G = 8, 8, 5, 4, 4
    w = rand_gn_conv_weights(r, C, C)
    x0 = r.standard_normal((C, H, W))
    x1 = x0 + 0.3 * r.standard_normal((C, H, W))
    _, tr = _two_step_gn_used("gn_conv", x0, x1, w, P, G, O.GN_STATS_LOCAL)
    np.testing.assert_allclose(tr["gn.used"], _library_moments(x1, P, G, bands=True), rtol=0, atol=1e-12)
    hb = H // P
    for p in range(P):
        crop = x1[:, p * hb:(p + 1) * hb, :]
        a = F.silu(F.group_norm(T64(crop)[None], G, T64(w["gn_gamma"]), T64(w["gn_beta"]), 1e-5))[0].numpy()
        np.testing.assert_allclose(tr["a"][:, p * hb:(p + 1) * hb, :], a, rtol=0, atol=1e-12)


def test_gn_variant_stale_uses_previous_steps_moments():
    """The stale-only variant normalises with the previous step's whole-image moments, whatever
    this step's input is."""
    r = rng(72)
    C, H, W, P, G = 8, 8, 5, 4, 4
    w = rand_res_weights(r, C, C)
    x0 = r.standard_normal((C, H, W))
    x1 = 1.5 * x0 + 0.7 + 0.3 * r.standard_normal((C, H, W))
    _, tr = _two_step_gn_used("resblock", x0, x1, w, P, G, O.GN_STATS_STALE)
    np.testing.assert_allclose(tr["gn1.used"], _library_moments(x0, P, G, bands=False), rtol=0, atol=1e-12)


@pytest.mark.parametrize("variant", [O.GN_STATS_CORRECTED, O.GN_STATS_LOCAL, O.GN_STATS_STALE,
                                     O.GN_STATS_SYNC])
def test_gn_variants_agree_when_nothing_changes_and_p1(variant):
    """With one band and an unchanged input every variant is the library's block; the variants
    differ from each other once the input drifts."""
    r = rng(73)
    C, H, W, G = 8, 6, 5, 4
    w = rand_res_weights(r, C, C)
    x = r.standard_normal((C, H, W))
    y, _ = _two_step_gn_used("resblock", x, x, w, 1, G, variant)
    np.testing.assert_allclose(y, lib_resblock(x, w, G, 1e-5), rtol=0, atol=1e-11)


def test_gn_variants_differ_under_drift():
    r = rng(74)
    C, H, W, P, G = 8, 8, 5, 4, 4
    w = rand_res_weights(r, C, C)
    x0 = r.standard_normal((C, H, W))
    x1 = x0 + 0.4 * r.standard_normal((C, H, W)) + 0.2
    ys = [_two_step_gn_used("resblock", x0, x1, w, P, G, v)[0]
          for v in (O.GN_STATS_CORRECTED, O.GN_STATS_LOCAL, O.GN_STATS_STALE, O.GN_STATS_SYNC)]
    for i in range(4):
        for j in range(i + 1, 4):
            assert np.linalg.norm(ys[i] - ys[j]) / np.linalg.norm(ys[j]) > 1e-4, (i, j)
    # sync and naive-step modes ignore the variant
    st = {}
    a = O.block_step("resblock", st, x0, w, P, G, 1e-5, 1.0, NAIVE, "none", gn_stats=O.GN_STATS_STALE)
    b = O.block_step("resblock", {}, x0, w, P, G, 1e-5, 1.0, NAIVE, "none")
    np.testing.assert_array_equal(a, b)


# ---------------------------------------------------------------- cross-attention
@pytest.mark.parametrize("Tq,Tk,heads", [(6, 5, 2), (8, 77, 3), (16, 1, 1)])
def test_cross_attention_equals_library_and_brute_force(Tq, Tk, heads):
    r = rng(80 + Tk)
    d = 4
    q, k, v = (r.standard_normal((T, heads * d)) for T in (Tq, Tk, Tk))
    o = O.attention_cross(q, k, v, heads, 0.37)
    sh = lambda z, T: T64(z).reshape(T, heads, d).permute(1, 0, 2)
    ref = F.scaled_dot_product_attention(sh(q, Tq), sh(k, Tk), sh(v, Tk), scale=0.37)
    np.testing.assert_allclose(o, ref.permute(1, 0, 2).reshape(Tq, heads * d).numpy(), rtol=0, atol=1e-12)
    # brute force: one query, one head at a time
    for t in range(Tq):
        for h in range(heads):
            w = [math.exp(0.37 * sum(q[t, h * d + i] * k[j, h * d + i] for i in range(d))) for j in range(Tk)]
            z = sum(w)
            for i in range(d):
                assert abs(o[t, h * d + i] - sum(w[j] * v[j, h * d + i] for j in range(Tk)) / z) < 1e-10


# ---------------------------------------------------------------- SDXL-shaped transformer block
def rand_transformer_weights(r, C, Cctx, heads, mult=2, depth=1):
    s = lambda *shape: r.standard_normal(shape) * (1.0 / math.sqrt(shape[-1]))
    w = {"gn_gamma": 1 + 0.3 * r.standard_normal(C), "gn_beta": 0.3 * r.standard_normal(C),
         "proj_in_w": s(C, C), "proj_in_b": 0.3 * r.standard_normal(C),
         "proj_out_w": s(C, C), "proj_out_b": 0.3 * r.standard_normal(C)}
    for layer in range(depth):
        p = "" if layer == 0 else f"l{layer}."
        for i in (1, 2, 3):
            w[f"{p}ln{i}_g"], w[f"{p}ln{i}_b"] = 1 + 0.3 * r.standard_normal(C), 0.3 * r.standard_normal(C)
        for n in ("wq", "wk", "wv", "wo"):
            w[p + n] = s(C, C)
        for n in ("bq", "bk", "bv", "bo", "co_b"):
            w[p + n] = 0.3 * r.standard_normal(C)
        w[p + "cq_w"], w[p + "co_w"] = s(C, C), s(C, C)
        w[p + "ck_w"], w[p + "cv_w"] = s(C, Cctx), s(C, Cctx)
        w[p + "ff1_w"], w[p + "ff1_b"] = s(2 * mult * C, C), 0.3 * r.standard_normal(2 * mult * C)
        w[p + "ff2_w"], w[p + "ff2_b"] = s(C, mult * C), 0.3 * r.standard_normal(C)
    return w


def lib_transformer(x, ctx, w, G, eps, heads, depth=1, prefix=""):
    """The same block composed from library operators, on the whole image: ``depth`` basic
    layers (the first named plainly, layer l >= 1 with an "l<l>." prefix)."""
    C, H, W = x.shape
    d = C // heads
    sh = lambda z: z.reshape(z.shape[0], heads, d).permute(1, 0, 2)
    un = lambda z: z.permute(1, 0, 2).reshape(-1, C)
    g0 = lambda n: T64(w[prefix + n])
    a = F.group_norm(T64(x)[None], G, g0("gn_gamma"), g0("gn_beta"), eps)[0].reshape(C, H * W).T
    h = F.linear(a, g0("proj_in_w"), g0("proj_in_b"))
    c = T64(ctx)
    for layer in range(depth):
        g = lambda n: T64(w[prefix + (n if layer == 0 else f"l{layer}.{n}")])
        t = F.layer_norm(h, (C,), g("ln1_g"), g("ln1_b"), 1e-5)
        o = F.scaled_dot_product_attention(sh(F.linear(t, g("wq"), g("bq"))), sh(F.linear(t, g("wk"), g("bk"))),
                                           sh(F.linear(t, g("wv"), g("bv"))))
        h = h + F.linear(un(o), g("wo"), g("bo"))
        t = F.layer_norm(h, (C,), g("ln2_g"), g("ln2_b"), 1e-5)
        o = F.scaled_dot_product_attention(sh(F.linear(t, g("cq_w"))), sh(F.linear(c, g("ck_w"))),
                                           sh(F.linear(c, g("cv_w"))))
        h = h + F.linear(un(o), g("co_w"), g("co_b"))
        t = F.layer_norm(h, (C,), g("ln3_g"), g("ln3_b"), 1e-5)
        a2, gate = F.linear(t, g("ff1_w"), g("ff1_b")).chunk(2, dim=-1)
        h = h + F.linear(a2 * F.gelu(gate), g("ff2_w"), g("ff2_b"))
    out = F.linear(h, g0("proj_out_w"), g0("proj_out_b")) + T64(x).reshape(C, H * W).T
    return out.T.reshape(C, H, W).numpy()


def test_layer_norm_gelu_geglu_equal_library():
    r = rng(90)
    x = r.standard_normal((7, 12)) * 2 + 0.3
    gm, bt = 1 + 0.3 * r.standard_normal(12), 0.3 * r.standard_normal(12)
    np.testing.assert_allclose(O.layer_norm(x, gm, bt, 1e-5),
                               F.layer_norm(T64(x), (12,), T64(gm), T64(bt), 1e-5).numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(O.gelu(x), F.gelu(T64(x)).numpy(), rtol=0, atol=1e-14)
    w1, b1 = r.standard_normal((16, 12)), r.standard_normal(16)
    w2, b2 = r.standard_normal((12, 8)), r.standard_normal(12)
    a, g = F.linear(T64(x), T64(w1), T64(b1)).chunk(2, dim=-1)
    ref = F.linear(a * F.gelu(g), T64(w2), T64(b2)).numpy()
    np.testing.assert_allclose(O.geglu_ff(x, w1, b1, w2, b2), ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("mode", [SYNC, DISPLACED, NAIVE])
def test_p1_transformer_equals_library(mode):
    r = rng(91)
    C, H, W, G, heads, Cctx, Tk = 8, 4, 6, 4, 2, 6, 5
    w = rand_transformer_weights(r, C, Cctx, heads)
    x, ctx = r.standard_normal((C, H, W)), r.standard_normal((Tk, Cctx))
    st = {}
    O.transformer_step(st, x, ctx, w, 1, G, 1e-5, 1.0, heads, SYNC, "none")
    y = O.transformer_step(st, x, ctx, w, 1, G, 1e-5, 1.0, heads, mode, "none")
    np.testing.assert_allclose(y, lib_transformer(x, ctx, w, G, 1e-5, heads), rtol=0, atol=1e-11)


@pytest.mark.parametrize("mode", [SYNC, DISPLACED, NAIVE])
def test_p1_transformer_depth3_equals_library(mode):
    """Three basic layers at one band equal the library's composition of three layers, and
    neither one nor two layers of the same weights give that result (so every layer runs,
    each with its own weights)."""
    r = rng(93)
    C, H, W, G, heads, Cctx, Tk = 8, 4, 6, 4, 2, 6, 5
    w = rand_transformer_weights(r, C, Cctx, heads, depth=3)
    x, ctx = r.standard_normal((C, H, W)), r.standard_normal((Tk, Cctx))
    st = {}
    O.transformer_step(st, x, ctx, w, 1, G, 1e-5, 1.0, heads, SYNC, "none", depth=3)
    y = O.transformer_step(st, x, ctx, w, 1, G, 1e-5, 1.0, heads, mode, "none", depth=3)
    np.testing.assert_allclose(y, lib_transformer(x, ctx, w, G, 1e-5, heads, depth=3), rtol=0, atol=1e-11)
    for fewer in (1, 2):
        assert np.abs(y - lib_transformer(x, ctx, w, G, 1e-5, heads, depth=fewer)).max() > 1e-3


def test_transformer_depth2_keeps_each_layers_stale_keys():
    """Two layers over four bands: with an unchanged input a displaced step equals a sync step
    (each layer's stale keys and values are its own, from the step before), the state holds
    one stale pair per layer, and band locality holds through both layers."""
    r = rng(96)
    C, H, W, P, G, heads, Cctx, Tk = 8, 8, 4, 4, 4, 2, 6, 5
    w = rand_transformer_weights(r, C, Cctx, heads, depth=2)
    x0, ctx = r.standard_normal((C, H, W)), r.standard_normal((Tk, Cctx))
    st = {}
    ys = O.transformer_step(st, x0, ctx, w, P, G, 1e-5, 1.0, heads, SYNC, "none", depth=2)
    assert {"k_stale", "v_stale", "l1.k_stale", "l1.v_stale"} <= set(st)
    assert not np.allclose(st["k_stale"], st["l1.k_stale"])
    yd = O.transformer_step(st, x0, ctx, w, P, G, 1e-5, 1.0, heads, DISPLACED, "none", depth=2)
    np.testing.assert_allclose(yd, ys, rtol=0, atol=1e-11)
    # a displaced step that took layer 0's stale pair for layer 1 would not equal sync
    bad = dict(st)
    bad["l1.k_stale"], bad["l1.v_stale"] = st["k_stale"], st["v_stale"]
    yb = O.transformer_step(bad, x0, ctx, w, P, G, 1e-5, 1.0, heads, DISPLACED, "none", depth=2)
    assert np.abs(yb - ys).max() > 1e-3
    x1 = x0 + 0.3 * r.standard_normal(x0.shape)
    hb, q = H // P, 1
    x1b = x1.copy()
    x1b[:, q * hb:(q + 1) * hb, :] += r.standard_normal((C, hb, W))
    outs = []
    for xin in (x1, x1b):
        s2 = {}
        O.transformer_step(s2, x0, ctx, w, P, G, 1e-5, 1.0, heads, SYNC, "none", depth=2)
        outs.append(O.transformer_step(s2, xin, ctx, w, P, G, 1e-5, 1.0, heads, DISPLACED, "none", depth=2))
    for p in range(P):
        rows = slice(p * hb, (p + 1) * hb)
        assert np.array_equal(outs[0][:, rows, :], outs[1][:, rows, :]) == (p != q), p


def test_transformer_displaced_band_locality():
    """A displaced step needs nothing of the current step from other bands: changing one
    band's input leaves every other band's output bit for bit the same (their GroupNorm
    statistics take only their own fresh moments, their self-attention the other bands'
    stale keys and values, and LayerNorm, cross-attention and the feed-forward act per
    token), while in a sync step the change reaches every band."""
    r = rng(97)
    C, H, W, P, G, heads, Cctx, Tk = 8, 8, 4, 4, 4, 2, 6, 5
    w = rand_transformer_weights(r, C, Cctx, heads)
    x0, ctx = r.standard_normal((C, H, W)), r.standard_normal((Tk, Cctx))
    x1 = x0 + 0.3 * r.standard_normal(x0.shape)
    hb, q = H // P, 2
    x1b = x1.copy()
    x1b[:, q * hb:(q + 1) * hb, :] += r.standard_normal((C, hb, W))
    for mode in (DISPLACED, SYNC):
        ys = []
        for xin in (x1, x1b):
            st = {}
            O.transformer_step(st, x0, ctx, w, P, G, 1e-5, 1.0, heads, SYNC, "none")
            ys.append(O.transformer_step(st, xin, ctx, w, P, G, 1e-5, 1.0, heads, mode, "none"))
        for p in range(P):
            rows = slice(p * hb, (p + 1) * hb)
            same = np.array_equal(ys[0][:, rows, :], ys[1][:, rows, :])
            assert same == (mode == DISPLACED and p != q), (mode, p)


def test_transformer_displaced_and_naive_invariants():
    """Unchanged input: displaced equals sync.  Naive: each band is an independent image."""
    r = rng(92)
    C, H, W, P, G, heads, Cctx, Tk = 8, 8, 4, 4, 4, 2, 6, 5
    w = rand_transformer_weights(r, C, Cctx, heads)
    x, ctx = r.standard_normal((C, H, W)), r.standard_normal((Tk, Cctx))
    outs = {}
    for m in (SYNC, DISPLACED):
        st = {}
        O.transformer_step(st, x, ctx, w, P, G, 1e-5, 1.0, heads, SYNC, "none")
        outs[m] = O.transformer_step(st, x, ctx, w, P, G, 1e-5, 1.0, heads, m, "none")
    np.testing.assert_allclose(outs[DISPLACED], outs[SYNC], rtol=0, atol=1e-11)
    y = O.transformer_step({}, x, ctx, w, P, G, 1e-5, 1.0, heads, NAIVE, "none")
    hb = H // P
    for p in range(P):
        crop = x[:, p * hb:(p + 1) * hb, :]
        np.testing.assert_allclose(y[:, p * hb:(p + 1) * hb, :], lib_transformer(crop, ctx, w, G, 1e-5, heads),
                                   rtol=0, atol=1e-11)
    # drift: displaced differs from sync, and from naive by more
    x1 = x + 0.3 * r.standard_normal(x.shape)
    res = {}
    for m in (SYNC, DISPLACED, NAIVE):
        st = {}
        O.transformer_step(st, x, ctx, w, P, G, 1e-5, 1.0, heads, SYNC, "none")
        res[m] = O.transformer_step(st, x1, ctx, w, P, G, 1e-5, 1.0, heads, m, "none")
    err = lambda m: np.linalg.norm(res[m] - res[SYNC]) / np.linalg.norm(res[SYNC])
    assert 0 < err(DISPLACED) < err(NAIVE)


def test_time_embedding_term_equals_library():
    """temb_w silu(temb) + temb_b is the library's linear of the library's SiLU; without
    temb_b it is the bare product, and a zero embedding leaves only temb_b (silu(0) = 0)."""
    r = rng(94)
    Ct, Co = 37, 11
    tw, tb, t = r.standard_normal((Co, Ct)), r.standard_normal(Co), 3 * r.standard_normal(Ct)
    ref = F.linear(F.silu(T64(t)), T64(tw), T64(tb)).numpy()
    np.testing.assert_allclose(O.time_embedding_term(t, tw, tb), ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(O.time_embedding_term(t, tw, None), ref - tb, rtol=0, atol=1e-12)
    np.testing.assert_array_equal(O.time_embedding_term(np.zeros(Ct), tw, tb), tb)


@pytest.mark.parametrize("mode", [SYNC, DISPLACED])
def test_p1_resblock_time_embedding_equals_library(mode):
    """A time embedding adds temb_w silu(temb) + temb_b to every pixel of conv1's output."""
    r = rng(93)
    C, H, W, G, Ct = 8, 5, 6, 4, 10
    w = rand_res_weights(r, C, C)
    w["temb_w"], w["temb_b"] = r.standard_normal((C, Ct)) / math.sqrt(Ct), 0.3 * r.standard_normal(C)
    x, temb = r.standard_normal((C, H, W)), r.standard_normal(Ct)
    st = {}
    O.resblock_step(st, x, w, 1, G, 1e-5, 1.0, SYNC, "none", temb=temb)
    y = O.resblock_step(st, x, w, 1, G, 1e-5, 1.0, mode, "none", temb=temb)
    g = lambda n: T64(w[n])
    t = F.silu(F.group_norm(T64(x)[None], G, g("gn1_gamma"), g("gn1_beta"), 1e-5))
    h = F.conv2d(t, g("conv1_w"), g("conv1_b"), padding=1)
    h = h + F.linear(F.silu(T64(temb)), g("temb_w"), g("temb_b"))[None, :, None, None]
    t = F.silu(F.group_norm(h, G, g("gn2_gamma"), g("gn2_beta"), 1e-5))
    ref = (F.conv2d(t, g("conv2_w"), g("conv2_b"), padding=1) + T64(x)[None])[0].numpy()
    np.testing.assert_allclose(y, ref, rtol=0, atol=1e-11)
    # without the embedding the block is the plain ResBlock
    np.testing.assert_allclose(O.resblock_step({}, x, w, 1, G, 1e-5, 1.0, SYNC, "none"),
                               lib_resblock(x, w, G, 1e-5), rtol=0, atol=1e-11)


def test_ddim_step_moves_exact_noise_to_the_previous_level():
    """With the exact noise of x_t = sqrt(abar_t) x0 + sqrt(1 - abar_t) e, the deterministic
    DDIM step lands exactly on sqrt(abar_prev) x0 + sqrt(1 - abar_prev) e: the defining
    property of the update (the same x0 and the same noise, one level less noisy)."""
    r = rng(95)
    x0, e = r.standard_normal((3, 5, 7)), r.standard_normal((3, 5, 7))
    for abar_t, abar_prev in [(0.0047, 0.0059), (0.3, 0.5), (0.98, 1.0)]:
        xt = math.sqrt(abar_t) * x0 + math.sqrt(1 - abar_t) * e
        want = math.sqrt(abar_prev) * x0 + math.sqrt(1 - abar_prev) * e
        np.testing.assert_allclose(O.ddim_step(xt, e, abar_t, abar_prev), want, rtol=0, atol=1e-12)
    # abar_prev = 1: the step returns the predicted clean sample itself
    np.testing.assert_allclose(O.ddim_step(math.sqrt(0.4) * x0 + math.sqrt(0.6) * e, e, 0.4, 1.0), x0,
                               rtol=0, atol=1e-12)


def test_ddim_step_identity_and_composition():
    """No change of level leaves x unchanged for any noise estimate; with a fixed noise
    estimate, two steps t -> s -> r equal the one step t -> r (the update is a change of
    noise level along one line); the step is affine in (x, eps)."""
    r = rng(96)
    x, e = r.standard_normal(40), r.standard_normal(40)
    np.testing.assert_allclose(O.ddim_step(x, e, 0.37, 0.37), x, rtol=0, atol=1e-13)
    two = O.ddim_step(O.ddim_step(x, e, 0.1, 0.25), e, 0.25, 0.7)
    np.testing.assert_allclose(two, O.ddim_step(x, e, 0.1, 0.7), rtol=0, atol=1e-12)
    x2, e2 = r.standard_normal(40), r.standard_normal(40)
    lin = O.ddim_step(2 * x - x2, 2 * e - e2, 0.2, 0.3)
    np.testing.assert_allclose(lin, 2 * O.ddim_step(x, e, 0.2, 0.3) - O.ddim_step(x2, e2, 0.2, 0.3),
                               rtol=0, atol=1e-12)


# ---------------------------------------------------------------- DPM-Solver++ (2M)
def test_dpm_solver_first_order_is_ddim():
    """The first-order step of DPM-Solver++ is the deterministic DDIM step: with
    exp(-h) = sigma_t alpha_s / (alpha_t sigma_s) the update becomes alpha_t x0 + sigma_t eps."""
    r = rng(120)
    x, e = r.standard_normal((3, 6, 5)), r.standard_normal((3, 6, 5))
    for abar_s, abar_t in [(0.0047, 0.0066), (0.3, 0.45), (0.9, 0.97), (0.6, 1.0)]:
        got, x0 = O.dpm_solver_2m_step(x, e, None, 0.0, abar_s, abar_t)
        np.testing.assert_allclose(got, O.ddim_step(x, e, abar_s, abar_t), rtol=0, atol=1e-11)
        np.testing.assert_allclose(x0, (x - math.sqrt(1 - abar_s) * e) / math.sqrt(abar_s), rtol=0,
                                   atol=1e-12)


def test_dpm_solver_second_order_with_constant_prediction_is_first_order():
    """D = x0 + (x0 - x0_prev) / (2r): an unchanged data prediction leaves the first-order step."""
    r = rng(121)
    x, e = r.standard_normal(30), r.standard_normal(30)
    _, x0 = O.dpm_solver_2m_step(x, e, None, 0.0, 0.2, 0.3)
    got, _ = O.dpm_solver_2m_step(x, e, x0, 0.12, 0.2, 0.3)
    np.testing.assert_allclose(got, O.dpm_solver_2m_step(x, e, None, 0.0, 0.2, 0.3)[0], rtol=0, atol=1e-12)
    # and a changed one moves it by alpha_t (1 - e^{-h}) (x0 - x0_prev) / (2r), the sign included
    got2, _ = O.dpm_solver_2m_step(x, e, x0 - 1.0, 0.12, 0.2, 0.3)
    lam = lambda ab: math.log(math.sqrt(ab) / math.sqrt(1 - ab))
    h, hp = lam(0.3) - lam(0.2), lam(0.2) - lam(0.12)
    shift = math.sqrt(0.3) * (1 - math.exp(-h)) * 1.0 / (2 * hp / h)
    np.testing.assert_allclose(got2 - got, shift, rtol=1e-12, atol=1e-12)


def _ode_errors(order, n_steps):
    """Integrates the data-prediction ODE x' = x + ... along lambda from -2 to 1, whose exact
    solution for the data prediction x0(lambda) = cos(lambda) is known in closed form:
    x(l) = (sigma_l / sigma_a) x(a) + sigma_l * integral_a^l e^u cos(u) du.  The solver sees
    eps = (x - alpha x0(lambda)) / sigma, i.e. an exact model.  Returns the final error."""
    lam = np.linspace(-2.0, 1.0, n_steps + 1)
    ab = lambda l: 1.0 / (1.0 + math.exp(-2.0 * l))          # alpha^2 with lambda = log(alpha/sigma)
    sig = lambda l: math.sqrt(1.0 - ab(l))
    prim = lambda u: math.exp(u) * (math.cos(u) + math.sin(u)) / 2.0
    exact = lambda l, x_a, a: sig(l) / sig(a) * x_a + sig(l) * (prim(l) - prim(a))
    x_a = 0.7
    x, x0_prev, ab_prev = x_a, None, 0.0
    for i in range(n_steps):
        l_s, l_t = lam[i], lam[i + 1]
        e = (x - math.sqrt(ab(l_s)) * math.cos(l_s)) / sig(l_s)
        use_prev = x0_prev if order == 2 else None
        x, x0_prev = O.dpm_solver_2m_step(np.array(x), np.array(e), use_prev, ab_prev if order == 2 else 0.0,
                                          ab(l_s), ab(l_t))
        x = float(x)
        ab_prev = ab(l_s)
    return abs(x - exact(lam[-1], x_a, lam[0]))


def test_dpm_solver_convergence_order():
    """Halving the step halves the first-order error and quarters the second-order one: the
    multistep correction has the published coefficient and sign."""
    e1 = [_ode_errors(1, n) for n in (20, 40, 80)]
    e2 = [_ode_errors(2, n) for n in (20, 40, 80)]
    for a, b in zip(e1, e1[1:]):
        assert 1.8 < a / b < 2.2, e1
    for a, b in zip(e2, e2[1:]):
        assert 3.5 < a / b < 4.5, e2
    assert e2[-1] < e1[-1] / 5      # and more accurate at the same step count


# ---------------------------------------------------------------- SDXL-shaped U-Net step
UNET_TINY = dict(Cl=4, base=8, depths=(0, 1, 2), head_dim=4, G=4, Tk=3, Cc=8, Ct=6)


def _sdxl_unet_case(seed, H, W, P, depths=UNET_TINY["depths"]):
    """Weights drawn from the workload's own names and shapes (random affine parameters and
    biases, so that no term hides behind a zero), a text context and a time embedding."""
    from displaced_patch_parallelism_b200 import synth
    t = UNET_TINY
    wl = synth.Workload(name="tiny_unet", kind="unet_sdxl", C=t["Cl"], H=H, W=W, P=P, G=t["G"],
                        base=t["base"], depths=depths, ctx_len=t["Tk"], ctx_dim=t["Cc"],
                        temb_dim=t["Ct"])
    r = rng(seed)
    mats, aff = synth.sdxl_unet_specs(wl)
    w = {n: r.standard_normal(shape) * std for n, shape, std in mats}
    for n, c, kind in aff:
        w[n] = (1 + 0.2 * r.standard_normal(c)) if kind == "gamma" else 0.2 * r.standard_normal(c)
    return w, r.standard_normal((t["Tk"], t["Cc"])), r.standard_normal(t["Ct"])


def lib_sdxl_unet(x, ctx, temb, w, depths=UNET_TINY["depths"], skip_first=False):
    """The SDXL-shaped U-Net composed from library operators on the whole image: conv2d
    (stride 1 and 2, padding 1), nearest interpolation, channel concatenation, the library
    ResBlock with its time-embedding term and the library transformer block.
    ``skip_first`` concatenates [skip, h] instead of [h, skip] (a plausible slip)."""
    t = UNET_TINY
    G, eps, hd = t["G"], 1e-5, t["head_dim"]
    conv = lambda z, n, s: F.conv2d(T64(z)[None], T64(w[n + "_w"]), T64(w[n + "_b"]), stride=s,
                                    padding=1)[0].numpy()
    res = lambda z, pre: lib_resblock(z, w, G, eps, pre, temb)
    tf = lambda z, pre, dp: lib_transformer(z, ctx, w, G, eps, z.shape[0] // hd, dp, pre)
    h = conv(x, "conv_in", 1)
    skips = [h]
    for lvl in range(3):
        for i in range(2):
            h = res(h, f"d{lvl}.r{i}.")
            if depths[lvl]:
                h = tf(h, f"d{lvl}.t{i}.", depths[lvl])
            skips.append(h)
        if lvl < 2:
            h = conv(h, f"d{lvl}.down", 2)
            skips.append(h)
    h = res(h, "mid.r0.")
    if depths[2]:
        h = tf(h, "mid.t.", depths[2])
    h = res(h, "mid.r1.")
    for lvl in (2, 1, 0):
        for i in range(3):
            sk = skips.pop()
            h = res(np.concatenate([sk, h] if skip_first else [h, sk]), f"u{lvl}.r{i}.")
            if depths[lvl]:
                h = tf(h, f"u{lvl}.t{i}.", depths[lvl])
        if lvl > 0:
            up = F.interpolate(T64(h)[None], scale_factor=2, mode="nearest")[0].numpy()
            h = conv(up, f"u{lvl}.up", 1)
    a = F.silu(F.group_norm(T64(h)[None], G, T64(w["out.gn_gamma"]), T64(w["out.gn_beta"]), eps))
    return F.conv2d(a, T64(w["out.conv_w"]), T64(w["out.conv_b"]), padding=1)[0].numpy()


def _unet(st, x, ctx, temb, w, P, mode, depths=UNET_TINY["depths"]):
    t = UNET_TINY
    return O.sdxl_unet_step(st, x, ctx, temb, w, P, t["G"], 1e-5, 1.0, mode, "none", base=t["base"],
                            depths=depths, head_dim=t["head_dim"])


def test_upsample_and_concat_are_the_library_ops():
    r = rng(120)
    x, y = r.standard_normal((3, 4, 5)), r.standard_normal((2, 4, 5))
    np.testing.assert_array_equal(O.upsample_nearest2x(x),
                                  F.interpolate(T64(x)[None], scale_factor=2, mode="nearest")[0].numpy())
    np.testing.assert_array_equal(O.concat_channels(x, y), torch.cat([T64(x), T64(y)]).numpy())


@pytest.mark.parametrize("mode", [SYNC, DISPLACED, NAIVE])
def test_p1_sdxl_unet_equals_library(mode):
    """One band: the whole U-Net step is the ordinary network composed from library operators
    (after a sync step, so a displaced step has stale state).  Swapping the skip order, or
    the transformer depths of the two deeper levels, changes the result."""
    w, ctx, temb = _sdxl_unet_case(121, 8, 8, 1)
    x = rng(122).standard_normal((UNET_TINY["Cl"], 8, 8))
    st = {}
    _unet(st, x, ctx, temb, w, 1, SYNC)
    y = _unet(st, x, ctx, temb, w, 1, mode)
    ref = lib_sdxl_unet(x, ctx, temb, w)
    np.testing.assert_allclose(y, ref, rtol=0, atol=1e-10 * np.abs(ref).max())
    assert np.abs(y - lib_sdxl_unet(x, ctx, temb, w, skip_first=True)).max() > 1e-3 * np.abs(ref).max()
    w2, _, _ = _sdxl_unet_case(121, 8, 8, 1, depths=(0, 2, 2))
    assert np.abs(_unet({}, x, ctx, temb, w2, 1, SYNC, depths=(0, 2, 2)) - ref).max() > 1e-3 * np.abs(ref).max()


def test_sdxl_unet_naive_equals_independent_crops():
    """Naive patches: every band is an independent image through the whole network."""
    P, H, W = 2, 16, 8
    w, ctx, temb = _sdxl_unet_case(123, H, W, P)
    x = rng(124).standard_normal((UNET_TINY["Cl"], H, W))
    y = _unet({}, x, ctx, temb, w, P, NAIVE)
    hb = H // P
    for p in range(P):
        ref = lib_sdxl_unet(x[:, p * hb:(p + 1) * hb], ctx, temb, w)
        np.testing.assert_allclose(y[:, p * hb:(p + 1) * hb], ref, rtol=0, atol=1e-10 * np.abs(ref).max())


def test_sdxl_unet_unchanged_input_displaced_equals_sync():
    """With the same input as the step before, every stale buffer (conv inputs, keys and
    values, GroupNorm statistics) holds what a sync step computes, so displaced equals sync."""
    P, H, W = 4, 16, 8
    w, ctx, temb = _sdxl_unet_case(125, H, W, P)
    x = rng(126).standard_normal((UNET_TINY["Cl"], H, W))
    st = {}
    ys = _unet(st, x, ctx, temb, w, P, SYNC)
    yd = _unet(st, x, ctx, temb, w, P, DISPLACED)
    np.testing.assert_allclose(yd, ys, rtol=0, atol=1e-10 * np.abs(ys).max())


def test_sdxl_unet_displaced_band_locality():
    """A displaced step takes nothing of the current step from other bands, through all
    levels, skips and up/down sampling: changing band q's input leaves every other band's
    output bit for bit the same; a sync step carries the change to every band; and a
    displaced step after drift lies closer to sync than naive does."""
    P, H, W, q = 4, 16, 8, 2
    w, ctx, temb = _sdxl_unet_case(127, H, W, P)
    r = rng(128)
    x0 = r.standard_normal((UNET_TINY["Cl"], H, W))
    x1 = x0 + 0.2 * r.standard_normal(x0.shape)
    hb = H // P
    x1b = x1.copy()
    x1b[:, q * hb:(q + 1) * hb] += r.standard_normal((UNET_TINY["Cl"], hb, W))
    res = {}
    for mode in (SYNC, DISPLACED, NAIVE):
        outs = []
        for xin in (x1, x1b):
            st = {}
            _unet(st, x0, ctx, temb, w, P, SYNC)
            outs.append(_unet(st, xin, ctx, temb, w, P, mode))
        res[mode] = outs[0]
        if mode == NAIVE:
            continue
        for p in range(P):
            rows = slice(p * hb, (p + 1) * hb)
            assert np.array_equal(outs[0][:, rows], outs[1][:, rows]) == (mode == DISPLACED and p != q), (mode, p)
    err = lambda m: np.linalg.norm(res[m] - res[SYNC]) / np.linalg.norm(res[SYNC])
    assert 0 < err(DISPLACED) < err(NAIVE)
