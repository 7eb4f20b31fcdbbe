"""Parity of every C-ABI kernel call against the CPU oracle, on seeded inputs.

Sizes span several tiles and ragged tails; every mode (sync, displaced,
naive) is covered.  Bar: see tests/helpers.py.
"""
import math

import numpy as np
import pytest
import torch

from displaced_patch_parallelism_b200 import binding as B
from oracle import dp_oracle as O
from tests.helpers import (F32_ATOL, F32_RL2, BF16_HALF_ULP, STATS_ATOL, check, conv_w_dev, dev_f32, dev_img,
                           dev_mat, host, host_img, rounded)

pytestmark = pytest.mark.gpu
MODES = [B.SYNC, B.DISPLACED, B.NAIVE]


def rng(seed):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------- GroupNorm
GN_CASES = [
    # C, H, W, P, G, dtype, silu
    (64, 32, 32, 2, 32, "fp32", True),
    (320, 32, 20, 4, 32, "bf16", True),
    (640, 16, 16, 4, 32, "bf16", False),
    (96, 24, 9, 8, 32, "bf16", True),
    (1280, 8, 8, 2, 32, "bf16", True),
    (320, 256, 240, 4, 32, "bf16", True),    # too big for shared memory: two-pass kernels
    (64, 512, 384, 8, 32, "fp32", False),    # two-pass, fp32
    (320, 32, 32, 1, 32, "bf16", True),      # one band: displaced == sync
]


@pytest.mark.parametrize("case", GN_CASES)
@pytest.mark.parametrize("mode", MODES)
def test_groupnorm_parity(case, mode):
    C, H, W, P, G, dtype, silu = case
    r = rng(C + H + mode)
    xs = rounded(r.standard_normal((C, H, W)) * 1.3 + 0.2, dtype)
    x = rounded(xs + 0.05 * r.standard_normal((C, H, W)) + 0.02, dtype)
    gamma = 1 + 0.3 * r.standard_normal(C)
    beta = 0.3 * r.standard_normal(C)
    sg, sl = O.refresh_stats(O.gn_fresh_local(xs, P, G))
    sg, sl = sg.astype(np.float32).astype(np.float64), sl.astype(np.float32).astype(np.float64)
    y_ref, f_ref, used_ref, _ = O.groupnorm_async(x, gamma, beta, P, G, 1e-5, 1.0, silu, mode, sg, sl)

    xd = dev_img(x, dtype)
    yd = torch.empty_like(xd)
    fresh = torch.zeros(P * G * 2, device="cuda")
    used = torch.zeros(P * G * 2, device="cuda")
    ws = torch.zeros(B.dp_groupnorm_workspace_size(H, W, C, G, P), dtype=torch.uint8, device="cuda")
    for _ in range(2):  # twice: the workspace must be left ready for reuse
        B.dp_groupnorm_async(xd, yd, dev_f32(gamma), dev_f32(beta), H, W, C, G, P, 1e-5, 1.0, silu,
                             mode, B.BF16 if dtype == "bf16" else B.FP32, dev_f32(sg), dev_f32(sl),
                             fresh, used, ws)
    torch.cuda.synchronize()
    np.testing.assert_allclose(host(fresh).reshape(P, G, 2), f_ref, rtol=0, atol=STATS_ATOL)
    np.testing.assert_allclose(host(used).reshape(P, G, 2), used_ref, rtol=0, atol=STATS_ATOL)
    if dtype == "fp32":
        check(host_img(yd), y_ref, atol=1e-4, rl2=1e-5, what="gn fp32")
    else:
        check(host_img(yd), y_ref, what="gn bf16", storage_rel=BF16_HALF_ULP)
    assert B.dp_device_status() == 0


@pytest.mark.parametrize("case", GN_CASES[:5])
def test_groupnorm_two_pass_with_minimal_workspace(case):
    """A workspace of only 256 + 128 P G bytes runs the two-kernel path even for
    tensors the single-pass kernel could hold (tiny bands, fewer pixels per
    block than SMs per band)."""
    C, H, W, P, G, dtype, silu = case
    mode = B.DISPLACED
    r = rng(3 * C + H)
    xs = rounded(r.standard_normal((C, H, W)) * 1.3 + 0.2, dtype)
    x = rounded(xs + 0.05 * r.standard_normal((C, H, W)) + 0.02, dtype)
    gamma = 1 + 0.3 * r.standard_normal(C)
    beta = 0.3 * r.standard_normal(C)
    sg, sl = O.refresh_stats(O.gn_fresh_local(xs, P, G))
    sg, sl = sg.astype(np.float32).astype(np.float64), sl.astype(np.float32).astype(np.float64)
    y_ref, f_ref, used_ref, _ = O.groupnorm_async(x, gamma, beta, P, G, 1e-5, 1.0, silu, mode, sg, sl)
    xd = dev_img(x, dtype)
    yd = torch.empty_like(xd)
    fresh = torch.zeros(P * G * 2, device="cuda")
    used = torch.zeros(P * G * 2, device="cuda")
    ws = torch.zeros(256 + 128 * P * G, dtype=torch.uint8, device="cuda")
    for _ in range(2):
        B.dp_groupnorm_async(xd, yd, dev_f32(gamma), dev_f32(beta), H, W, C, G, P, 1e-5, 1.0, silu,
                             mode, B.BF16 if dtype == "bf16" else B.FP32, dev_f32(sg), dev_f32(sl),
                             fresh, used, ws)
    torch.cuda.synchronize()
    np.testing.assert_allclose(host(fresh).reshape(P, G, 2), f_ref, rtol=0, atol=STATS_ATOL)
    np.testing.assert_allclose(host(used).reshape(P, G, 2), used_ref, rtol=0, atol=STATS_ATOL)
    if dtype == "fp32":
        check(host_img(yd), y_ref, atol=1e-4, rl2=1e-5, what="gn fp32 two-pass")
    else:
        check(host_img(yd), y_ref, what="gn bf16 two-pass", storage_rel=BF16_HALF_ULP)
    assert B.dp_device_status() == 0


def test_groupnorm_full_size_stats():
    """Statistics at the 1x320x480x480, P = 8 size, displaced mode."""
    C, H, W, P, G = 320, 480, 480, 8, 32
    r = rng(5)
    xs = rounded(r.standard_normal((C, H, W), dtype=np.float32), "bf16")
    x = rounded(xs + 0.05 * r.standard_normal((C, H, W), dtype=np.float32), "bf16")
    sg, sl = O.refresh_stats(O.gn_fresh_local(xs, P, G))
    f_ref = O.gn_fresh_local(x, P, G)
    used_ref, _ = O.gn_used_stats(f_ref, B.DISPLACED, sg, sl, 1.0)
    xd = dev_img(x, "bf16")
    yd = torch.empty_like(xd)
    fresh = torch.zeros(P * G * 2, device="cuda")
    used = torch.zeros(P * G * 2, device="cuda")
    ws = torch.zeros(B.dp_groupnorm_workspace_size(H, W, C, G, P), dtype=torch.uint8, device="cuda")
    B.dp_groupnorm_async(xd, yd, dev_f32(np.ones(C)), dev_f32(np.zeros(C)), H, W, C, G, P, 1e-5,
                         1.0, 1, B.DISPLACED, B.BF16, dev_f32(sg), dev_f32(sl), fresh, used, ws)
    torch.cuda.synchronize()
    np.testing.assert_allclose(host(fresh).reshape(P, G, 2), f_ref, rtol=0, atol=STATS_ATOL)
    np.testing.assert_allclose(host(used).reshape(P, G, 2), used_ref, rtol=0, atol=STATS_ATOL)
    # sampled rows of the output: band edges and interiors
    rows = [0, 59, 60, 61, 239, 240, 479]
    y = yd[rows].float().cpu().permute(2, 0, 1).double().numpy()
    sub = np.stack([x[:, rr, :] for rr in rows], axis=1)
    ref_rows = np.empty_like(sub)
    for i, rr in enumerate(rows):
        u = used_ref[rr // (H // P)]
        one = O.gn_apply(sub[:, i:i + 1, :], u[None], np.ones(C), np.zeros(C), 1, G, 1e-5, True)
        ref_rows[:, i:i + 1, :] = one
    check(y, ref_rows, what="gn full-size rows")


# ---------------------------------------------------------------- conv
CONV_CASES = [
    # Cin, Cout, H, W, P, stride, dtype, residual
    (64, 64, 16, 16, 4, 1, "bf16", False),
    (128, 96, 12, 20, 3, 1, "bf16", True),
    (64, 160, 32, 40, 4, 1, "bf16", True),
    (320, 320, 16, 24, 4, 1, "bf16", True),
    (64, 64, 16, 16, 2, 2, "bf16", False),
    (128, 64, 24, 36, 3, 2, "bf16", True),
    (320, 320, 12, 20, 3, 1, "bf16", True),     # pair kernel, ragged width
    (64, 320, 24, 16, 4, 1, "bf16", False),     # pair kernel, odd tile count
    (64, 320, 16, 16, 2, 2, "bf16", True),      # pair kernel, stride 2
    (320, 640, 8, 136, 2, 1, "bf16", True),     # pair kernel, 128-pixel rows, ragged
    (320, 320, 64, 256, 4, 1, "bf16", True),    # halo-row pair kernel, 256x320 tiles
    (320, 160, 6, 240, 3, 1, "bf16", False),    # halo-row pair kernel, 256x160, ragged row
    (64, 64, 16, 16, 2, 1, "fp32", False),
    (64, 128, 8, 10, 2, 1, "fp32", True),
    (32, 64, 9, 40, 3, 1, "fp32", True),        # fp32: ragged 32-column block, 16-channel slices
    (64, 32, 16, 20, 2, 2, "fp32", True),       # fp32, stride 2
    (16, 96, 8, 8, 1, 1, "fp32", False),        # fp32, one band
    (320, 320, 32, 48, 1, 1, "bf16", True),     # one band: no halo from other bands
    (64, 64, 16, 16, 1, 2, "bf16", False),      # one band, stride 2
]


@pytest.mark.parametrize("case", CONV_CASES)
@pytest.mark.parametrize("mode", MODES)
def test_conv3x3_halo_parity(case, mode):
    Cin, Cout, H, W, P, stride, dtype, use_res = case
    r = rng(Cin + Cout + H + W + stride + mode)
    af = rounded(r.standard_normal((Cin, H, W)), dtype)
    ast = rounded(r.standard_normal((Cin, H, W)), dtype)
    wt = rounded(r.standard_normal((Cout, Cin, 3, 3)) * math.sqrt(2 / (9 * Cin)), dtype)
    b = 0.3 * r.standard_normal(Cout)
    Ho, Wo = (H - 1) // stride + 1, (W - 1) // stride + 1
    res = rounded(r.standard_normal((Cout, Ho, Wo)), dtype) if use_res else None
    ref = O.conv3x3_halo(af, ast, wt, b, res, P, mode, stride)
    out = torch.empty(Ho, Wo, Cout, dtype=torch.bfloat16 if dtype == "bf16" else torch.float32,
                      device="cuda")
    B.dp_conv3x3_halo(dev_img(af, dtype), dev_img(ast, dtype), conv_w_dev(wt, dtype), dev_f32(b),
                      dev_img(res, dtype) if use_res else None, out, H, W, Cin, Cout, stride, P,
                      mode, B.BF16 if dtype == "bf16" else B.FP32)
    torch.cuda.synchronize()
    if dtype == "fp32":
        check(host_img(out), ref, atol=F32_ATOL, rl2=F32_RL2, what=f"conv {case} mode {mode}")
    else:
        check(host_img(out), ref, what=f"conv {case} mode {mode}", storage_rel=BF16_HALF_ULP)
    assert B.dp_device_status() == 0


SPLIT_K_CONV_CASES = [
    # Cin, Cout, H, W, P, stride, residual: few output tiles, long K
    (640, 640, 16, 16, 2, 1, True),      # 2 pair tiles of 256x320, K runs across the GPU
    (640, 1280, 32, 32, 4, 1, False),    # the 1280-channel stage shape
    (640, 640, 64, 64, 4, 2, True),      # stride 2, 32x32 output
    (640, 640, 24, 40, 4, 1, True),      # 8-pixel-wide tiles of 16 rows, ragged band
]


@pytest.mark.parametrize("case", SPLIT_K_CONV_CASES)
@pytest.mark.parametrize("mode", [B.DISPLACED, B.SYNC])
def test_conv3x3_split_k_parity(case, mode):
    """With a workspace, convs with too few output tiles cut K into runs whose
    fp32 partials the last run sums; checked against the oracle twice in a row
    (the second call reuses the workspace's run counters)."""
    Cin, Cout, H, W, P, stride, use_res = case
    r = rng(7 * Cin + Cout + H + W + stride + mode)
    af = rounded(r.standard_normal((Cin, H, W)), "bf16")
    ast = rounded(r.standard_normal((Cin, H, W)), "bf16")
    wt = rounded(r.standard_normal((Cout, Cin, 3, 3)) * math.sqrt(2 / (9 * Cin)), "bf16")
    b = 0.3 * r.standard_normal(Cout)
    Ho, Wo = (H - 1) // stride + 1, (W - 1) // stride + 1
    res = rounded(r.standard_normal((Cout, Ho, Wo)), "bf16") if use_res else None
    ref = O.conv3x3_halo(af, ast, wt, b, res, P, mode, stride)
    nws = B.dp_gemm_workspace_size()
    ws = torch.zeros(nws, dtype=torch.uint8, device="cuda")
    out = torch.empty(Ho, Wo, Cout, dtype=torch.bfloat16, device="cuda")
    for call in range(2):
        out.zero_()
        B.dp_conv3x3_halo(dev_img(af, "bf16"), dev_img(ast, "bf16"), conv_w_dev(wt, "bf16"), dev_f32(b),
                          dev_img(res, "bf16") if use_res else None, out, H, W, Cin, Cout, stride, P,
                          mode, B.BF16, ws, nws)
        torch.cuda.synchronize()
        check(host_img(out), ref, what=f"split-K conv {case} mode {mode} call {call}",
              storage_rel=BF16_HALF_ULP)
    assert B.dp_device_status() == 0


def test_linear_split_k_parity():
    r = rng(99)
    M, N, K = 1024, 640, 5120
    x = rounded(r.standard_normal((M, K)), "bf16")
    w = rounded(r.standard_normal((N, K)) / math.sqrt(K), "bf16")
    b = 0.3 * r.standard_normal(N)
    res = rounded(r.standard_normal((M, N)), "bf16")
    ref = x @ w.T + b + res
    nws = B.dp_gemm_workspace_size()
    ws = torch.zeros(nws, dtype=torch.uint8, device="cuda")
    out = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    B.dp_linear(dev_mat(x), dev_mat(w), dev_f32(b), dev_mat(res), out, None, None, M, N, K, N, ws, nws)
    torch.cuda.synchronize()
    check(host(out), ref, what="split-K linear", storage_rel=BF16_HALF_ULP)
    assert B.dp_device_status() == 0


def test_conv_small_parity():
    for mode in MODES:
        r = rng(40 + mode)
        Cin, Cout, H, W, P = 4, 64, 16, 12, 4
        af = rounded(r.standard_normal((Cin, H, W)), "bf16")
        ast = rounded(r.standard_normal((Cin, H, W)), "bf16")
        wt = rounded(r.standard_normal((Cout, Cin, 3, 3)) * math.sqrt(2 / (9 * Cin)), "bf16")
        b = 0.3 * r.standard_normal(Cout)
        ref = O.conv3x3_halo(af, ast, wt, b, None, P, mode)
        out = torch.empty(H, W, Cout, dtype=torch.bfloat16, device="cuda")
        B.dp_conv3x3_halo_small(dev_img(af, "bf16"), dev_img(ast, "bf16"), conv_w_dev(wt, "bf16"),
                                dev_f32(b), out, H, W, Cin, Cout, P, mode)
        torch.cuda.synchronize()
        check(host_img(out), ref, what=f"small conv mode {mode}", storage_rel=BF16_HALF_ULP)


# ---------------------------------------------------------------- linear
@pytest.mark.parametrize("M,N,K,split,use_res", [(300, 192, 128, 192, True), (256, 384, 128, 128, False),
                                                 (4096, 1920, 640, 640, False),
                                                 (1000, 640, 320, 640, True),
                                                 (384, 960, 128, 320, False),
                                                 (130, 320, 64, 320, True),
                                                 # pair tiles with a residual; several tiles per
                                                 # SM pair reuse both accumulators; ragged M
                                                 (4096, 640, 640, 640, True),
                                                 (3000, 1280, 512, 1280, True)])
def test_linear_parity(M, N, K, split, use_res):
    r = rng(M + N + K)
    x = rounded(r.standard_normal((M, K)), "bf16")
    w = rounded(r.standard_normal((N, K)) / math.sqrt(K), "bf16")
    b = 0.3 * r.standard_normal(N)
    res = rounded(r.standard_normal((M, N)), "bf16") if use_res else None
    ref = x @ w.T + b + (res if use_res else 0)
    outs = [torch.empty(M, split, dtype=torch.bfloat16, device="cuda") for _ in range(N // split)]
    outs += [None] * (3 - len(outs))
    B.dp_linear(dev_mat(x), dev_mat(w), dev_f32(b), dev_mat(res) if use_res else None, outs[0],
                outs[1], outs[2], M, N, K, split)
    torch.cuda.synchronize()
    got = np.concatenate([host(o) for o in outs if o is not None], axis=1)
    check(got, ref, what="linear", storage_rel=BF16_HALF_ULP)


# ---------------------------------------------------------------- attention
@pytest.mark.parametrize("T,heads,P,qscale", [(512, 2, 2, 1.0), (512, 2, 4, 3.0), (1024, 3, 2, 1.0),
                                              (1536, 5, 2, 2.0), (2048, 4, 16, 1.0), (4096, 10, 4, 1.0),
                                              (512, 3, 1, 1.0), (384, 2, 1, 2.0)])
@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("split", [True, False], ids=["split", "whole_tiles"])
def test_attention_parity(T, heads, P, qscale, mode, split):
    """With a workspace the key tiles of a query tile may be cut between CTAs
    (the cost model cuts them at T=1024, 1536, 2048 and 4096) and the partial
    softmax sums are merged; without one every CTA takes whole tiles.  Bands
    of 256, 512, 768 and 1024 tokens run the two-query-tile kernel, bands of
    128 tokens the one-tile kernel."""
    r = rng(T + heads + P + mode)
    C = heads * 64
    q = rounded(qscale * r.standard_normal((T, C)), "bf16")
    kf, vf, ks, vs = (rounded(r.standard_normal((T, C)), "bf16") for _ in range(4))
    ref = O.attention_stale_kv(q, kf, vf, ks, vs, P, heads, 0.125, mode)
    o = torch.empty(T, C, dtype=torch.bfloat16, device="cuda")
    nws = B.dp_attn_workspace_size()
    ws = torch.zeros(nws, dtype=torch.uint8, device="cuda") if split else None
    for _ in range(2):   # the second call reuses the workspace's flags
        o.zero_()
        B.dp_attn_stale_kv(dev_mat(q), dev_mat(kf), dev_mat(vf), dev_mat(ks), dev_mat(vs), o, T, heads,
                           64, P, 0.125, mode, ws, nws if split else 0)
        torch.cuda.synchronize()
        check(host(o), ref, what=f"attention T={T} P={P} mode={mode} split={split}")
    assert B.dp_device_status() == 0


@pytest.mark.parametrize("Tq,Tk,heads", [(1024, 77, 10), (4096, 77, 10), (256, 128, 2), (512, 200, 4),
                                          (256, 1, 2), (768, 300, 3)])
@pytest.mark.parametrize("split", [True, False], ids=["split", "whole_tiles"])
def test_cross_attention_parity(Tq, Tk, heads, split):
    """Queries over a context of Tk keys every band sees whole (77 = an SDXL text context); a
    ragged last key tile is masked."""
    r = rng(Tq + Tk + heads)
    C = heads * 64
    q = rounded(r.standard_normal((Tq, C)), "bf16")
    k, v = (rounded(r.standard_normal((Tk, C)), "bf16") for _ in range(2))
    ref = O.attention_cross(q, k, v, heads, 0.125)
    o = torch.empty(Tq, C, dtype=torch.bfloat16, device="cuda")
    nws = B.dp_attn_workspace_size()
    ws = torch.zeros(nws, dtype=torch.uint8, device="cuda") if split else None
    for _ in range(2):   # the second call reuses the workspace's flags
        o.zero_()
        B.dp_attn_cross(dev_mat(q), dev_mat(k), dev_mat(v), o, Tq, Tk, heads, 64, 0.125, ws,
                        nws if split else 0)
        torch.cuda.synchronize()
        check(host(o), ref, what=f"cross-attention Tq={Tq} Tk={Tk} split={split}")
    assert B.dp_device_status() == 0


# ---------------------------------------------------------------- per-token operators
@pytest.mark.parametrize("T,C", [(4096, 640), (1024, 1280), (300, 320), (7, 8), (33, 2048)])
def test_layernorm_parity(T, C):
    r = rng(T + C)
    x = rounded(1.5 * r.standard_normal((T, C)) + 0.4, "bf16")
    g, b = 1 + 0.3 * r.standard_normal(C), 0.3 * r.standard_normal(C)
    y = torch.empty(T, C, dtype=torch.bfloat16, device="cuda")
    B.dp_layernorm(dev_mat(x), y, dev_f32(g), dev_f32(b), T, C, 1e-5)
    torch.cuda.synchronize()
    check(host(y), O.layer_norm(x, g, b, 1e-5), what=f"layernorm T={T} C={C}", storage_rel=BF16_HALF_ULP)


@pytest.mark.parametrize("T,F", [(4096, 2560), (1024, 5120), (77, 8), (5, 24)])
def test_geglu_parity(T, F):
    r = rng(T + F)
    h = rounded(2.0 * r.standard_normal((T, 2 * F)), "bf16")
    y = torch.empty(T, F, dtype=torch.bfloat16, device="cuda")
    B.dp_geglu(dev_mat(h), y, T, F)
    torch.cuda.synchronize()
    check(host(y), h[:, :F] * O.gelu(h[:, F:]), what=f"geglu T={T} F={F}", storage_rel=BF16_HALF_ULP)


# ---------------------------------------------------------------- refresh
def test_refresh_is_an_exact_copy():
    g = torch.Generator(device="cpu").manual_seed(3)
    H, W, C, P = 64, 48, 320, 4
    fresh = torch.randint(-2 ** 15, 2 ** 15, (H, W, C), generator=g, dtype=torch.int16).cuda()
    stale = torch.zeros_like(fresh)
    B.dp_refresh_stale(fresh, stale, W * C * 2, H, P, 2)
    torch.cuda.synchronize()
    hb = H // P
    assert torch.equal(stale[2 * hb:3 * hb], fresh[2 * hb:3 * hb])
    assert int(stale[:2 * hb].abs().sum()) == 0 and int(stale[3 * hb:].abs().sum()) == 0
    B.dp_refresh_stale(fresh, stale, W * C * 2, H, P, -1)
    torch.cuda.synchronize()
    assert torch.equal(stale, fresh)


@pytest.mark.parametrize("H,W,C,P,above,below", [(480, 480, 320, 8, 1, 1), (128, 128, 320, 4, 1, 0),
                                                  (12, 8, 64, 3, 2, 3), (16, 8, 64, 1, 1, 1),
                                                  (16, 8, 64, 4, 4, 4)])
def test_refresh_halo_copies_exactly_the_band_edge_rows(H, W, C, P, above, below):
    g = torch.Generator(device="cpu").manual_seed(4)
    fresh = torch.randint(-2 ** 15, 2 ** 15, (H, W, C), generator=g, dtype=torch.int16).cuda()
    stale = torch.randint(-2 ** 15, 2 ** 15, (H, W, C), generator=g, dtype=torch.int16).cuda()
    want = stale.clone()
    hb = H // P
    for e in range(P - 1):
        r0, r1 = (e + 1) * hb - above, (e + 1) * hb + below
        want[r0:r1] = fresh[r0:r1]
    B.dp_refresh_halo(fresh, stale, W * C * 2, H, P, above, below)
    torch.cuda.synchronize()
    assert torch.equal(stale, want)


@pytest.mark.parametrize("stride", [1, 2])
def test_halo_refresh_is_all_a_displaced_conv_reads(stride):
    """A displaced conv gives the same bits whether its stale buffer was refreshed whole or only
    at the band-edge rows it reads (1 above and 1 below for stride 1, 1 above for stride 2)."""
    r = rng(77 + stride)
    H, W, C, P = 64, 48, 128, 4
    prev = torch.from_numpy(r.standard_normal((H, W, C)).astype(np.float32)).to(torch.bfloat16).cuda()
    cur = torch.from_numpy(r.standard_normal((H, W, C)).astype(np.float32)).to(torch.bfloat16).cuda()
    wt = torch.from_numpy(0.05 * r.standard_normal((C, 3, 3, C)).astype(np.float32)).to(torch.bfloat16).cuda()
    b = torch.zeros(C, device="cuda")
    full = prev.clone()
    halo = torch.from_numpy(r.standard_normal((H, W, C)).astype(np.float32)).to(torch.bfloat16).cuda()
    B.dp_refresh_stale(prev, full, W * C * 2, H, P, -1)
    B.dp_refresh_halo(prev, halo, W * C * 2, H, P, 1, 1 if stride == 1 else 0)
    Ho, Wo = (H - 1) // stride + 1, (W - 1) // stride + 1
    o_full = torch.empty(Ho, Wo, C, dtype=torch.bfloat16, device="cuda")
    o_halo = torch.empty_like(o_full)
    B.dp_conv3x3_halo(cur, full, wt, b, None, o_full, H, W, C, C, stride, P, B.DISPLACED, B.BF16)
    B.dp_conv3x3_halo(cur, halo, wt, b, None, o_halo, H, W, C, C, stride, P, B.DISPLACED, B.BF16)
    torch.cuda.synchronize()
    assert torch.equal(o_full, o_halo)
    assert not torch.equal(full, halo)   # the interiors really differ


def test_refresh_stats():
    P, G = 4, 32
    f = torch.randn(P * G * 2, device="cuda")
    sl = torch.zeros_like(f)
    sg = torch.zeros(G * 2, device="cuda")
    B.dp_refresh_stats(f, sl, sg, P, G)
    torch.cuda.synchronize()
    assert torch.equal(sl, f)
    torch.testing.assert_close(sg.view(G, 2), f.view(P, G, 2).double().mean(0).float(), rtol=0, atol=1e-6)
