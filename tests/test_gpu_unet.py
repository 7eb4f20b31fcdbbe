"""GPU parity of the SDXL-shaped U-Net step and its up-path kernels.

The channel concatenation and the nearest 2x upsampling are copies, compared bit for bit with
the oracle; the narrow-output 3x3 conv (a U-Net's conv_out back to 4 latent channels) is held
to the stated bar in bf16 and to the fp32 bar in fp32, in every mode, at stride 1 and 2 and
with a ragged tile.  The whole U-Net step (base width 64, transformer depths 0 / 1 / 1, a
4x64x64 latent over 2 bands) runs a sync step and displaced steps of a drifting latent, with a
time embedding and a text context, against the oracle end to end (check_chain: the chain
stores some 150 intermediates in bf16).
"""
import numpy as np
import pytest
import torch

from displaced_patch_parallelism_b200 import binding as B
from displaced_patch_parallelism_b200 import synth
from displaced_patch_parallelism_b200.weights import unet_sdxl_weights
from oracle import dp_oracle as O
from tests.helpers import (BF16_HALF_ULP, F32_ATOL, F32_RL2, check, check_chain, conv_w_dev, dev_f32,
                           dev_img, host_img, rounded)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_concat_and_upsample_are_exact(dtype):
    r = np.random.default_rng(130)
    H, W, Ca, Cb = 24, 40, 64, 24
    a = rounded(r.standard_normal((Ca, H, W)), dtype)
    b = rounded(r.standard_normal((Cb, H, W)), dtype)
    dt = B.BF16 if dtype == "bf16" else B.FP32
    out = torch.empty(H, W, Ca + Cb, dtype=dev_img(a, dtype).dtype, device="cuda")
    B.dp_concat_channels(dev_img(a, dtype), dev_img(b, dtype), out, H * W, Ca, Cb, dt)
    up = torch.empty(2 * H, 2 * W, Ca, dtype=out.dtype, device="cuda")
    B.dp_upsample_nearest2x(dev_img(a, dtype), up, H, W, Ca, dt)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host_img(out), O.concat_channels(a, b))
    np.testing.assert_array_equal(host_img(up), O.upsample_nearest2x(a))


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("stride", [1, 2])
@pytest.mark.parametrize("mode", [B.SYNC, B.DISPLACED, B.NAIVE])
@pytest.mark.parametrize("cout", [4, 7, 16])
def test_narrow_conv(dtype, stride, mode, cout):
    """3x3 conv to 4, 7 and 16 channels (the CUDA-core path), 72 columns (a ragged 64-pixel
    tile), four bands, bias and (stride 1) residual, against the oracle's halo conv.  Outputs
    reach |y| ~ 9, where storing in bf16 alone moves a value by more than 2e-2: the bf16 case
    takes the storage-aware bound (2e-2 + half an ulp of the output)."""
    r = np.random.default_rng(131 + cout + 10 * stride + 100 * mode)
    H, W, Cin, P = 32, 72, 128, 4
    af = rounded(r.standard_normal((Cin, H, W)), dtype)
    ast = rounded(r.standard_normal((Cin, H, W)), dtype)
    wt = rounded(r.standard_normal((cout, Cin, 3, 3)) * np.sqrt(2.0 / (9 * Cin)), dtype)
    bias = r.standard_normal(cout).astype(np.float32).astype(np.float64)
    Ho, Wo = (H - 1) // stride + 1, (W - 1) // stride + 1
    res = rounded(r.standard_normal((cout, Ho, Wo)), dtype) if stride == 1 else None
    dt = B.BF16 if dtype == "bf16" else B.FP32
    out = torch.empty(Ho, Wo, cout, dtype=dev_img(af, dtype).dtype, device="cuda")
    B.dp_conv3x3_halo(dev_img(af, dtype), dev_img(ast, dtype), conv_w_dev(wt, dtype), dev_f32(bias),
                      None if res is None else dev_img(res, dtype), out, H, W, Cin, cout, stride, P, mode, dt)
    torch.cuda.synchronize()
    ref = O.conv3x3_halo(af, ast, wt, bias, res, P, mode, stride)
    if dtype == "bf16":
        check(host_img(out), ref, what=f"narrow conv {cout} stride {stride} mode {mode}",
              storage_rel=BF16_HALF_ULP)
    else:
        check(host_img(out), ref, atol=F32_ATOL, rl2=F32_RL2, what=f"fp32 narrow conv {cout}")


UNET = dict(C=4, H=64, W=64, P=2, G=32, base=64, depths=(0, 1, 1), Tk=77, Cc=128, Ct=128)


def _unet_workload():
    u = UNET
    return synth.Workload(name="unet_sdxl_test", kind="unet_sdxl", C=u["C"], H=u["H"], W=u["W"],
                          P=u["P"], G=u["G"], base=u["base"], depths=u["depths"], ctx_len=u["Tk"],
                          ctx_dim=u["Cc"], temb_dim=u["Ct"], weight_seed=17)


def test_unet_sdxl_plan_matches_the_stages():
    """The block's weight list is the marshalled stage list plus context and time embedding."""
    u = UNET
    wl = _unet_workload()
    blk = B.Block(B.UNET_SDXL, u["H"], u["W"], u["C"], u["C"], u["G"], u["P"], 0, B.BF16, True, 1e-5,
                  1.0, context=(u["Tk"], u["Cc"], 0), temb_dim=u["Ct"], unet=(u["base"],) + u["depths"])
    dw = unet_sdxl_weights(synth.make_weights(wl, True), synth.sdxl_unet_stages(u["base"], u["depths"]),
                           u["depths"])
    assert len(dw) + 2 == B.dp_block_weight_count(blk.desc)


@pytest.mark.parametrize("context_fixed", [False, True])
def test_unet_sdxl_step(context_fixed):
    """The whole U-Net step on the GPU against the oracle: a sync step, three displaced steps
    of a drifting latent and a naive step of a fresh state, every output compared (with a
    fixed context, every transformer layer's context keys and values come from the first
    step)."""
    u = UNET
    wl = _unet_workload()
    wts = synth.make_weights(wl, random_affine=True)
    stages = synth.sdxl_unet_stages(u["base"], u["depths"])
    dev_w = unet_sdxl_weights(wts, stages, u["depths"])
    g = torch.Generator().manual_seed(18)
    ctx = torch.randn(u["Tk"], u["Cc"], generator=g).to(torch.bfloat16).to(torch.float32)
    temb = torch.randn(u["Ct"], generator=g)
    dev_w += [ctx.to(torch.bfloat16).cuda(), temb.cuda()]
    w64 = {n: v.double().numpy() for n, v in wts.items()}
    c64, t64 = ctx.double().numpy(), temb.double().numpy()

    def oracle(st, xr, mode, storage, final):
        return O.sdxl_unet_step(st, xr, c64, t64, w64, u["P"], u["G"], 1e-5, 1.0, mode, storage,
                                base=u["base"], depths=u["depths"], final_storage=final)

    def make_block():
        return B.Block(B.UNET_SDXL, u["H"], u["W"], u["C"], u["C"], u["G"], u["P"], 0, B.BF16, True,
                       1e-5, 1.0, context=(u["Tk"], u["Cc"], 0), temb_dim=u["Ct"],
                       unet=(u["base"],) + u["depths"], context_fixed=context_fixed)

    blk = make_block()
    st, st_exact = {}, {}
    x = torch.randn(u["C"], u["H"], u["W"], generator=g)
    for k, mode in enumerate([B.SYNC, B.DISPLACED, B.DISPLACED, B.DISPLACED]):
        if k:
            x = x + 0.05 * torch.randn(x.shape, generator=g)
        xr = x.to(torch.bfloat16).double().numpy()
        out = torch.empty(u["H"], u["W"], u["C"], dtype=torch.bfloat16, device="cuda")
        blk.step(dev_img(xr, "bf16"), out, dev_w, mode)
        ref = oracle(st, xr, mode, "bf16", "none")
        exact = oracle(st_exact, xr, mode, "none", None)
        torch.cuda.synchronize()
        print(check_chain(host_img(out), exact, ref, what=f"SDXL U-Net step {k} mode {mode}"))
    assert blk.status() == 0 and B.dp_device_status() == 0
    naive = make_block()
    out = torch.empty(u["H"], u["W"], u["C"], dtype=torch.bfloat16, device="cuda")
    naive.step(dev_img(xr, "bf16"), out, dev_w, B.NAIVE)
    ref = oracle({}, xr, B.NAIVE, "bf16", "none")
    exact = oracle({}, xr, B.NAIVE, "none", None)
    torch.cuda.synchronize()
    print(check_chain(host_img(out), exact, ref, what="SDXL U-Net naive step"))


def test_unet_sdxl_step_eight_bands():
    """The U-Net step over 8 bands of a 4x128x128 latent (base 64, depths 0 / 1 / 1): 16-row
    bands at the first level, 8 at the second and 4 (128 tokens) at the third, so every conv
    halo and every down / up sampling crosses band edges at every level.  A sync step and two
    displaced steps of a drifting latent against the oracle, end to end (check_chain)."""
    wl = synth.Workload(name="unet_sdxl_p8", kind="unet_sdxl", C=4, H=128, W=128, P=8, G=32, base=64,
                        depths=(0, 1, 1), ctx_len=77, ctx_dim=128, temb_dim=128, weight_seed=19)
    wts = synth.make_weights(wl, random_affine=True)
    dev_w = unet_sdxl_weights(wts, synth.sdxl_unet_stages(wl.base, wl.depths), wl.depths)
    g = torch.Generator().manual_seed(20)
    ctx = torch.randn(wl.ctx_len, wl.ctx_dim, generator=g).to(torch.bfloat16).to(torch.float32)
    temb = torch.randn(wl.temb_dim, generator=g)
    dev_w += [ctx.to(torch.bfloat16).cuda(), temb.cuda()]
    w64 = {n: v.double().numpy() for n, v in wts.items()}
    c64, t64 = ctx.double().numpy(), temb.double().numpy()
    blk = B.Block(B.UNET_SDXL, wl.H, wl.W, wl.C, wl.C, wl.G, wl.P, 0, B.BF16, True, 1e-5, 1.0,
                  context=(wl.ctx_len, wl.ctx_dim, 0), temb_dim=wl.temb_dim, unet=(wl.base,) + wl.depths,
                  context_fixed=True)
    st, st_exact = {}, {}
    x = torch.randn(wl.C, wl.H, wl.W, generator=g)
    for k, mode in enumerate([B.SYNC, B.DISPLACED, B.DISPLACED]):
        if k:
            x = x + 0.05 * torch.randn(x.shape, generator=g)
        xr = x.to(torch.bfloat16).double().numpy()
        out = torch.empty(wl.H, wl.W, wl.C, dtype=torch.bfloat16, device="cuda")
        blk.step(dev_img(xr, "bf16"), out, dev_w, mode)
        kw = dict(base=wl.base, depths=wl.depths)
        ref = O.sdxl_unet_step(st, xr, c64, t64, w64, wl.P, wl.G, 1e-5, 1.0, mode, "bf16", final_storage="none", **kw)
        exact = O.sdxl_unet_step(st_exact, xr, c64, t64, w64, wl.P, wl.G, 1e-5, 1.0, mode, "none", **kw)
        torch.cuda.synchronize()
        print(check_chain(host_img(out), exact, ref, what=f"SDXL U-Net P=8 step {k} mode {mode}"))
    assert blk.status() == 0 and B.dp_device_status() == 0


def test_unet_sdxl_full_size_properties():
    """SDXL's whole U-Net at 1024 px (latent 4x128x128, 8 bands, depths 0 / 2 / 10, the
    benchmark's workload), beyond the oracle's reach at this size, held to properties that hold
    at any size: a displaced step of an unchanged latent reproduces the sync step (every stale
    buffer then holds what a sync step computes; only rounding differs), both are finite, and a
    naive step (no context between bands) lies much further from them; graph replays of the
    displaced step agree with it as well; no bounded wait ran out."""
    wl = synth.WORKLOADS["unet_sdxl_4x128x128"]
    dev = torch.device("cuda")
    wts = synth.make_weights(wl, device=dev)
    dw = unet_sdxl_weights(wts, synth.sdxl_unet_stages(wl.base, wl.depths), wl.depths, torch.bfloat16, dev)
    del wts
    dw += [synth.context(wl).to(torch.bfloat16).to(dev), synth.randn((wl.temb_dim,), wl.seed + 600).to(dev)]

    def block():
        return B.Block(B.UNET_SDXL, wl.H, wl.W, wl.C, wl.C, wl.G, wl.P, 0, B.BF16, True, wl.eps, 1.0,
                       context=(wl.ctx_len, wl.ctx_dim, 0), temb_dim=wl.temb_dim,
                       unet=(wl.base,) + tuple(wl.depths), context_fixed=True)

    x = synth.nchw_to_nhwc(synth.InputStream(wl).x(0)).to(torch.bfloat16).to(dev)
    outs = {m: torch.empty(wl.H, wl.W, wl.C, dtype=torch.bfloat16, device=dev) for m in ("s", "d", "n", "g")}
    blk = block()
    blk.step(x, outs["s"], dw, B.SYNC)
    blk.step(x, outs["d"], dw, B.DISPLACED)
    naive = block()
    naive.step(x, outs["n"], dw, B.NAIVE)
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        g = blk.graph(x, outs["g"], dw, B.DISPLACED, stream)
        # the plain step above ran at one parity: replay twice so one replay has that parity
        g.launch(stream)
        first = outs["g"].clone()
        g.launch(stream)
    torch.cuda.synchronize()
    g.close()
    s, d, n = (outs[k].double() for k in "sdn")
    assert torch.isfinite(s).all() and torch.isfinite(d).all() and torch.isfinite(n).all()
    rel = lambda a, b: float(torch.linalg.norm(a - b) / torch.linalg.norm(b))
    r_d, r_n = rel(d, s), rel(n, s)
    print({"displaced_vs_sync": r_d, "naive_vs_sync": r_n})
    # measured on B200: 1.5e-2 (the sync step's grid-wide GroupNorm and the displaced step's
    # cluster GroupNorm add in different orders; over ~150 bf16-stored stages, ten-layer
    # transformers included, those last-bit differences grow) against 0.59 for naive patches
    assert r_d < 5e-2, r_d
    assert r_n > 10 * r_d, (r_n, r_d)
    # every displaced step of this unchanged latent computes the same thing, so the graph
    # replays agree with the sync step as closely as the plain displaced step does
    assert rel(first.double(), s) < 5e-2 and rel(outs["g"].double(), s) < 5e-2
    assert blk.status() == 0 and naive.status() == 0 and B.dp_device_status() == 0
