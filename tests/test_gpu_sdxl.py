"""GPU parity of the SDXL-shaped parts: the transformer block kind and the ResBlock time
embedding, through dp_block_step and dp_time_embedding_bias.

The transformer block (GroupNorm and self-attention whose other-band context is the previous
step's, then per-token LayerNorms, cross-attention over a text context every band sees whole,
and a GELU-gated feed-forward) and a ResBlock with a time embedding that changes every step
run a sync step and displaced steps of a drifting input on the GPU and in the oracle from the
same seeded inputs; every step's output is compared.
"""
import numpy as np
import pytest
import torch

from displaced_patch_parallelism_b200 import binding as B
from displaced_patch_parallelism_b200 import synth
from displaced_patch_parallelism_b200.weights import block_weights
from oracle import dp_oracle as O
from tests.helpers import BF16_HALF_ULP, check, dev_img, host_img

pytestmark = pytest.mark.gpu


# The transformer block stores its residual stream and every intermediate in bf16 at about
# fourteen points (GroupNorm, proj_in, three LayerNorms, q/k/v, both attention outputs, the
# context projections, the two feed-forward intermediates and three residual sums).  The GPU
# and the oracle round at the same points, so an element whose fp32 value differs in the last
# bits can round to neighbouring bf16 values on the two sides, and that difference then feeds
# every later stage: as for the mini U-Net chain, the per-element bound carries a chain term,
# 2^-5 of the output's largest magnitude, while rel-L2 keeps the 5e-3 bar.
TRANSFORMER_SCALE = 2.0 ** -5


def test_transformer_block():
    """SDXL-shaped transformer block (GroupNorm and self-attention with stale context, then
    per-token LayerNorms, cross-attention over a 77-token text context and a gated feed-forward)
    against the oracle, through a sync step and two displaced steps of a drifting input."""
    C, H, W, P, G, heads, Tk, Cc, F = 320, 32, 32, 4, 32, 5, 77, 128, 1280
    g = torch.Generator().manual_seed(11)
    rnd = lambda *shape, std=1.0: torch.randn(*shape, generator=g) * std
    bf = lambda t: t.to(torch.bfloat16).to(torch.float32)        # matrices are stored in bf16
    wts = {"gn_gamma": 1 + 0.2 * rnd(C), "gn_beta": 0.2 * rnd(C),
           "proj_in_w": bf(rnd(C, C, std=C ** -0.5)), "proj_in_b": 0.1 * rnd(C),
           "proj_out_w": bf(rnd(C, C, std=C ** -0.5)), "proj_out_b": 0.1 * rnd(C),
           "cq_w": bf(rnd(C, C, std=C ** -0.5)), "ck_w": bf(rnd(C, Cc, std=Cc ** -0.5)),
           "cv_w": bf(rnd(C, Cc, std=Cc ** -0.5)), "co_w": bf(rnd(C, C, std=C ** -0.5)),
           "co_b": 0.1 * rnd(C), "ff1_w": bf(rnd(2 * F, C, std=C ** -0.5)), "ff1_b": 0.1 * rnd(2 * F),
           "ff2_w": bf(rnd(C, F, std=F ** -0.5)), "ff2_b": 0.1 * rnd(C)}
    for n in ("wq", "wk", "wv", "wo"):
        wts[n] = bf(rnd(C, C, std=C ** -0.5))
    for n in ("bq", "bk", "bv", "bo"):
        wts[n] = 0.1 * rnd(C)
    for i in (1, 2, 3):
        wts[f"ln{i}_g"], wts[f"ln{i}_b"] = 1 + 0.2 * rnd(C), 0.2 * rnd(C)
    ctx = bf(rnd(Tk, Cc))
    dev_w = block_weights("transformer", wts) + [ctx.to(torch.bfloat16).cuda()]
    blk = B.Block(B.TRANSFORMER, H, W, C, C, G, P, heads, B.BF16, False, 1e-5, 1.0,
                  context=(Tk, Cc, F))
    w64 = {n: v.double().numpy() for n, v in wts.items()}
    st = {}
    x = rnd(C, H, W)
    for k, mode in enumerate([B.SYNC, B.DISPLACED, B.DISPLACED]):
        if k:
            x = x + 0.05 * rnd(C, H, W)
        xr = bf(x).double().numpy()
        out = torch.empty(H, W, C, dtype=torch.bfloat16, device="cuda")
        blk.step(dev_img(xr, "bf16"), out, dev_w, mode)
        ref = O.transformer_step(st, xr, ctx.double().numpy(), w64, P, G, 1e-5, 1.0, heads, mode, "bf16",
                                 final_storage="none")
        torch.cuda.synchronize()
        check(host_img(out), ref, what=f"transformer step {k} mode {mode}", storage_rel=BF16_HALF_ULP,
              scale_rel=TRANSFORMER_SCALE)
    assert B.dp_device_status() == 0


@pytest.mark.parametrize("Ct,Cout,with_biases", [(1280, 320, True), (1280, 1280, False),
                                                 (77, 9, True), (1, 1, True), (8192, 40, True)])
def test_time_embedding_bias(Ct, Cout, with_biases):
    """conv_b + temb_w silu(temb) + temb_b per output channel, against the oracle's term.
    fp32 accumulation over Ct terms: each output is held to 1e-6 + 2^-14 of the sum of its
    terms' magnitudes, well above fp32 summation and expf error at these lengths."""
    g = torch.Generator().manual_seed(Ct + Cout)
    temb = torch.randn(Ct, generator=g) * 2.0
    tw = torch.randn(Cout, Ct, generator=g) * Ct ** -0.5
    tb = torch.randn(Cout, generator=g) * 0.3 if with_biases else None
    cb = torch.randn(Cout, generator=g) * 0.3 if with_biases else None
    bias = torch.full((Cout,), float("nan"), device="cuda")
    dev = lambda t: None if t is None else t.cuda()
    B.dp_time_embedding_bias(dev(temb), dev(tw), dev(tb), dev(cb), bias, Ct, Cout)
    torch.cuda.synchronize()
    t64 = temb.double().numpy()
    ref = O.time_embedding_term(t64, tw.double().numpy(), None if tb is None else tb.double().numpy())
    mag = np.abs(tw.double().numpy()) @ np.abs(t64 / (1.0 + np.exp(-t64)))
    if cb is not None:
        ref = ref + cb.double().numpy()
        mag = mag + np.abs(tb.double().numpy()) + np.abs(cb.double().numpy())
    got = bias.cpu().double().numpy()
    assert np.isfinite(got).all()
    assert (np.abs(got - ref) <= 1e-6 + 2.0 ** -14 * mag).all(), float(np.abs(got - ref).max())


def test_resblock_time_embedding():
    """A 320->640 ResBlock whose time embedding changes every step (as a denoising loop's
    timestep does): sync, then two displaced steps of a drifting input."""
    wl = synth.Workload(name="resblock_temb_320to640x64x64", kind="resblock", C=320, Cout=640,
                        H=64, W=64, P=4)
    Ct = 1280
    wts = synth.make_weights(wl, random_affine=True)
    g = torch.Generator().manual_seed(5)
    wts["temb_w"] = torch.randn(wl.cout, Ct, generator=g) * Ct ** -0.5
    wts["temb_b"] = torch.randn(wl.cout, generator=g) * 0.3
    dev_w = block_weights("resblock", wts, torch.bfloat16)
    blk = B.Block(B.RESBLOCK, wl.H, wl.W, wl.C, wl.cout, wl.G, wl.P, 0, B.BF16, True, wl.eps, 1.0,
                  temb_dim=Ct)
    assert len(dev_w) + 1 == B.dp_block_weight_count(blk.desc)
    w64 = {n: v.double().numpy() for n, v in wts.items()}
    xs = synth.InputStream(wl)
    st = {}
    for k, mode in enumerate([B.SYNC, B.DISPLACED, B.DISPLACED]):
        temb = torch.randn(Ct, generator=g) * 2.0
        x = xs.x(k)[0].double().numpy()
        out = torch.empty(wl.H, wl.W, wl.cout, dtype=torch.bfloat16, device="cuda")
        blk.step(dev_img(x, "bf16"), out, dev_w + [temb.cuda()], mode)
        ref = O.resblock_step(st, x, w64, wl.P, wl.G, wl.eps, 1.0, mode, "bf16", final_storage="none",
                              temb=temb.double().numpy())
        torch.cuda.synchronize()
        check(host_img(out), ref, what=f"temb resblock step {k} mode {mode}", storage_rel=BF16_HALF_ULP,
              scale_rel=2.0 ** -7)
    assert B.dp_device_status() == 0
