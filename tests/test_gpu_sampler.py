"""GPU parity of the sampler update (dp_ddim_step) and of a DDIM-shaped step loop.

The kernel is compared element by element with the oracle's deterministic DDIM step on the
same inputs, for both storage types, ragged lengths and in-place use.  The loop runs a
displaced GroupNorm + conv block as the noise estimator of a few sampler steps (sync warm-up,
then displaced), updating the latent in place on the GPU and in the oracle from the same
seeded start, and compares the latent after every step.
"""
import math

import numpy as np
import pytest
import torch

from displaced_patch_parallelism_b200 import binding as B
from displaced_patch_parallelism_b200 import synth
from displaced_patch_parallelism_b200.weights import block_weights
from oracle import dp_oracle as O
from tests.helpers import F32_ATOL, F32_RL2, check, dev_img, host_img

pytestmark = pytest.mark.gpu


def coef_magnitude(x, e, abar_t, abar_prev):
    """|ca x| + |ce e| with the update's two coefficients written out: the scale of the fp32
    rounding of each output."""
    ca = math.sqrt(abar_prev / abar_t)
    ce = abs(math.sqrt(1 - abar_prev)) + math.sqrt(abar_prev * (1 - abar_t) / abar_t)
    return ca * np.abs(x) + ce * np.abs(e)


@pytest.mark.parametrize("dtype", [B.BF16, B.FP32], ids=["bf16", "fp32"])
@pytest.mark.parametrize("n", [1, 7, 12345, (1 << 22) + 3])
@pytest.mark.parametrize("in_place", [False, True], ids=["out", "inplace"])
def test_ddim_step_kernel(dtype, n, in_place):
    """fp32: within 2^-21 of |ca x| + |ce e| (a few roundings of fp32 coefficients, one FMA);
    bf16: one bf16 ulp of the result on top of that."""
    g = torch.Generator().manual_seed(n + 2 * in_place + dtype)
    tdt = torch.bfloat16 if dtype == B.BF16 else torch.float32
    x = (torch.randn(n, generator=g) * 1.5).to(tdt)
    e = torch.randn(n, generator=g).to(tdt)
    x64, e64 = x.double().numpy(), e.double().numpy()
    for abar_t, abar_prev in [synth.ddim_alpha_bars()[0], synth.ddim_alpha_bars()[30],
                              synth.ddim_alpha_bars()[-1]]:
        xd, ed = x.cuda(), e.cuda()
        y = xd if in_place else torch.full_like(xd, float("nan"))
        B.dp_ddim_step(xd, ed, y, n, abar_t, abar_prev, dtype)
        torch.cuda.synchronize()
        got = y.cpu().double().numpy()
        ref = O.ddim_step(x64, e64, abar_t, abar_prev)
        bound = 2.0 ** -21 * coef_magnitude(x64, e64, abar_t, abar_prev)
        if dtype == B.BF16:
            bound = bound + 2.0 ** -8 * np.abs(ref)
        assert np.isfinite(got).all()
        worst = float(np.max(np.abs(got - ref) - bound))
        assert worst <= 0, (abar_t, abar_prev, worst)


def test_ddim_loop_with_displaced_block():
    """Four sampler steps of the 64-channel fp32 GroupNorm + conv block used as the noise
    estimator, one warm-up step, the latent updated in place; the GPU's latent after every
    step against the oracle's (each side feeds its own latent to the next step)."""
    wl = synth.WORKLOADS["tiny_fp32_gn_conv"]
    wts = synth.make_weights(wl, random_affine=True)
    dev_w = block_weights(wl.kind, wts, torch.float32)
    w64 = {n: v.double().numpy() for n, v in wts.items()}
    blk = B.Block(B.GN_CONV, wl.H, wl.W, wl.C, wl.cout, wl.G, wl.P, 0, B.FP32, wl.silu, wl.eps, 1.0)
    x = synth.InputStream(wl).x(0)[0].double().numpy()
    xd = dev_img(x, "fp32")
    eps_d = torch.empty_like(xd)
    st = {}
    for k, (abar_t, abar_prev) in enumerate(synth.ddim_alpha_bars()[:4]):
        mode = B.dp_mode_for_step(k, 1)
        blk.step(xd, eps_d, dev_w, mode)
        B.dp_ddim_step(xd, eps_d, xd, xd.numel(), abar_t, abar_prev, B.FP32)
        eps = O.block_step(wl.kind, st, x, w64, wl.P, wl.G, wl.eps, 1.0, mode, "fp32", silu=wl.silu,
                           final_storage="none")
        x = O.ddim_step(x, eps, abar_t, abar_prev)
        torch.cuda.synchronize()
        check(host_img(xd), x, atol=F32_ATOL, rl2=F32_RL2, what=f"ddim loop step {k} mode {mode}")
    assert B.dp_device_status() == 0
