"""GPU parity of the multistep second-order DPM-Solver++ update (dp_dpm_solver_step) against
the oracle: the kernel at several lengths and both storage types, its first-order, second-order
and final-step forms, and a four-step sampler loop with the fp32 GroupNorm + conv block as the
noise estimator (one warm-up step, then displaced steps)."""
import numpy as np
import pytest
import torch

from displaced_patch_parallelism_b200 import binding as B
from displaced_patch_parallelism_b200 import synth
from displaced_patch_parallelism_b200.weights import block_weights
from oracle import dp_oracle as O
from tests.helpers import F32_ATOL, F32_RL2, check, dev_img, host_img, rounded

pytestmark = pytest.mark.gpu


def _levels(k):
    """(abar_prev, abar_s, abar_t) of sampler step k of a 10-step schedule (abar_prev = 0 at k = 0)."""
    ab = synth.ddim_alpha_bars(10)
    abar_s, abar_t = ab[k]
    return (ab[k - 1][0] if k > 0 else 0.0), abar_s, abar_t


@pytest.mark.parametrize("n", [8, 1000, 4096 * 320 + 5])
@pytest.mark.parametrize("dtype", [B.BF16, B.FP32], ids=["bf16", "fp32"])
@pytest.mark.parametrize("k", [0, 3, 9], ids=["first-order", "second-order", "final"])
def test_dpm_solver_step(n, dtype, k):
    """x_next and the data prediction left in x0_buf, against the oracle on the values the
    kernel stores.  fp32: within 2^-20 of the terms' magnitudes (three fp32 FMAs with
    coefficients rounded to fp32); bf16: the output's storage rounding (half an ulp) on top."""
    abar_prev, abar_s, abar_t = _levels(k)
    r = np.random.default_rng(n + k)
    s = "bf16" if dtype == B.BF16 else "fp32"
    x = rounded(r.standard_normal(n) * 3.0, s)
    e = rounded(r.standard_normal(n), s)
    x0p = rounded(r.standard_normal(n) * 2.0, s)
    tdt = torch.bfloat16 if dtype == B.BF16 else torch.float32
    xd = torch.from_numpy(x.astype(np.float32)).to(tdt).cuda()
    ed = torch.from_numpy(e.astype(np.float32)).to(tdt).cuda()
    x0d = torch.from_numpy(x0p.astype(np.float32)).to(tdt).cuda() if k > 0 else \
        torch.full((n,), float("nan"), dtype=tdt, device="cuda")   # a first-order step ignores it
    out = torch.empty_like(xd)
    B.dp_dpm_solver_step(xd, ed, x0d, out, n, abar_prev, abar_s, abar_t, dtype)
    torch.cuda.synchronize()
    want, want_x0 = O.dpm_solver_2m_step(x, e, x0p if k > 0 else None, abar_prev, abar_s, abar_t)
    got = out.float().cpu().double().numpy()
    got_x0 = x0d.float().cpu().double().numpy()
    scale = np.abs(x) / np.sqrt(abar_s) + np.abs(e) * np.sqrt(1 - abar_s) / np.sqrt(abar_s) + 3 * np.abs(x0p)
    tol = 2.0 ** -20 * scale + (2.0 ** -8 if dtype == B.BF16 else 0.0) * np.abs(want)
    assert np.isfinite(got).all() and np.isfinite(got_x0).all()
    assert (np.abs(got - want) <= tol + 1e-30).all(), float(np.max(np.abs(got - want) - tol))
    tol0 = 2.0 ** -20 * scale + (2.0 ** -8 if dtype == B.BF16 else 0.0) * np.abs(want_x0)
    assert (np.abs(got_x0 - want_x0) <= tol0 + 1e-30).all(), float(np.max(np.abs(got_x0 - want_x0) - tol0))


def test_dpm_solver_in_place():
    n = 4096
    abar_prev, abar_s, abar_t = _levels(4)
    r = np.random.default_rng(7)
    x, e, x0p = (r.standard_normal(n) for _ in range(3))
    xd = torch.from_numpy(x.astype(np.float32)).cuda()
    ed = torch.from_numpy(e.astype(np.float32)).cuda()
    x0d = torch.from_numpy(x0p.astype(np.float32)).cuda()
    want, _ = O.dpm_solver_2m_step(x.astype(np.float32), e.astype(np.float32), x0p.astype(np.float32),
                                   abar_prev, abar_s, abar_t)
    B.dp_dpm_solver_step(xd, ed, x0d, xd, n, abar_prev, abar_s, abar_t, B.FP32)
    torch.cuda.synchronize()
    np.testing.assert_allclose(xd.cpu().double().numpy(), want, rtol=0, atol=1e-5)


def test_dpm_solver_loop_with_displaced_block():
    """Four steps of a 10-step DPM-Solver++ schedule with the 64-channel fp32 GroupNorm + conv
    block as the noise estimator, one synchronous warm-up step, the latent updated in place:
    the GPU's latent after every step against the oracle's (each side feeds its own latent on)."""
    wl = synth.WORKLOADS["tiny_fp32_gn_conv"]
    wts = synth.make_weights(wl, random_affine=True)
    dev_w = block_weights(wl.kind, wts, torch.float32)
    w64 = {n_: v.double().numpy() for n_, v in wts.items()}
    blk = B.Block(B.GN_CONV, wl.H, wl.W, wl.C, wl.cout, wl.G, wl.P, 0, B.FP32, wl.silu, wl.eps, 1.0)
    x = synth.InputStream(wl).x(0)[0].double().numpy()
    xd = dev_img(x, "fp32")
    eps_d = torch.empty_like(xd)
    x0_d = torch.empty_like(xd)
    st, x0_prev = {}, None
    for k in range(4):
        abar_prev, abar_s, abar_t = _levels(k)
        mode = B.dp_mode_for_step(k, 1)
        blk.step(xd, eps_d, dev_w, mode)
        B.dp_dpm_solver_step(xd, eps_d, x0_d, xd, xd.numel(), abar_prev, abar_s, abar_t, B.FP32)
        eps = O.block_step(wl.kind, st, x, w64, wl.P, wl.G, wl.eps, 1.0, mode, "fp32", silu=wl.silu,
                           final_storage="none")
        x, x0_prev = O.dpm_solver_2m_step(x, eps, x0_prev, abar_prev, abar_s, abar_t)
        torch.cuda.synchronize()
        check(host_img(xd), x, atol=F32_ATOL, rl2=F32_RL2, what=f"dpm loop step {k} mode {mode}")
    assert blk.status() == 0 and B.dp_device_status() == 0
