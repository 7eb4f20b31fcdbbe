"""Failure detection on the GPU without a fault: every pipeline wait in the library's
kernels is bounded, and a wait that runs out records DP_ERR_TIMEOUT and lets the kernel
return.  dp_selftest_bounded_wait runs the library's own bounded-wait code on a wait that
nothing ends (an mbarrier no thread arrives at; a global flag no thread writes) with a
limit of a few hundred microseconds; the status must come back as DP_ERR_TIMEOUT, the read
must clear it, and the context must stay usable for the next normal call.  Block steps
report into their own state's word, separate from the library's."""
import numpy as np
import pytest
import torch

from displaced_patch_parallelism_b200 import binding as B
from displaced_patch_parallelism_b200 import synth
from displaced_patch_parallelism_b200.weights import block_weights
from oracle import dp_oracle as O
from tests.helpers import BF16_HALF_ULP, check, dev_f32, dev_img, host_img, rounded

pytestmark = pytest.mark.gpu


def _groupnorm_against_oracle(seed=5):
    """One ordinary sync GroupNorm call, checked against the oracle."""
    C, H, W, P, G = 64, 16, 16, 2, 32
    r = np.random.default_rng(seed)
    x = rounded(r.standard_normal((C, H, W)), "bf16")
    gamma = np.float32(1 + 0.3 * r.standard_normal(C)).astype(np.float64)
    beta = np.float32(0.3 * r.standard_normal(C)).astype(np.float64)
    xd = dev_img(x, "bf16")
    y = torch.empty_like(xd)
    f = torch.zeros(P * G * 2, device="cuda")
    u = torch.zeros(P * G * 2, device="cuda")
    ws = torch.zeros(B.dp_groupnorm_workspace_size(H, W, C, G, P), dtype=torch.uint8, device="cuda")
    B.dp_groupnorm_async(xd, y, dev_f32(gamma), dev_f32(beta), H, W, C, G, P, 1e-5, 1.0, 1, B.SYNC,
                         B.BF16, None, None, f, u, ws)
    torch.cuda.synchronize()
    ref, *_ = O.groupnorm_async(x, gamma, beta, P, G, 1e-5, 1.0, True, B.SYNC, None, None)
    check(host_img(y), ref, what="groupnorm after a timeout", storage_rel=BF16_HALF_ULP)


@pytest.mark.parametrize("kind", [B.SELFTEST_WAIT_MBARRIER, B.SELFTEST_WAIT_FLAG],
                         ids=["mbarrier", "flag"])
def test_bounded_wait_runs_out_and_reports_timeout(kind):
    assert B.dp_device_status() == B.DP_OK
    B.dp_selftest_bounded_wait(kind, 300)
    assert B.dp_device_status() == B.DP_ERR_TIMEOUT
    assert B.dp_device_status() == B.DP_OK          # the read cleared it
    _groupnorm_against_oracle()                      # the context is still usable
    assert B.dp_device_status() == B.DP_OK


def test_block_steps_report_into_their_own_state():
    """A timeout recorded in the library's word does not show in a block's word, and a block
    that completed its steps reads DP_OK."""
    wl = synth.Workload(name="gn_conv_64x16x16", kind="gn_conv", C=64, H=16, W=16, P=2)
    wts = synth.make_weights(wl, random_affine=True)
    dw = block_weights(wl.kind, wts, torch.bfloat16)
    blocks = [B.Block(B.GN_CONV, wl.H, wl.W, wl.C, wl.cout, wl.G, wl.P, 0, B.BF16, 1, wl.eps, 1.0)
              for _ in range(2)]
    x = synth.nchw_to_nhwc(synth.InputStream(wl).x(0)).to(torch.bfloat16).cuda()
    out = torch.empty_like(x)
    for blk in blocks:
        blk.step(x, out, dw, B.SYNC)
    B.dp_selftest_bounded_wait(B.SELFTEST_WAIT_FLAG, 200)
    assert [blk.status() for blk in blocks] == [B.DP_OK, B.DP_OK]
    assert B.dp_device_status() == B.DP_ERR_TIMEOUT
    assert B.dp_device_status() == B.DP_OK
