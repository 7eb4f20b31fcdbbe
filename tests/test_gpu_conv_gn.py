"""GPU parity of the GroupNorm -> 3x3 conv pair run as dp_groupnorm_stats + dp_conv3x3_halo_gn
(the conv normalises its own input tiles), against the oracle's GroupNorm and halo conv.

Cases cover the three modes, widths that are and are not multiples of the 128-column tile,
output widths of one 160-column tile pair slice, two (320) and three n tiles (480), with and
without SiLU and a residual.  The normalised band-edge rows the call writes to a_next (the next
step's stale rows) are checked against the oracle's normalised input, and every other row of
a_next is checked to be untouched.
"""
import numpy as np
import pytest
import torch

from displaced_patch_parallelism_b200 import binding as B
from oracle import dp_oracle as O
from tests.helpers import (BF16_HALF_ULP, STATS_ATOL, check, conv_w_dev, dev_f32, dev_img, host,
                           host_img, rounded)

pytestmark = pytest.mark.gpu

CASES = [
    # H, W, Cin, Cout, P, mode, silu, residual
    (16, 128, 64, 160, 2, B.SYNC, 1, False),
    (16, 128, 64, 160, 2, B.DISPLACED, 1, True),
    (16, 128, 64, 160, 2, B.NAIVE, 1, False),
    (24, 200, 128, 320, 4, B.DISPLACED, 1, True),
    (24, 200, 128, 320, 4, B.SYNC, 0, False),
    (8, 256, 320, 320, 2, B.DISPLACED, 1, False),
    (8, 160, 64, 480, 2, B.DISPLACED, 1, True),
    (12, 384, 64, 160, 3, B.NAIVE, 0, True),
    (9, 128, 64, 160, 3, B.DISPLACED, 1, False),      # odd tile count: a pair's second tile is empty
]


@pytest.mark.parametrize("H,W,Cin,Cout,P,mode,silu,with_res", CASES)
def test_groupnorm_conv_parity(H, W, Cin, Cout, P, mode, silu, with_res):
    G, eps = 32, 1e-5
    r = np.random.default_rng(H * 1000 + W + Cout + mode)
    f32 = lambda a: np.asarray(a, dtype=np.float32).astype(np.float64)
    x_prev = rounded(r.standard_normal((Cin, H, W)), "bf16")
    x = rounded(x_prev + 0.05 * r.standard_normal((Cin, H, W)), "bf16")
    gamma, beta = f32(1 + 0.3 * r.standard_normal(Cin)), f32(0.3 * r.standard_normal(Cin))
    wt = rounded(r.standard_normal((Cout, Cin, 3, 3)) * np.sqrt(2.0 / (9 * Cin)), "bf16")
    bias = f32(0.3 * r.standard_normal(Cout))
    res = rounded(r.standard_normal((Cout, H, W)), "bf16") if with_res else None
    # the previous step: its statistics and its normalised activations (the stale buffer)
    a_prev, f_prev, _, _ = O.groupnorm_async(x_prev, gamma, beta, P, G, eps, 1.0, bool(silu), B.SYNC,
                                             None, None)
    a_prev = O.store(a_prev, "bf16")
    sg, sl = (f32(v) for v in O.refresh_stats(f_prev))

    xd = dev_img(x, "bf16")
    used = torch.zeros(P * G * 2, device="cuda")
    fresh = torch.zeros(P * G * 2, device="cuda")
    ws = torch.zeros(B.dp_groupnorm_workspace_size(H, W, Cin, G, P), dtype=torch.uint8, device="cuda")
    B.dp_groupnorm_stats(xd, H, W, Cin, G, P, 1.0, mode, B.BF16, dev_f32(sg), dev_f32(sl), fresh, used,
                         ws)
    a_next = torch.full((H, W, Cin), float("nan"), dtype=torch.bfloat16, device="cuda")
    out = torch.empty(H, W, Cout, dtype=torch.bfloat16, device="cuda")
    B.dp_conv3x3_halo_gn(xd, dev_img(a_prev, "bf16"), a_next, used, dev_f32(gamma), dev_f32(beta), G, eps,
                         silu, conv_w_dev(wt, "bf16"), dev_f32(bias),
                         dev_img(res, "bf16") if with_res else None, out, H, W, Cin, Cout, P, mode)
    torch.cuda.synchronize()

    a, f, u, _ = O.groupnorm_async(x, gamma, beta, P, G, eps, 1.0, bool(silu), mode, sg, sl)
    np.testing.assert_allclose(host(fresh), f.reshape(-1), rtol=0, atol=STATS_ATOL)
    np.testing.assert_allclose(host(used), u.reshape(-1), rtol=0, atol=STATS_ATOL)
    a = O.store(a, "bf16")
    ref = O.conv3x3_halo(a, a_prev, wt, bias, res, P, mode)
    check(host_img(out), ref, what=f"conv_gn {H}x{W} {Cin}->{Cout} P={P} mode={mode}",
          storage_rel=BF16_HALF_ULP)
    # a_next: the first and last row of every band, normalised; nothing else written
    hb = H // P
    edge = sorted({p * hb for p in range(P)} | {p * hb + hb - 1 for p in range(P)})
    got = host_img(a_next)
    check(got[:, edge], a[:, edge], what="a_next edge rows", storage_rel=BF16_HALF_ULP)
    other = [i for i in range(H) if i not in edge]
    assert np.isnan(got[:, other]).all(), "a_next rows other than band edges were written"
    assert B.dp_device_status() == 0


def test_groupnorm_conv_without_next_buffer():
    """a_next may be NULL: the conv alone, against the oracle."""
    H, W, Cin, Cout, P, G = 8, 128, 64, 160, 2, 32
    r = np.random.default_rng(3)
    x = rounded(r.standard_normal((Cin, H, W)), "bf16")
    wt = rounded(r.standard_normal((Cout, Cin, 3, 3)) * 0.06, "bf16")
    gamma, beta = np.ones(Cin), np.zeros(Cin)
    xd = dev_img(x, "bf16")
    used = torch.zeros(P * G * 2, device="cuda")
    fresh = torch.zeros(P * G * 2, device="cuda")
    ws = torch.zeros(B.dp_groupnorm_workspace_size(H, W, Cin, G, P), dtype=torch.uint8, device="cuda")
    B.dp_groupnorm_stats(xd, H, W, Cin, G, P, 1.0, B.SYNC, B.BF16, None, None, fresh, used, ws)
    out = torch.empty(H, W, Cout, dtype=torch.bfloat16, device="cuda")
    B.dp_conv3x3_halo_gn(xd, None, None, used, dev_f32(gamma), dev_f32(beta), G, 1e-5, 1,
                         conv_w_dev(wt, "bf16"), None, None, out, H, W, Cin, Cout, P, B.SYNC)
    torch.cuda.synchronize()
    a, *_ = O.groupnorm_async(x, gamma, beta, P, G, 1e-5, 1.0, True, B.SYNC, None, None)
    ref = O.conv3x3_halo(O.store(a, "bf16"), None, wt, None, None, P, B.SYNC)
    check(host_img(out), ref, what="conv_gn without a_next", storage_rel=BF16_HALF_ULP)
