"""The GroupNorm entry point that allocates nothing, against the workspace one and the oracle.

dp_groupnorm_async_noalloc serves callers that cannot allocate device memory
(code that must not trigger cudaMalloc's device synchronisation, hosts with a
fixed memory budget, C callers without an allocator).  It keeps its scratch in
a fixed array inside the library instead of a caller workspace.  This file is
named so that pytest collects it last: if it fails, a run that stops at the
first failure has already run every other test.  It also passes on its own in
a fresh process, because the library sets its scratch up on the first call.
"""
import numpy as np
import pytest
import torch

from displaced_patch_parallelism_b200 import binding as B
from oracle import dp_oracle as O
from tests.helpers import BF16_HALF_ULP, STATS_ATOL, check, dev_f32, dev_img, host, host_img, rounded

pytestmark = pytest.mark.gpu


def _inputs(seed, C, H, W, P, G):
    r = np.random.default_rng(seed)
    xs = rounded(r.standard_normal((C, H, W)), "bf16")
    x = rounded(xs + 0.05 * r.standard_normal((C, H, W)), "bf16")
    sg, sl = O.refresh_stats(O.gn_fresh_local(xs, P, G))
    return x, 1 + 0.3 * r.standard_normal(C), 0.3 * r.standard_normal(C), sg, sl


def test_groupnorm_noalloc_matches_workspace_call_twice_in_a_row():
    C, H, W, P, G = 320, 64, 48, 4, 32
    for call, (seed, mode) in enumerate([(11, B.DISPLACED), (12, B.SYNC)]):
        x, gamma, beta, sg, sl = _inputs(seed, C, H, W, P, G)
        xd = dev_img(x, "bf16")
        args = (dev_f32(gamma), dev_f32(beta), H, W, C, G, P, 1e-5, 1.0, 1, mode, B.BF16,
                dev_f32(sg), dev_f32(sl))
        # existing entry point, with a caller-allocated workspace
        y_ref = torch.empty_like(xd)
        f_ref = torch.zeros(P * G * 2, device="cuda")
        u_ref = torch.zeros(P * G * 2, device="cuda")
        ws = torch.zeros(B.dp_groupnorm_workspace_size(H, W, C, G, P), dtype=torch.uint8,
                         device="cuda")
        B.dp_groupnorm_async(xd, y_ref, *args, f_ref, u_ref, ws)
        # the entry point without a workspace
        y = torch.empty_like(xd)
        f = torch.zeros(P * G * 2, device="cuda")
        u = torch.zeros(P * G * 2, device="cuda")
        B.dp_groupnorm_async_noalloc(xd, y, *args, f, u)
        torch.cuda.synchronize()
        np.testing.assert_allclose(host(f), host(f_ref), rtol=0, atol=STATS_ATOL)
        np.testing.assert_allclose(host(u), host(u_ref), rtol=0, atol=STATS_ATOL)
        check(host_img(y), host_img(y_ref), what=f"noalloc call {call}", storage_rel=BF16_HALF_ULP)
        # and against the oracle itself: output, fresh moments and the moments used
        f32 = lambda a: np.asarray(a, dtype=np.float32).astype(np.float64)   # as the device holds them
        y_o, f_o, u_o, _ = O.groupnorm_async(x, f32(gamma), f32(beta), P, G, 1e-5, 1.0, True, mode,
                                             f32(sg), f32(sl))
        np.testing.assert_allclose(host(f), f_o.reshape(-1), rtol=0, atol=STATS_ATOL)
        np.testing.assert_allclose(host(u), u_o.reshape(-1), rtol=0, atol=STATS_ATOL)
        check(host_img(y), y_o, what=f"noalloc call {call} vs oracle", storage_rel=BF16_HALF_ULP)
    assert B.dp_device_status() == 0


def test_groupnorm_noalloc_rejects_oversized_requests():
    with pytest.raises(B.DPError) as e:
        # P * G = 8 * 512 = 4096 is a valid GroupNorm but needs 512 KiB of scratch
        B.dp_groupnorm_async_noalloc(16, 32, 16, 16, 8, 8, 1024, 512, 8, 1e-5, 1.0, 1, B.SYNC,
                                     B.BF16, None, None, 16, 16)
    assert e.value.code == B.DP_ERR_UNSUPPORTED
    assert "static scratch" in B.lib().dp_last_error().decode()
