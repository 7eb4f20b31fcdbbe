"""Block-step parity on the five synthetic workloads' shapes, through dp_block_step.

Each test runs a short step chain (sync warm-up, then displaced; or naive
first for zero warm-up) on the GPU and in the oracle from the same seeded
inputs, and compares every step's block output.  The 320x480x480 workload is
checked on sampled output rows (band edges and interiors), which the oracle
computes one row at a time.
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
KIND = {"gn_conv": B.GN_CONV, "resblock": B.RESBLOCK, "attn": B.ATTN}


def make_block(wl):
    return B.Block(KIND[wl.kind], wl.H, wl.W, wl.C, wl.cout, wl.G, wl.P, wl.heads,
                   B.BF16 if wl.dtype == "bf16" else B.FP32, wl.silu, wl.eps, 1.0)


def run_chain(wl, modes, random_affine, storage_rel=0.0):
    wts = synth.make_weights(wl, random_affine=random_affine)
    tdt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    dev_w = block_weights(wl.kind, wts, tdt)
    blk = make_block(wl)
    xs = synth.InputStream(wl)
    st = {}
    for k, mode in enumerate(modes):
        x = xs.x(k)[0].double().numpy()
        xd = dev_img(x, wl.dtype)
        out = torch.empty(wl.H, wl.W, wl.cout, dtype=tdt, device="cuda")
        blk.step(xd, out, dev_w, mode)
        ref = O.block_step(wl.kind, st, x, {n: v.double().numpy() for n, v in wts.items()}, wl.P,
                           wl.G, wl.eps, 1.0, mode, wl.dtype, heads=wl.heads, silu=wl.silu,
                           final_storage="none")
        torch.cuda.synchronize()
        check(host_img(out), ref, what=f"{wl.name} step {k} mode {mode}", storage_rel=storage_rel)
    assert B.dp_device_status() == 0


@pytest.mark.parametrize("random_affine", [False, True])
def test_tiny_fp32_gn_conv(random_affine):
    wl = synth.WORKLOADS["tiny_fp32_gn_conv"]
    run_chain(wl, [B.SYNC, B.DISPLACED], random_affine)


def test_resblock_320x128x128():
    wl = synth.WORKLOADS["resblock_320x128x128"]
    run_chain(wl, [B.SYNC, B.DISPLACED, B.DISPLACED], True)


def test_resblock_zero_warmup():
    wl = synth.WORKLOADS["resblock_320x128x128"]
    run_chain(wl, [B.NAIVE, B.DISPLACED], False)


def test_resblock_channel_change():
    wl = synth.Workload(name="resblock_320to640x64x64", kind="resblock", C=320, Cout=640, H=64, W=64,
                        P=4)
    run_chain(wl, [B.SYNC, B.DISPLACED], True, storage_rel=BF16_HALF_ULP)


def test_attn_640x64x64():
    wl = synth.WORKLOADS["attn_640x64x64"]
    run_chain(wl, [B.SYNC, B.DISPLACED], True)


def test_attn_1280x32x32_zero_warmup():
    wl = synth.Workload(name="attn_1280x32x32", kind="attn", C=1280, H=32, W=32, P=4, heads=20,
                        silu=False)
    run_chain(wl, [B.NAIVE, B.DISPLACED, B.SYNC], True, storage_rel=BF16_HALF_ULP)


def test_gn_conv_320x480x480_sampled_rows():
    wl = synth.WORKLOADS["gn_conv_320x480x480"]
    wts = synth.make_weights(wl, random_affine=True)
    dev_w = block_weights(wl.kind, wts, torch.bfloat16)
    W64 = {n: v.double().numpy() for n, v in wts.items()}
    blk = make_block(wl)
    xs = synth.InputStream(wl)
    rows = [0, 1, 58, 59, 60, 61, 120, 299, 300, 420, 478, 479]
    gn = O.GNState()
    a_prev = None
    for k, mode in enumerate([B.SYNC, B.DISPLACED]):
        x = xs.x(k)[0].double().numpy()
        out = torch.empty(wl.H, wl.W, wl.C, dtype=torch.bfloat16, device="cuda")
        blk.step(dev_img(x, "bf16"), out, dev_w, mode)
        a, f, used, _ = O.groupnorm_async(x, W64["gn_gamma"], W64["gn_beta"], wl.P, wl.G, wl.eps, 1.0,
                                          True, mode, gn.stale_global, gn.stale_local)
        a = O.store(a, "bf16")
        ref = O.conv3x3_halo_rows(a, a_prev, W64["conv_w"], W64["conv_b"], wl.P, mode, rows)
        torch.cuda.synchronize()
        got = out[rows].float().cpu().permute(2, 0, 1).double().numpy()
        check(got, ref, what=f"gn_conv 480 step {k}")
        gn.refresh(f)
        a_prev = a


def test_displaced_before_any_step_is_a_state_error():
    wl = synth.WORKLOADS["tiny_fp32_gn_conv"]
    wts = synth.make_weights(wl)
    blk = make_block(wl)
    x = torch.zeros(wl.H, wl.W, wl.C, device="cuda")
    out = torch.empty_like(x)
    with pytest.raises(B.DPError) as e:
        blk.step(x, out, block_weights(wl.kind, wts, torch.float32), B.DISPLACED)
    assert e.value.code == B.DP_ERR_STATE
