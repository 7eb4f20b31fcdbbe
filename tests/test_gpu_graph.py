"""Block steps replayed as CUDA graphs (dp_block_graph_*) against the same steps launched one
by one: two states of one descriptor take the same inputs (copied into the captured input
buffer before each launch) and must give the same bits, step after step, with the parity and
step count advancing as dp_block_step advances them."""
import numpy as np
import pytest
import torch

from displaced_patch_parallelism_b200 import binding as B
from displaced_patch_parallelism_b200 import synth
from displaced_patch_parallelism_b200.weights import block_weights, unet_sdxl_weights

pytestmark = pytest.mark.gpu


def _cases():
    res = synth.Workload(name="g_res", kind="resblock", C=320, H=64, W=64, P=4, Cout=640)
    tf = synth.Workload(name="g_tf", kind="transformer", C=320, H=32, W=32, P=4, heads=5, silu=False,
                        ctx_len=77, ctx_dim=128, ff_inner=1280, depth=2)
    un = synth.Workload(name="g_unet", kind="unet_sdxl", C=4, H=64, W=64, P=2, base=64, depths=(0, 1, 1),
                        ctx_len=77, ctx_dim=128, temb_dim=128)
    return {"resblock": res, "transformer": tf, "unet_sdxl": un}


def _setup(wl):
    wts = synth.make_weights(wl, random_affine=True)
    kind = {"resblock": B.RESBLOCK, "transformer": B.TRANSFORMER, "unet_sdxl": B.UNET_SDXL}[wl.kind]
    kw = {}
    if wl.kind == "transformer":
        dw = block_weights("transformer", wts, depth=wl.depth) + [synth.context(wl).to(torch.bfloat16).cuda()]
        kw = dict(context=(wl.ctx_len, wl.ctx_dim, wl.ff_inner), depth=wl.depth, context_fixed=True)
    elif wl.kind == "unet_sdxl":
        dw = unet_sdxl_weights(wts, synth.sdxl_unet_stages(wl.base, wl.depths), wl.depths)
        dw += [synth.context(wl).to(torch.bfloat16).cuda(), synth.randn((wl.temb_dim,), 5).cuda()]
        kw = dict(context=(wl.ctx_len, wl.ctx_dim, 0), temb_dim=wl.temb_dim, unet=(wl.base,) + wl.depths,
                  context_fixed=True)
    else:
        dw = block_weights("resblock", wts)

    def make():
        return B.Block(kind, wl.H, wl.W, wl.C, wl.cout, wl.G, wl.P, wl.heads, B.BF16, wl.silu, wl.eps, 1.0, **kw)
    return dw, make


@pytest.mark.parametrize("name", ["resblock", "transformer", "unet_sdxl"])
def test_graph_steps_equal_plain_steps(name):
    wl = _cases()[name]
    dw, make = _setup(wl)
    xs = synth.InputStream(wl)
    xin = [synth.nchw_to_nhwc(xs.x(k)).to(torch.bfloat16).cuda() for k in range(5)]
    Ho, Wo, Co = wl.H, wl.W, wl.cout
    plain, replay = make(), make()
    out_p = torch.empty(Ho, Wo, Co, dtype=torch.bfloat16, device="cuda")
    out_g = torch.empty_like(out_p)
    xbuf = torch.empty_like(xin[0])
    plain.step(xin[0], out_p, dw, B.SYNC)
    xbuf.copy_(xin[0])
    replay.step(xbuf, out_g, dw, B.SYNC)
    torch.cuda.synchronize()
    assert torch.equal(out_p, out_g)
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        graph = replay.graph(xbuf, out_g, dw, B.DISPLACED, stream)
        for k in range(1, 5):
            plain.step(xin[k], out_p, dw, B.DISPLACED, stream)
            xbuf.copy_(xin[k])
            cur = replay.state.cur
            graph.launch(stream)
            assert replay.state.cur == cur ^ 1 and replay.state.steps_done == k + 1
            stream.synchronize()
            assert torch.equal(out_p, out_g), f"{name}: step {k} differs"
    graph.close()
    assert plain.status() == 0 and replay.status() == 0 and B.dp_device_status() == 0


def test_graph_runs_only_on_its_own_state():
    wl = _cases()["resblock"]
    dw, make = _setup(wl)
    a, b = make(), make()
    x = synth.nchw_to_nhwc(synth.InputStream(wl).x(0)).to(torch.bfloat16).cuda()
    out = torch.empty(wl.H, wl.W, wl.cout, dtype=torch.bfloat16, device="cuda")
    stream = torch.cuda.Stream()
    with pytest.raises(B.DPError) as e:
        a.graph(x, out, dw, B.SYNC, stream)          # before the state's first step
    assert e.value.code == B.DP_ERR_STATE
    a.step(x, out, dw, B.SYNC)
    b.step(x, out, dw, B.SYNC)
    g = a.graph(x, out, dw, B.DISPLACED, stream)
    with pytest.raises(B.DPError) as e:
        B.dp_block_graph_launch(g.handle, b.state, stream)
    assert e.value.code == B.DP_ERR_INVALID_ARG
    g.launch(stream)
    stream.synchronize()
    g.close()
    assert a.status() == 0


@pytest.mark.parametrize("name", ["resblock_320x128x128", "tiny_fp32_gn_conv"])
def test_sync_graph_steps_equal_plain_steps(name):
    """Graphs of sync steps (whose GroupNorm takes the grid-wide cooperative single pass) capture
    and replay the plain steps' bits, in bf16 and in fp32."""
    wl = synth.WORKLOADS[name]
    tdt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    dw = block_weights(wl.kind, synth.make_weights(wl, random_affine=True), tdt)
    kind = {"resblock": B.RESBLOCK, "gn_conv": B.GN_CONV}[wl.kind]

    def make():
        return B.Block(kind, wl.H, wl.W, wl.C, wl.cout, wl.G, wl.P, 0, B.BF16 if wl.dtype == "bf16" else B.FP32,
                       wl.silu, wl.eps, 1.0)
    xs = synth.InputStream(wl)
    xin = [synth.nchw_to_nhwc(xs.x(k)).to(tdt).cuda() for k in range(4)]
    plain, replay = make(), make()
    out_p = torch.empty(wl.H, wl.W, wl.cout, dtype=tdt, device="cuda")
    out_g = torch.empty_like(out_p)
    xbuf = xin[0].clone()
    plain.step(xin[0], out_p, dw, B.SYNC)
    replay.step(xbuf, out_g, dw, B.SYNC)
    torch.cuda.synchronize()
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        graph = replay.graph(xbuf, out_g, dw, B.SYNC, stream)
        for k in range(1, 4):
            plain.step(xin[k], out_p, dw, B.SYNC, stream)
            xbuf.copy_(xin[k])
            graph.launch(stream)
            stream.synchronize()
            assert torch.equal(out_p, out_g), f"{name}: sync step {k} differs"
    graph.close()
    assert plain.status() == 0 and replay.status() == 0 and B.dp_device_status() == 0
