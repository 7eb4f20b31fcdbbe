"""Block-step parity of the SDXL-shaped transformer block kind through dp_block_step.

The block (GroupNorm and self-attention whose other-band context is the previous step's,
then per-token LayerNorms, cross-attention over a text context every band sees whole, and a
GELU-gated feed-forward) runs a sync step and two displaced steps of a drifting input on the
GPU and in the oracle from the same seeded inputs; every step's output is compared.
"""
import pytest
import torch

from displaced_patch_parallelism_b200 import binding as B
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
