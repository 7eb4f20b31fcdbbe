"""Seeded synthetic inputs for the displaced-patch block step.

This module is shared by the CPU oracle's tests, the CUDA parity tests and the
benchmark.  It holds no arithmetic of the method itself: only random draws, the
bf16 storage rounding of those draws, the workload shapes and the sampler's noise
schedule (``ddim_alpha_bars``, an input of the sampler update).

The shapes stand in for the SDXL workloads that "DistriFusion: Distributed
Parallel Inference for High-Resolution Diffusion Models" (study.space summary,
Experiments; atlas.scime.ai summary, Key results) evaluates on COCO Captions
with the SDXL model: 1024x1024 images (latent 128x128) and 3840x3840 images
(latent 480x480).  Neither the dataset nor the weights exist here, so every
tensor is drawn from a seeded ``torch.Generator`` on the CPU.

Drawing rules (one reading, stated once):
  * step-0 activations ~ N(0, 1) with the workload seed;
  * step k >= 1 adds N(0, drift^2) drawn with seed ``drift_seed_base + k``
    to the previous step's fp32 activations (the 1x64x32x32 case uses seed 1
    for its only displaced step);
  * conv weights are Kaiming-normal, std sqrt(2 / (Cin * 9));
  * attention projection weights ~ N(0, 0.02^2);
  * all of a block's weights come from ONE generator seeded once, drawn in the
    order listed by ``Workload.weight_specs``;
  * bf16 workloads store every drawn tensor rounded to bf16 (round to nearest
    even); fp32 workloads keep fp32.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional, Tuple

import torch

# Step modes (same numbering as the C ABI).
SYNC, DISPLACED, NAIVE = 0, 1, 2
MODE_NAMES = {SYNC: "sync", DISPLACED: "displaced", NAIVE: "naive"}


def mode_for_step(step: int, warmup: int) -> int:
    """Mode of denoising step ``step`` given ``warmup`` synchronous steps.

    Warm-up steps run synchronously (atlas.scime.ai summary, ablation rows on
    warm-up steps).  With zero warm-up there is no previous step to borrow
    context from, so step 0 runs as independent patches (the naive baseline).
    """
    if step < warmup:
        return SYNC
    if step == 0:
        return NAIVE
    return DISPLACED


def randn(shape, seed: int, std: float = 1.0) -> torch.Tensor:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    t = torch.randn(*shape, generator=g, dtype=torch.float32)
    return t * std if std != 1.0 else t


def store(t: torch.Tensor, dtype: str) -> torch.Tensor:
    """Round an fp32 tensor to the workload's storage type, returned as fp32."""
    if dtype == "bf16":
        return t.to(torch.bfloat16).to(torch.float32)
    if dtype == "fp32":
        return t.to(torch.float32)
    raise ValueError(dtype)


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: a block kind, its shapes and its seeds."""

    name: str
    kind: str                 # "gn_conv" | "resblock" | "attn" | "transformer" | "unet_mini" | "unet_sdxl"
    C: int                    # channels of the block input
    H: int
    W: int
    P: int                    # virtual row patches
    dtype: str = "bf16"
    G: int = 32
    eps: float = 1e-5
    heads: int = 0
    head_dim: int = 64
    Cout: int = 0             # output channels (0 = same as C)
    silu: bool = True
    steps: int = 50
    warmup: int = 4
    drift: float = 0.05
    seed: int = 0
    drift_seed_base: int = 1000
    weight_seed: int = 2
    first_drift_seed: Optional[int] = None  # overrides drift_seed_base + 1
    ctx_len: int = 0          # transformer: text context tokens
    ctx_dim: int = 0          # transformer: text context width
    ff_inner: int = 0         # transformer: feed-forward inner width
    depth: int = 1            # transformer: basic layers between proj_in and proj_out
    base: int = 320           # unet_sdxl: level widths base, 2 base, 4 base
    depths: Tuple[int, int, int] = (0, 2, 10)   # unet_sdxl: transformer depth of each level
    temb_dim: int = 0         # unet_sdxl: time-embedding width

    @property
    def cout(self) -> int:
        return self.Cout or self.C

    def drift_seed(self, step: int) -> int:
        if step == 1 and self.first_drift_seed is not None:
            return self.first_drift_seed
        return self.drift_seed_base + step

    def weight_specs(self) -> List[Tuple[str, Tuple[int, ...], float]]:
        """(name, shape, std) of every weight, in draw order."""
        C, Co = self.C, self.cout
        if self.kind == "gn_conv":
            return [("conv_w", (Co, C, 3, 3), math.sqrt(2.0 / (C * 9)))]
        if self.kind == "resblock":
            specs = [("conv1_w", (Co, C, 3, 3), math.sqrt(2.0 / (C * 9))),
                     ("conv2_w", (Co, Co, 3, 3), math.sqrt(2.0 / (Co * 9)))]
            if Co != C:
                specs.append(("short_w", (Co, C, 1, 1), math.sqrt(2.0 / C)))
            return specs
        if self.kind == "attn":
            return [("wq", (C, C), 0.02), ("wk", (C, C), 0.02),
                    ("wv", (C, C), 0.02), ("wo", (C, C), 0.02)]
        if self.kind == "unet_mini":
            return unet_mini_weight_specs(self.C)
        if self.kind == "transformer":
            return transformer_weight_specs("", C, self.ctx_dim, self.ff_inner, self.depth)
        if self.kind == "unet_sdxl":
            return sdxl_unet_specs(self)[0]
        raise ValueError(self.kind)


def transformer_weight_specs(pre: str, C: int, Cc: int, F: int,
                             depth: int) -> List[Tuple[str, Tuple[int, ...], float]]:
    """Matrices of a transformer block (names prefixed by ``pre``), in draw order; layers
    after the first are drawn after proj_out, so depth 1 draws what it always did."""
    def layer(lp):
        sq = [(lp + n, (C, C), C ** -0.5) for n in ("wq", "wk", "wv", "wo", "cq_w")]
        return sq + [(lp + "ck_w", (C, Cc), Cc ** -0.5), (lp + "cv_w", (C, Cc), Cc ** -0.5),
                     (lp + "co_w", (C, C), C ** -0.5), (lp + "ff1_w", (2 * F, C), C ** -0.5),
                     (lp + "ff2_w", (C, F), F ** -0.5)]
    s = [(pre + "proj_in_w", (C, C), C ** -0.5)] + layer(pre) + [(pre + "proj_out_w", (C, C), C ** -0.5)]
    for i in range(1, depth):
        s += layer(f"{pre}l{i}.")
    return s


def transformer_affine_specs(pre: str, C: int, F: int, depth: int) -> List[Tuple[str, int, str]]:
    def layer(lp):
        return [(lp + "ln1_g", C, "gamma"), (lp + "ln1_b", C, "beta"), (lp + "bq", C, "bias"),
                (lp + "bk", C, "bias"), (lp + "bv", C, "bias"), (lp + "bo", C, "bias"),
                (lp + "ln2_g", C, "gamma"), (lp + "ln2_b", C, "beta"), (lp + "co_b", C, "bias"),
                (lp + "ln3_g", C, "gamma"), (lp + "ln3_b", C, "beta"),
                (lp + "ff1_b", 2 * F, "bias"), (lp + "ff2_b", C, "bias")]
    s = [(pre + "gn_gamma", C, "gamma"), (pre + "gn_beta", C, "beta"), (pre + "proj_in_b", C, "bias")]
    s += layer(pre) + [(pre + "proj_out_b", C, "bias")]
    for i in range(1, depth):
        s += layer(f"{pre}l{i}.")
    return s


def sdxl_unet_stages(base: int, depths) -> List[Tuple[str, str, int, int]]:
    """The SDXL-shaped U-Net's stages in execution order: (kind, weight prefix, input channels,
    output channels), kind one of "conv_in", "resblock", "transformer", "down", "up", "out".
    Names only: the weight names a caller draws and marshals (the latent's channel count is
    filled in as 0 here)."""
    ch = (base, 2 * base, 4 * base)
    s = [("conv_in", "conv_in", 0, ch[0])]
    skips = [ch[0]]
    c = ch[0]
    for lvl in range(3):
        for i in range(2):
            s.append(("resblock", f"d{lvl}.r{i}.", c, ch[lvl]))
            c = ch[lvl]
            if depths[lvl]:
                s.append(("transformer", f"d{lvl}.t{i}.", c, c))
            skips.append(c)
        if lvl < 2:
            s.append(("down", f"d{lvl}.down", c, c))
            skips.append(c)
    s.append(("resblock", "mid.r0.", c, c))
    if depths[2]:
        s.append(("transformer", "mid.t.", c, c))
    s.append(("resblock", "mid.r1.", c, c))
    for lvl in (2, 1, 0):
        for i in range(3):
            s.append(("resblock", f"u{lvl}.r{i}.", c + skips.pop(), ch[lvl]))
            c = ch[lvl]
            if depths[lvl]:
                s.append(("transformer", f"u{lvl}.t{i}.", c, c))
        if lvl > 0:
            s.append(("up", f"u{lvl}.up", c, c))
    s.append(("out", "out.", c, 0))
    return s


def sdxl_unet_specs(wl: "Workload"):
    """(matrix specs, affine specs) of an SDXL-shaped U-Net workload, in draw order."""
    mats: List[Tuple[str, Tuple[int, ...], float]] = []
    aff: List[Tuple[str, int, str]] = []
    depth_of = {"d0": wl.depths[0], "d1": wl.depths[1], "d2": wl.depths[2], "mid": wl.depths[2],
                "u2": wl.depths[2], "u1": wl.depths[1], "u0": wl.depths[0]}
    conv = lambda name, co, ci: (name, (co, ci, 3, 3), math.sqrt(2.0 / (ci * 9)))
    for kind, pre, ci, co in sdxl_unet_stages(wl.base, wl.depths):
        if kind == "conv_in":
            mats.append(conv("conv_in_w", co, wl.C))
            aff.append(("conv_in_b", co, "bias"))
        elif kind in ("down", "up"):
            mats.append(conv(pre + "_w", co, ci))
            aff.append((pre + "_b", co, "bias"))
        elif kind == "resblock":
            mats += [conv(pre + "conv1_w", co, ci), conv(pre + "conv2_w", co, co)]
            if ci != co:
                mats.append((pre + "short_w", (co, ci, 1, 1), math.sqrt(2.0 / ci)))
            mats.append((pre + "temb_w", (co, wl.temb_dim), wl.temb_dim ** -0.5))
            aff += [(pre + "gn1_gamma", ci, "gamma"), (pre + "gn1_beta", ci, "beta"),
                    (pre + "conv1_b", co, "bias"), (pre + "gn2_gamma", co, "gamma"),
                    (pre + "gn2_beta", co, "beta"), (pre + "conv2_b", co, "bias")]
            if ci != co:
                aff.append((pre + "short_b", co, "bias"))
            aff.append((pre + "temb_b", co, "bias"))
        elif kind == "transformer":
            depth = depth_of[pre.split(".")[0]]
            mats += transformer_weight_specs(pre, ci, wl.ctx_dim, 4 * ci, depth)
            aff += transformer_affine_specs(pre, ci, 4 * ci, depth)
        else:   # out: GroupNorm + SiLU + conv_out back to the latent's channels
            mats.append(conv("out.conv_w", wl.C, ci))
            aff += [("out.gn_gamma", ci, "gamma"), ("out.gn_beta", ci, "beta"), ("out.conv_b", wl.C, "bias")]
    return mats, aff


def unet_mini_weight_specs(cin: int) -> List[Tuple[str, Tuple[int, ...], float]]:
    """Weights of the mini U-Net chain, in draw order (Kaiming for convs)."""
    def conv(name, co, ci, k=3):
        return (name, (co, ci, k, k), math.sqrt(2.0 / (ci * k * k)))

    def lin(name, c):
        return (name, (c, c), math.sqrt(2.0 / c))

    s = [conv("conv_in_w", 320, cin)]
    s += [conv("rb1.conv1_w", 320, 320), conv("rb1.conv2_w", 320, 320)]
    s += [conv("down1_w", 320, 320)]
    s += [conv("rb2.conv1_w", 640, 320), conv("rb2.conv2_w", 640, 640),
          ("rb2.short_w", (640, 320, 1, 1), math.sqrt(2.0 / 320))]
    s += [lin("at2.wq", 640), lin("at2.wk", 640), lin("at2.wv", 640), lin("at2.wo", 640)]
    s += [conv("down2_w", 640, 640)]
    s += [conv("rb3.conv1_w", 1280, 640), conv("rb3.conv2_w", 1280, 1280),
          ("rb3.short_w", (1280, 640, 1, 1), math.sqrt(2.0 / 640))]
    s += [lin("at3.wq", 1280), lin("at3.wk", 1280), lin("at3.wv", 1280), lin("at3.wo", 1280)]
    return s


# The synthetic workloads (logical NCHW shapes, N = 1).
WORKLOADS: Dict[str, Workload] = {
    "tiny_fp32_gn_conv": Workload(
        name="tiny_fp32_gn_conv", kind="gn_conv", C=64, H=32, W=32, P=2,
        dtype="fp32", steps=2, warmup=1, drift=0.05, seed=0, first_drift_seed=1,
        weight_seed=2),
    "resblock_320x128x128": Workload(
        name="resblock_320x128x128", kind="resblock", C=320, H=128, W=128, P=4,
        steps=50, warmup=4, drift=0.05),
    "attn_640x64x64": Workload(
        name="attn_640x64x64", kind="attn", C=640, H=64, W=64, P=4, heads=10,
        head_dim=64, silu=False, steps=50, warmup=4, drift=0.05),
    # SDXL 1024 px transformer block shape ("next" item; not a headline workload): 640
    # channels at 64x64, 10 heads, a 77-token text context of width 2048, feed-forward 4C
    "transformer_640x64x64": Workload(
        name="transformer_640x64x64", kind="transformer", C=640, H=64, W=64, P=4, heads=10,
        head_dim=64, silu=False, steps=50, warmup=4, drift=0.05, ctx_len=77, ctx_dim=2048,
        ff_inner=2560),
    # SDXL's innermost transformer level at 1024 px ("next" item; not a headline workload):
    # 1280 channels at 32x32 (1024 tokens), 20 heads, ten basic layers, the 77-token text
    # context of width 2048, feed-forward 4C (0.35 billion parameters)
    "transformer_1280x32x32": Workload(
        name="transformer_1280x32x32", kind="transformer", C=1280, H=32, W=32, P=8, heads=20,
        head_dim=64, silu=False, steps=20, warmup=4, drift=0.05, ctx_len=77, ctx_dim=2048,
        ff_inner=5120, depth=10),
    "gn_conv_320x480x480": Workload(
        name="gn_conv_320x480x480", kind="gn_conv", C=320, H=480, W=480, P=8,
        steps=50, warmup=4, drift=0.05),
    # SDXL's whole U-Net at 1024 px (latent 4x128x128), one step of batch 1, over 8 bands:
    # base width 320, transformer depths 0 / 2 / 10, 77-token context of width 2048, time
    # embedding of width 1280 (2.56 billion parameters)
    "unet_sdxl_4x128x128": Workload(
        name="unet_sdxl_4x128x128", kind="unet_sdxl", C=4, H=128, W=128, P=8, steps=10, warmup=2,
        drift=0.03, weight_seed=21, base=320, depths=(0, 2, 10), ctx_len=77, ctx_dim=2048,
        temb_dim=1280),
    "unet_mini_4x128x128": Workload(
        name="unet_mini_4x128x128", kind="unet_mini", C=4, H=128, W=128, P=4, Cout=1280,
        steps=10, warmup=2, drift=0.03, weight_seed=7),
}


# The five block workloads the parity and benchmark configurations are built on; the
# transformer block and the whole SDXL U-Net are the wider SDXL-shaped workloads.
CONFIG_WORKLOADS = ("tiny_fp32_gn_conv", "resblock_320x128x128", "attn_640x64x64",
                    "gn_conv_320x480x480", "unet_mini_4x128x128")


def make_weights(wl: Workload, random_affine: bool = False,
                 affine_seed: int = 99, device=None) -> Dict[str, torch.Tensor]:
    """All weights of ``wl`` as fp32 tensors holding storage-rounded values.

    GroupNorm scale/shift are 1/0 and biases 0 as the workloads state; with
    ``random_affine`` they are drawn instead (unit tests use this so that an
    indexing slip in gamma, beta or a bias cannot hide behind zeros).  With a
    ``device`` the matrices are drawn there by that device's generator, seeded
    the same way (the benchmark's whole-U-Net workload: 2.56 billion parameters),
    so their values differ from the CPU draw; the rules are the same.
    """
    g = torch.Generator(device=device or "cpu")
    g.manual_seed(int(wl.weight_seed))
    out: Dict[str, torch.Tensor] = {}
    for name, shape, std in wl.weight_specs():
        out[name] = store(torch.randn(*shape, generator=g, device=device) * std, wl.dtype)
    # affine parameters and biases
    ga = torch.Generator(device="cpu")
    ga.manual_seed(int(affine_seed))

    def vec(n, kind):
        if not random_affine:
            return torch.ones(n) if kind == "gamma" else torch.zeros(n)
        if kind == "gamma":
            return 1.0 + 0.25 * torch.randn(n, generator=ga)
        return 0.25 * torch.randn(n, generator=ga)

    for name, c, kind in affine_specs(wl):
        out[name] = vec(c, kind).to(torch.float32)
    return out


def affine_specs(wl: Workload) -> List[Tuple[str, int, str]]:
    C, Co = wl.C, wl.cout
    if wl.kind == "gn_conv":
        return [("gn_gamma", C, "gamma"), ("gn_beta", C, "beta"), ("conv_b", Co, "bias")]
    if wl.kind == "resblock":
        s = [("gn1_gamma", C, "gamma"), ("gn1_beta", C, "beta"), ("conv1_b", Co, "bias"),
             ("gn2_gamma", Co, "gamma"), ("gn2_beta", Co, "beta"), ("conv2_b", Co, "bias")]
        if Co != C:
            s.append(("short_b", Co, "bias"))
        return s
    if wl.kind == "attn":
        return [("gn_gamma", C, "gamma"), ("gn_beta", C, "beta"), ("bq", C, "bias"),
                ("bk", C, "bias"), ("bv", C, "bias"), ("bo", C, "bias")]
    if wl.kind == "unet_mini":
        s = [("conv_in_b", 320, "bias")]
        for pre, ci, co in (("rb1", 320, 320), ("rb2", 320, 640), ("rb3", 640, 1280)):
            s += [(pre + ".gn1_gamma", ci, "gamma"), (pre + ".gn1_beta", ci, "beta"),
                  (pre + ".conv1_b", co, "bias"), (pre + ".gn2_gamma", co, "gamma"),
                  (pre + ".gn2_beta", co, "beta"), (pre + ".conv2_b", co, "bias")]
            if ci != co:
                s.append((pre + ".short_b", co, "bias"))
        s += [("down1_b", 320, "bias"), ("down2_b", 640, "bias")]
        for pre, c in (("at2", 640), ("at3", 1280)):
            s += [(pre + ".gn_gamma", c, "gamma"), (pre + ".gn_beta", c, "beta"),
                  (pre + ".bq", c, "bias"), (pre + ".bk", c, "bias"),
                  (pre + ".bv", c, "bias"), (pre + ".bo", c, "bias")]
        return s
    if wl.kind == "transformer":
        return transformer_affine_specs("", C, wl.ff_inner, wl.depth)
    if wl.kind == "unet_sdxl":
        return sdxl_unet_specs(wl)[1]
    raise ValueError(wl.kind)


def context(wl: Workload) -> torch.Tensor:
    """A transformer workload's text context (ctx_len, ctx_dim): N(0, 1), storage-rounded,
    drawn with seed ``seed + 500``; the same for every step, as a prompt's encoding is."""
    return store(randn((wl.ctx_len, wl.ctx_dim), wl.seed + 500), wl.dtype)


class InputStream:
    """The per-step block inputs x_0, x_1, ... of a workload (logical NCHW).

    ``x(k)`` returns the storage-rounded input of step k as fp32 (1, C, H, W).
    The fp32 chain is kept unrounded between steps; only what a step consumes
    is rounded.
    """

    def __init__(self, wl: Workload, shape: Optional[Tuple[int, ...]] = None):
        self.wl = wl
        self.shape = shape or (1, wl.C, wl.H, wl.W)
        self._chain = [randn(self.shape, wl.seed)]

    def x(self, k: int) -> torch.Tensor:
        while len(self._chain) <= k:
            j = len(self._chain)
            self._chain.append(self._chain[-1] + randn(self.shape, self.wl.drift_seed(j), self.wl.drift))
        return store(self._chain[k], self.wl.dtype)


def ddim_alpha_bars(steps: int = 50, train_steps: int = 1000, beta_start: float = 0.00085,
                    beta_end: float = 0.012) -> List[Tuple[float, float]]:
    """(abar_t, abar_prev) of each sampler step, first to last: the scaled-linear noise
    schedule of the Stable Diffusion family (betas evenly spaced in sqrt between beta_start
    and beta_end over train_steps, abar = cumulative product of 1 - beta) at `steps` evenly
    spaced timesteps from the noisiest down; the last step's previous level is abar = 1
    (the clean sample).  Sampler inputs only."""
    betas = torch.linspace(beta_start ** 0.5, beta_end ** 0.5, train_steps, dtype=torch.float64) ** 2
    abar = torch.cumprod(1.0 - betas, dim=0)
    stride = train_steps // steps
    ts = [train_steps - 1 - k * stride for k in range(steps)]
    out = []
    for k, t in enumerate(ts):
        prev = abar[ts[k + 1]] if k + 1 < steps else 1.0
        out.append((float(abar[t]), float(prev)))
    return out


def nchw_to_nhwc(t: torch.Tensor) -> torch.Tensor:
    """(1, C, H, W) -> contiguous (H, W, C)."""
    return t[0].permute(1, 2, 0).contiguous()


def nhwc_to_nchw(t: torch.Tensor) -> torch.Tensor:
    """(H, W, C) -> (1, C, H, W)."""
    return t.permute(2, 0, 1).unsqueeze(0).contiguous()


def conv_weight_to_device(w: torch.Tensor) -> torch.Tensor:
    """(Cout, Cin, kh, kw) -> contiguous (Cout, kh, kw, Cin): one K-major row per output channel."""
    return w.permute(0, 2, 3, 1).contiguous()
