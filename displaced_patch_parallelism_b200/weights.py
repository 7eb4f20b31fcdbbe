"""Marshalling of a block's weights into the device layouts ``dp_block_step`` expects.

Layout changes only (no arithmetic of the method): conv filters go from
(Cout, Cin, 3, 3) to [Cout][3][3][Cin]; the q, k and v projection matrices are
stacked into one [3C][C] matrix so a single GEMM produces all three; a
transformer's gated feed-forward projection has its value and gate rows
interleaved in blocks of 16; GroupNorm scale/shift and biases are fp32.
"""
from __future__ import annotations

from typing import Dict, List

import torch


def _t(a, dtype, device):
    t = a if isinstance(a, torch.Tensor) else torch.as_tensor(a)
    return t.to(torch.float32).to(dtype).contiguous().to(device)


def _interleave16(w):
    """Rows [a (F rows) | g (F rows)] of a gated feed-forward projection -> blocks of 16:
    rows 32k..32k+15 are a rows 16k..16k+15, rows 32k+16..32k+31 the matching g rows."""
    t = w if isinstance(w, torch.Tensor) else torch.as_tensor(w)
    F = t.shape[0] // 2
    rest = tuple(t.shape[1:])
    return t.reshape(2, F // 16, 16, *rest).transpose(0, 1).reshape(2 * F, *rest)


def _conv(w, dtype, device):
    t = w if isinstance(w, torch.Tensor) else torch.as_tensor(w)
    return t.to(torch.float32).permute(0, 2, 3, 1).contiguous().to(dtype).to(device)


def block_weights(kind: str, wts: Dict, dtype: torch.dtype = torch.bfloat16, device="cuda",
                  prefix: str = "", depth: int = 1) -> List[torch.Tensor]:
    """Device tensors in the order ``dp_block_step`` documents for ``kind`` (a TRANSFORMER
    block's per-step text context, its last pointer, and a RESBLOCK's per-step time
    embedding, its last pointer, are appended by the caller).  ``depth`` is a TRANSFORMER
    block's number of basic layers; layer l >= 1 has its weights named "l<l>.<name>"."""
    g = lambda n: wts[prefix + n]
    f32 = torch.float32
    if kind == "gn_conv":
        return [_t(g("gn_gamma"), f32, device), _t(g("gn_beta"), f32, device),
                _conv(g("conv_w"), dtype, device), _t(g("conv_b"), f32, device)]
    if kind == "resblock":
        out = [_t(g("gn1_gamma"), f32, device), _t(g("gn1_beta"), f32, device),
               _conv(g("conv1_w"), dtype, device), _t(g("conv1_b"), f32, device),
               _t(g("gn2_gamma"), f32, device), _t(g("gn2_beta"), f32, device),
               _conv(g("conv2_w"), dtype, device), _t(g("conv2_b"), f32, device)]
        if (prefix + "short_w") in wts:
            sw = g("short_w")
            sw = sw if isinstance(sw, torch.Tensor) else torch.as_tensor(sw)
            out += [_t(sw.reshape(sw.shape[0], sw.shape[1]), dtype, device),
                    _t(g("short_b"), f32, device)]
        if (prefix + "temb_w") in wts:   # the step's time embedding is appended by the caller
            out += [_t(g("temb_w"), f32, device), _t(g("temb_b"), f32, device)]
        return out
    if kind == "attn":
        cat = lambda *xs: torch.cat([x if isinstance(x, torch.Tensor) else torch.as_tensor(x) for x in xs])
        return [_t(g("gn_gamma"), f32, device), _t(g("gn_beta"), f32, device),
                _t(cat(g("wq"), g("wk"), g("wv")), dtype, device),
                _t(cat(g("bq"), g("bk"), g("bv")), f32, device),
                _t(g("wo"), dtype, device), _t(g("bo"), f32, device)]
    if kind == "transformer":
        cat = lambda *xs: torch.cat([x if isinstance(x, torch.Tensor) else torch.as_tensor(x) for x in xs])
        v = lambda n: _t(g(n), f32, device)
        m = lambda n: _t(g(n), dtype, device)
        out = [v("gn_gamma"), v("gn_beta"), m("proj_in_w"), v("proj_in_b")]
        for i in range(depth):
            p = "" if i == 0 else f"l{i}."     # layer i's weight names
            out += [v(p + "ln1_g"), v(p + "ln1_b"),
                    _t(cat(g(p + "wq"), g(p + "wk"), g(p + "wv")), dtype, device),
                    _t(cat(g(p + "bq"), g(p + "bk"), g(p + "bv")), f32, device), m(p + "wo"), v(p + "bo"),
                    v(p + "ln2_g"), v(p + "ln2_b"), m(p + "cq_w"),
                    _t(cat(g(p + "ck_w"), g(p + "cv_w")), dtype, device), m(p + "co_w"), v(p + "co_b"),
                    v(p + "ln3_g"), v(p + "ln3_b"), _t(_interleave16(g(p + "ff1_w")), dtype, device),
                    _t(_interleave16(g(p + "ff1_b")), f32, device), m(p + "ff2_w"), v(p + "ff2_b")]
        return out + [m("proj_out_w"), v("proj_out_b")]
    if kind == "unet_sdxl":
        raise ValueError("use unet_sdxl_weights for a UNET_SDXL block")
    if kind == "unet_mini":
        out = [_conv(g("conv_in_w"), dtype, device), _t(g("conv_in_b"), f32, device)]
        out += block_weights("resblock", wts, dtype, device, prefix + "rb1.")
        out += [_conv(g("down1_w"), dtype, device), _t(g("down1_b"), f32, device)]
        out += block_weights("resblock", wts, dtype, device, prefix + "rb2.")
        out += block_weights("attn", wts, dtype, device, prefix + "at2.")
        out += [_conv(g("down2_w"), dtype, device), _t(g("down2_b"), f32, device)]
        out += block_weights("resblock", wts, dtype, device, prefix + "rb3.")
        out += block_weights("attn", wts, dtype, device, prefix + "at3.")
        return out
    raise ValueError(kind)


def unet_sdxl_weights(wts: Dict, stages, depths, dtype: torch.dtype = torch.bfloat16,
                      device="cuda") -> List[torch.Tensor]:
    """Device tensors of a UNET_SDXL block in the order ``dp_block_step`` documents, from
    ``stages`` (the (kind, prefix, cin, cout) list of ``synth.sdxl_unet_stages``) and the
    levels' transformer ``depths``; the step's context and time embedding, its last two
    pointers, are appended by the caller."""
    f32 = torch.float32
    depth_of = {"d0": depths[0], "d1": depths[1], "d2": depths[2], "mid": depths[2],
                "u2": depths[2], "u1": depths[1], "u0": depths[0]}
    out: List[torch.Tensor] = []
    for kind, pre, _ci, _co in stages:
        if kind == "conv_in":
            out += [_conv(wts["conv_in_w"], dtype, device), _t(wts["conv_in_b"], f32, device)]
        elif kind in ("down", "up"):
            out += [_conv(wts[pre + "_w"], dtype, device), _t(wts[pre + "_b"], f32, device)]
        elif kind == "resblock":
            out += block_weights("resblock", wts, dtype, device, pre)
        elif kind == "transformer":
            out += block_weights("transformer", wts, dtype, device, pre, depth_of[pre.split(".")[0]])
        else:
            out += block_weights("gn_conv", wts, dtype, device, pre)
    return out
