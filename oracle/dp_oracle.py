"""CPU oracle for the displaced-patch-parallelism block step.  TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg
may import this module.  The product path (the CUDA library and its Python
binding) never does, and shares no code with it.

What it computes is the method of "DistriFusion: Distributed Parallel Inference
for High-Resolution Diffusion Models": the image latent is split into P row
patches; each patch computes its own rows with fresh activations and takes the
context it needs from other patches out of the previous denoising step's
("stale", "displaced") activations (study.space summary, Method; atlas.scime.ai
summary, Approach), with a corrected asynchronous GroupNorm (atlas.scime.ai
summary, Approach and the GroupNorm ablation rows).  Attention keeps the full
set of keys and values, fresh for the patch's own tokens and stale for the
others (gist.science PipeFusion explainer, Problem Statement and Memory
Efficiency, describing DistriFusion's full-spatial K/V buffers).

Arithmetic is fp64 numpy throughout.  Where the GPU stores an intermediate in
bf16 (GroupNorm output, conv output feeding the next GroupNorm, q/k/v, the
attention output, block outputs) the oracle rounds to bf16 at the same point
(``store``); pass ``storage="none"`` to keep everything unrounded.

Readings of what the pages leave open:
  R1  corrected statistics on raw moments (E[x], E[x^2]):
        used = stale_global + w * (fresh_local - stale_local),  w = 1 by default
  R2  a negative corrected variance falls back to the patch's fresh variance
  R3  zero warm-up: step 0 runs as independent patches (zero context)
  R4  equal row bands of H/P rows; equal-weight averages across bands
  R5  the stale tensor of a conv is its input (after GroupNorm and SiLU)
  R6  block structures: see ``gn_conv_step``, ``resblock_step``, ``attn_step``,
      ``unet_mini_step``
  R7  every 3x3 conv, stride 1 or 2, pads by one and takes halo rows from
      other bands per mode; stride-2 output bands are Ho/P rows
  R12 the GroupNorm ablation's alternatives for displaced steps (band-local,
      stale-only and exact statistics): see ``gn_variant_mode``
  R15 the pages' sampler is "50-step DDIM" with no update printed: the
      deterministic DDIM step (``ddim_step``), alpha-bar values from the caller
  R16 the pages' warm-up ablation names a "10-step DPM-Solver" with no update
      printed: the multistep second-order DPM-Solver++ (``dpm_solver_2m_step``)
  R13 the pages name SDXL but not its blocks' insides: the plainest SDXL
      transformer block (``transformer_step``) and ResBlock time embedding
      (``resblock_step``'s ``temb``); only GroupNorm statistics and
      self-attention keys/values cross bands
  R18 the whole SDXL-shaped U-Net (``sdxl_unet_step``): SDXL's level layout
      (widths base, 2 base, 4 base; transformer depths per level), [h, skip]
      concatenation, nearest 2x upsampling; one GroupNorm epsilon for all
      GroupNorms; the caller gives the step's time embedding vector

Parity pins (the tests under tests/test_oracle_*.py): P = 1 reduces to the
library full-image block (torch group_norm / conv2d / softmax attention);
brute-force loops on tiny inputs; naive mode equals independent crops; an
unchanged input makes displaced equal sync; a uniform drift makes the
corrected statistics exact; halo and attention locality; zero warm-up differs
from sync; the GroupNorm variants equal the library GroupNorm of the whole
image, of each band's crop and of the previous step's image; the transformer
block and the time-embedding ResBlock equal the same blocks composed from
library operators at P = 1; ``time_embedding_term`` is the library linear of
the library SiLU; ``ddim_step`` moves an exactly known noise to the previous
level, is the identity at an unchanged level, composes, and is affine.
``dpm_solver_2m_step`` in its first-order form equals the DDIM step, its
second-order form equals the first when the data prediction does not change,
and on an ODE whose exact solution is known it converges at second order (the
first-order form at first order).
``sdxl_unet_step`` at P = 1 equals the U-Net composed from library operators
(and differs from it with the skip order swapped or other depths), equals
independent crops in naive mode, equals sync under an unchanged input, and a
displaced step keeps every other band bit for bit when one band's input changes.
``unet_mini_step`` at P = 1 equals the same chain composed from library
operators (conv2d with stride 1 and 2, the library ResBlock and attention with
10 and 20 heads); its naive step at P = 4 equals that library chain on each
band's crop; and at P = 4 an unchanged input makes its displaced step equal its
synchronous one.
"""
from __future__ import annotations

import math
from typing import Dict, Optional, Tuple

import numpy as np
import torch

SYNC, DISPLACED, NAIVE = 0, 1, 2


# --------------------------------------------------------------------------
# storage rounding
# --------------------------------------------------------------------------
def to_bf16(x: np.ndarray) -> np.ndarray:
    """Round to bf16 (nearest even) and return as fp64.

    fp64 -> fp32 -> bf16: the GPU rounds an fp32 value, so the oracle rounds
    through fp32 as well.
    """
    f32 = np.ascontiguousarray(x, dtype=np.float32)
    u = f32.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    u = (u + 0x7FFF + lsb) >> 16 << 16
    nan = np.isnan(f32)
    out = (u & 0xFFFFFFFF).astype(np.uint32).view(np.float32).astype(np.float64)
    out[nan] = np.nan
    return out


def store(x: np.ndarray, storage: str) -> np.ndarray:
    if storage == "bf16":
        return to_bf16(x)
    if storage == "fp32":
        return np.asarray(x, dtype=np.float32).astype(np.float64)
    if storage == "none":
        return np.asarray(x, dtype=np.float64)
    raise ValueError(storage)


# --------------------------------------------------------------------------
# GroupNorm (atlas.scime.ai summary: Approach; GroupNorm ablation rows)
# --------------------------------------------------------------------------
def gn_fresh_local(x: np.ndarray, P: int, G: int) -> np.ndarray:
    """Per (band p, group g) raw moments of the fresh input.

    x: (C, H, W).  Band p is rows [p*H/P, (p+1)*H/P); group g is channels
    [g*C/G, (g+1)*C/G).  Returns f[p, g] = (mean x, mean x^2).
    """
    C, H, W = x.shape
    hb, cg = H // P, C // G
    f = np.empty((P, G, 2))
    for p in range(P):
        for g in range(G):
            v = x[g * cg:(g + 1) * cg, p * hb:(p + 1) * hb, :]
            f[p, g, 0] = v.mean()
            f[p, g, 1] = (v * v).mean()
    return f


def gn_used_stats(f: np.ndarray, mode: int, stale_global: Optional[np.ndarray],
                  stale_local: Optional[np.ndarray], w: float = 1.0
                  ) -> Tuple[np.ndarray, int]:
    """Statistics each band normalises with.  Returns (used[p, g] = (mean, var), fallbacks).

    sync:       the exact whole-image moments, i.e. the average of the bands'
                moments (equal bands);
    displaced:  stale whole-image moments corrected by the band's own drift,
                stale_global + w * (fresh_local - stale_local)   (reading R1);
    naive:      the band's own moments only.
    var = E[x^2] - E[x]^2; a negative var falls back to the band's fresh var (R2).
    """
    P, G, _ = f.shape
    if mode == SYNC:
        m = np.broadcast_to(f.mean(axis=0), f.shape).copy()
    elif mode == DISPLACED:
        if stale_global is None or stale_local is None:
            raise ValueError("displaced GroupNorm needs the previous step's statistics")
        m = stale_global[None, :, :] + w * (f - stale_local)
    elif mode == NAIVE:
        m = f.copy()
    else:
        raise ValueError(mode)
    mean = m[..., 0]
    var = m[..., 1] - mean * mean
    fresh_var = f[..., 1] - f[..., 0] * f[..., 0]
    neg = var < 0
    var = np.where(neg, fresh_var, var)
    return np.stack([mean, var], axis=-1), int(neg.sum())


def gn_apply(x: np.ndarray, used: np.ndarray, gamma: np.ndarray, beta: np.ndarray,
             P: int, G: int, eps: float, silu: bool) -> np.ndarray:
    """y = (x - mean) / sqrt(var + eps) * gamma_c + beta_c, per band and group; then SiLU."""
    C, H, W = x.shape
    hb, cg = H // P, C // G
    y = np.empty_like(x, dtype=np.float64)
    for p in range(P):
        for g in range(G):
            cs = slice(g * cg, (g + 1) * cg)
            rs = slice(p * hb, (p + 1) * hb)
            mean, var = used[p, g]
            y[cs, rs, :] = ((x[cs, rs, :] - mean) / math.sqrt(var + eps)
                            * gamma[cs, None, None] + beta[cs, None, None])
    if silu:
        y = y / (1.0 + np.exp(-y))
    return y


def groupnorm_async(x, gamma, beta, P, G, eps, w, silu, mode, stale_global, stale_local):
    """One GroupNorm layer: returns (y, fresh_local, used, fallbacks)."""
    f = gn_fresh_local(x, P, G)
    used, nneg = gn_used_stats(f, mode, stale_global, stale_local, w)
    return gn_apply(x, used, gamma, beta, P, G, eps, silu), f, used, nneg


def refresh_stats(f: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Next step's stale statistics: (stale_global = mean over bands, stale_local = f)."""
    return f.mean(axis=0), f.copy()


# --------------------------------------------------------------------------
# 3x3 convolution with stale halo rows (study.space summary, Method)
# --------------------------------------------------------------------------
def conv3x3_halo(a_fresh: np.ndarray, a_stale: Optional[np.ndarray], weight: np.ndarray,
                 bias: Optional[np.ndarray], residual: Optional[np.ndarray], P: int,
                 mode: int, stride: int = 1) -> np.ndarray:
    """3x3 conv, padding 1, whose input rows depend on the band being computed.

    Output row r of band p reads input row rho = stride*r + kh - 1:
      rho outside [0, H)         -> zeros (ordinary padding)
      rho in band p              -> a_fresh
      rho in another band        -> sync: a_fresh, displaced: a_stale, naive: zeros
    Columns use ordinary zero padding.  Then + bias (+ residual).
    a_*: (Cin, H, W); weight: (Cout, Cin, 3, 3); returns (Cout, Ho, Wo).
    """
    Cin, H, W = a_fresh.shape
    Cout = weight.shape[0]
    Ho = (H - 1) // stride + 1
    Wo = (W - 1) // stride + 1
    hb_in, hb_out = H // P, Ho // P
    if mode == DISPLACED and a_stale is None:
        raise ValueError("displaced conv needs the previous step's activations")
    out = np.zeros((Cout, Ho, Wo))
    for p in range(P):
        r0, r1 = p * hb_out, (p + 1) * hb_out
        lo = stride * r0 - 1
        hi = stride * (r1 - 1) + 1
        used = np.zeros((Cin, hi - lo + 1, W + 2))
        for rho in range(lo, hi + 1):
            if rho < 0 or rho >= H:
                continue
            if rho // hb_in == p or mode == SYNC:
                src = a_fresh
            elif mode == DISPLACED:
                src = a_stale
            else:
                continue
            used[:, rho - lo, 1:W + 1] = src[:, rho, :]
        nr = r1 - r0
        for kh in range(3):
            for kw in range(3):
                patch = used[:, kh:kh + stride * (nr - 1) + 1:stride,
                             kw:kw + stride * (Wo - 1) + 1:stride]
                out[:, r0:r1, :] += np.tensordot(weight[:, :, kh, kw], patch, axes=(1, 0))
    if bias is not None:
        out += bias[:, None, None]
    if residual is not None:
        out += residual
    return out


def conv3x3_halo_rows(a_fresh: np.ndarray, a_stale: Optional[np.ndarray], weight: np.ndarray,
                      bias: Optional[np.ndarray], P: int, mode: int, rows, stride: int = 1
                      ) -> np.ndarray:
    """Only the output rows ``rows`` of ``conv3x3_halo`` (no residual), one row at a time.

    Same rule as ``conv3x3_halo``, applied to the three input rows one output
    row reads; used to check single rows of full-size images.
    Returns (Cout, len(rows), Wo).
    """
    Cin, H, W = a_fresh.shape
    Ho = (H - 1) // stride + 1
    Wo = (W - 1) // stride + 1
    hb_in, hb_out = H // P, Ho // P
    out = np.zeros((weight.shape[0], len(rows), Wo))
    for i, r in enumerate(rows):
        p = r // hb_out
        for kh in range(3):
            rho = stride * r + kh - 1
            if rho < 0 or rho >= H:
                continue
            if rho // hb_in == p or mode == SYNC:
                src = a_fresh
            elif mode == DISPLACED:
                src = a_stale
            else:
                continue
            line = np.zeros((Cin, W + 2))
            line[:, 1:W + 1] = src[:, rho, :]
            for kw in range(3):
                seg = line[:, kw:kw + stride * (Wo - 1) + 1:stride]
                out[:, i, :] += weight[:, :, kh, kw] @ seg
    if bias is not None:
        out += bias[:, None, None]
    return out


def conv1x1(x: np.ndarray, weight: np.ndarray, bias: Optional[np.ndarray]) -> np.ndarray:
    """Pointwise conv (the ResBlock shortcut when channels change)."""
    out = np.tensordot(weight[:, :, 0, 0], x, axes=(1, 0))
    if bias is not None:
        out += bias[:, None, None]
    return out


# --------------------------------------------------------------------------
# self-attention over stitched fresh / stale K and V
# (gist.science PipeFusion explainer, Problem Statement, on DistriFusion)
# --------------------------------------------------------------------------
def attention_stale_kv(q: np.ndarray, k_fresh: np.ndarray, v_fresh: np.ndarray,
                       k_stale: Optional[np.ndarray], v_stale: Optional[np.ndarray],
                       P: int, heads: int, scale: float, mode: int) -> np.ndarray:
    """Per band p and head: softmax(q_p K^T * scale) V over the keys band p sees.

    Keys and values of band p's own tokens are fresh.  The others are stale
    (displaced), fresh (sync) or left out (naive).  q, k, v: (T, heads*d).
    """
    T, Cq = q.shape
    d = Cq // heads
    tb = T // P
    if mode == DISPLACED and (k_stale is None or v_stale is None):
        raise ValueError("displaced attention needs the previous step's keys and values")
    o = np.zeros_like(q, dtype=np.float64)
    for p in range(P):
        own = slice(p * tb, (p + 1) * tb)
        if mode == NAIVE:
            K, V = k_fresh[own], v_fresh[own]
        elif mode == SYNC:
            K, V = k_fresh, v_fresh
        elif mode == DISPLACED:
            K, V = k_stale.copy(), v_stale.copy()
            K[own], V[own] = k_fresh[own], v_fresh[own]
        else:
            raise ValueError(mode)
        for h in range(heads):
            hs = slice(h * d, (h + 1) * d)
            s = (q[own, hs] @ K[:, hs].T) * scale
            s = s - s.max(axis=1, keepdims=True)
            e = np.exp(s)
            o[own, hs] = (e / e.sum(axis=1, keepdims=True)) @ V[:, hs]
    return o


def attention_cross(q: np.ndarray, k: np.ndarray, v: np.ndarray, heads: int,
                    scale: float) -> np.ndarray:
    """Cross-attention over a context every band sees whole (an SDXL block's text keys and
    values): per head, softmax(q K^T * scale) V.  q: (Tq, heads*d); k, v: (Tk, heads*d)."""
    Tq, Cq = q.shape
    d = Cq // heads
    o = np.zeros((Tq, Cq))
    for h in range(heads):
        hs = slice(h * d, (h + 1) * d)
        s = (q[:, hs] @ k[:, hs].T) * scale
        s = s - s.max(axis=1, keepdims=True)
        e = np.exp(s)
        o[:, hs] = (e / e.sum(axis=1, keepdims=True)) @ v[:, hs]
    return o


def linear(x: np.ndarray, w: np.ndarray, b: Optional[np.ndarray]) -> np.ndarray:
    """x @ w.T + b with w stored (out, in)."""
    y = x @ w.T
    return y + b if b is not None else y


# --------------------------------------------------------------------------
# blocks (reading R6) with their cross-step state
# --------------------------------------------------------------------------
class GNState:
    def __init__(self):
        self.stale_global = None  # (G, 2)
        self.stale_local = None   # (P, G, 2)

    def refresh(self, f):
        self.stale_global, self.stale_local = refresh_stats(f)


# GroupNorm statistics variants of a displaced step ("DistriFusion",
# atlas.scime.ai summary, the GroupNorm ablation rows): the method's corrected
# statistics, statistics of the band alone, the stale statistics alone, or an
# exact synchronous pass.  Only displaced steps change; the halos and the
# keys/values stay stale.
GN_STATS_CORRECTED, GN_STATS_LOCAL, GN_STATS_STALE, GN_STATS_SYNC = 0, 1, 2, 3


def gn_variant_mode(mode: int, w: float, gn_stats: int) -> Tuple[int, float]:
    """(statistics mode, drift weight) a GroupNorm of a step in ``mode`` uses.

    corrected: displaced statistics with weight w; band-local: the band's own
    moments (as in a naive step); stale-only: displaced with w = 0, i.e. the
    previous step's whole-image moments; sync: the exact whole-image moments.
    """
    if mode != DISPLACED or gn_stats == GN_STATS_CORRECTED:
        return mode, w
    if gn_stats == GN_STATS_LOCAL:
        return NAIVE, w
    if gn_stats == GN_STATS_STALE:
        return DISPLACED, 0.0
    if gn_stats == GN_STATS_SYNC:
        return SYNC, w
    raise ValueError(gn_stats)


def _gn(st: GNState, x, gamma, beta, P, G, eps, w, silu, mode, trace, key, gn_stats=GN_STATS_CORRECTED):
    gmode, gw = gn_variant_mode(mode, w, gn_stats)
    y, f, used, nneg = groupnorm_async(x, gamma, beta, P, G, eps, gw, silu, gmode,
                                       st.stale_global, st.stale_local)
    if trace is not None:
        trace[key + ".fresh_local"] = f
        trace[key + ".used"] = used
        trace[key + ".fallbacks"] = nneg
    return y, f


def _a(x) -> np.ndarray:
    if isinstance(x, torch.Tensor):
        return x.detach().to(torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def gn_conv_step(state: Dict, x, wts: Dict, P: int, G: int, eps: float, w: float,
                 silu: bool, mode: int, storage: str, trace: Optional[Dict] = None,
                 final_storage: Optional[str] = None, gn_stats: int = GN_STATS_CORRECTED,
                 prefix: str = ""):
    """GroupNorm (+SiLU) -> 3x3 conv with stale halo.  x: (C, H, W)."""
    x = _a(x)
    gn = state.setdefault("gn", GNState())
    a, f = _gn(gn, x, _a(wts[prefix + "gn_gamma"]), _a(wts[prefix + "gn_beta"]), P, G, eps, w, silu,
               mode, trace, prefix + "gn", gn_stats)
    a = store(a, storage)
    out = conv3x3_halo(a, state.get("a_stale"), _a(wts[prefix + "conv_w"]), _a(wts[prefix + "conv_b"]),
                       None, P, mode)
    out = store(out, final_storage or storage)
    if trace is not None:
        trace[prefix + "a"] = a
    gn.refresh(f)
    state["a_stale"] = a
    return out


def time_embedding_term(temb, temb_w, temb_b) -> np.ndarray:
    """temb_w silu(temb) + temb_b: the per-channel term an SDXL ResBlock adds to its first
    conv's output (reading R13), with temb_w stored (out, in); temb_b may be None."""
    tv = _a(temb)
    return linear((tv / (1.0 + np.exp(-tv)))[None, :], _a(temb_w),
                  None if temb_b is None else _a(temb_b))[0]


def ddim_step(x, eps, abar_t: float, abar_prev: float) -> np.ndarray:
    """The sampler update between two denoising steps (reading R15): deterministic DDIM,
    eta = 0 (Song, Meng and Ermon, "Denoising Diffusion Implicit Models", section 4.1 with
    sigma = 0), the sampler of the pages' 50-step DDIM results (atlas.scime.ai summary, Key
    results).  The clean sample is predicted from x and the noise estimate, then put back at
    the previous timestep's noise level with the same noise estimate."""
    x, eps = _a(x), _a(eps)
    x0 = (x - math.sqrt(1.0 - abar_t) * eps) / math.sqrt(abar_t)
    return math.sqrt(abar_prev) * x0 + math.sqrt(1.0 - abar_prev) * eps


def dpm_solver_2m_step(x, eps, x0_prev, abar_prev: float, abar_s: float, abar_t: float):
    """One step of the multistep second-order DPM-Solver++ (reading R16; Lu, Zhou, Bao, Chen,
    Li and Zhu, "DPM-Solver++: Fast Solver for Guided Sampling of Diffusion Probabilistic
    Models", the multistep second-order solver in data prediction), the sampler of the pages'
    "10-step DPM-Solver" warm-up ablation (atlas.scime.ai summary).  Moves the latent x from
    the level abar_s to the less noisy level abar_t.  Returns (x_t, x0), x0 being this step's
    data prediction, which the next step takes as its x0_prev.

    With alpha = sqrt(abar), sigma = sqrt(1 - abar), lambda = log(alpha / sigma), h = lambda_t -
    lambda_s:  x0 = (x - sigma_s eps) / alpha_s;  D = x0 for a first-order step (x0_prev None or
    abar_prev <= 0, and the final step to abar_t = 1), otherwise D = x0 + (x0 - x0_prev) / (2 r)
    with r = (lambda_s - lambda_prev) / h;  x_t = (sigma_t / sigma_s) x - alpha_t (exp(-h) - 1) D.
    """
    x, eps = _a(x), _a(eps)
    a_s, s_s = math.sqrt(abar_s), math.sqrt(1.0 - abar_s)
    x0 = (x - s_s * eps) / a_s
    if abar_t >= 1.0:                      # the final step: the clean sample, first order
        return x0.copy(), x0
    a_t, s_t = math.sqrt(abar_t), math.sqrt(1.0 - abar_t)
    lam_s, lam_t = math.log(a_s / s_s), math.log(a_t / s_t)
    h = lam_t - lam_s
    D = x0
    if x0_prev is not None and abar_prev > 0.0:
        lam_p = math.log(math.sqrt(abar_prev) / math.sqrt(1.0 - abar_prev))
        r = (lam_s - lam_p) / h
        D = x0 + (x0 - _a(x0_prev)) / (2.0 * r)
    return (s_t / s_s) * x - a_t * (math.exp(-h) - 1.0) * D, x0


def resblock_step(state: Dict, x, wts: Dict, P: int, G: int, eps: float, w: float,
                  mode: int, storage: str, trace: Optional[Dict] = None, prefix: str = "",
                  final_storage: Optional[str] = None, gn_stats: int = GN_STATS_CORRECTED,
                  temb: Optional[np.ndarray] = None):
    """GN -> SiLU -> conv1 -> GN -> SiLU -> conv2 -> + x (or + 1x1 shortcut(x)).

    With a time embedding ``temb`` (and weights temb_w (Cout, Ct), temb_b), conv1's output
    gets the per-channel term temb_w silu(temb) + temb_b, as in an SDXL ResBlock (reading R13):
    a step-dependent bias that is the same for every band."""
    x = _a(x)
    W_ = lambda n: _a(wts[prefix + n])
    gn1 = state.setdefault("gn1", GNState())
    gn2 = state.setdefault("gn2", GNState())
    a1, f1 = _gn(gn1, x, W_("gn1_gamma"), W_("gn1_beta"), P, G, eps, w, True, mode, trace,
                 prefix + "gn1", gn_stats)
    a1 = store(a1, storage)
    b1 = W_("conv1_b")
    if temb is not None:
        b1 = b1 + time_embedding_term(temb, W_("temb_w"), W_("temb_b"))
    h = store(conv3x3_halo(a1, state.get("a1_stale"), W_("conv1_w"), b1, None, P, mode), storage)
    a2, f2 = _gn(gn2, h, W_("gn2_gamma"), W_("gn2_beta"), P, G, eps, w, True, mode, trace,
                 prefix + "gn2", gn_stats)
    a2 = store(a2, storage)
    if (prefix + "short_w") in wts:
        res = store(conv1x1(x, W_("short_w"), W_("short_b")), storage)
    else:
        res = x
    out = store(conv3x3_halo(a2, state.get("a2_stale"), W_("conv2_w"), W_("conv2_b"), res, P,
                             mode), final_storage or storage)
    if trace is not None:
        trace[prefix + "a1"], trace[prefix + "h"], trace[prefix + "a2"] = a1, h, a2
    gn1.refresh(f1)
    gn2.refresh(f2)
    state["a1_stale"], state["a2_stale"] = a1, a2
    return out


def attn_step(state: Dict, x, wts: Dict, P: int, G: int, eps: float, w: float, heads: int,
              mode: int, storage: str, trace: Optional[Dict] = None, prefix: str = "",
              final_storage: Optional[str] = None, gn_stats: int = GN_STATS_CORRECTED):
    """GN (no SiLU) -> q, k, v projections -> stale-K/V attention -> out proj + bias -> + x.

    x: (C, H, W); tokens are pixels in raster order, so band p's tokens are
    rows [p*H/P, (p+1)*H/P) of the image.
    """
    x = _a(x)
    C, H, Wd = x.shape
    W_ = lambda n: _a(wts[prefix + n])
    gn = state.setdefault("gn", GNState())
    a, f = _gn(gn, x, W_("gn_gamma"), W_("gn_beta"), P, G, eps, w, False, mode, trace,
               prefix + "gn", gn_stats)
    a = store(a, storage)
    tok = a.reshape(C, H * Wd).T                       # (T, C)
    q = store(linear(tok, W_("wq"), W_("bq")), storage)
    k = store(linear(tok, W_("wk"), W_("bk")), storage)
    v = store(linear(tok, W_("wv"), W_("bv")), storage)
    d = C // heads
    o = store(attention_stale_kv(q, k, v, state.get("k_stale"), state.get("v_stale"), P,
                                 heads, 1.0 / math.sqrt(d), mode), storage)
    out_tok = linear(o, W_("wo"), W_("bo")) + x.reshape(C, H * Wd).T
    out = store(out_tok.T.reshape(C, H, Wd), final_storage or storage)
    if trace is not None:
        trace[prefix + "a"], trace[prefix + "q"] = a, q
        trace[prefix + "k"], trace[prefix + "v"], trace[prefix + "o"] = k, v, o
    gn.refresh(f)
    state["k_stale"], state["v_stale"] = k, v
    return out


# --------------------------------------------------------------------------
# SDXL-shaped transformer block (a "next" extension beyond the hot path)
# --------------------------------------------------------------------------
# The pages name SDXL as the model DistriFusion runs but do not spell out its
# blocks.  Reading (R13): the plainest SDXL transformer block --
#   GroupNorm -> proj_in -> [LN -> self-attention] + -> [LN -> cross-attention
#   over the text context] + -> [LN -> GEGLU feed-forward] + -> proj_out -> + x
# Only the GroupNorm statistics and the self-attention keys/values cross
# bands, so only they are stale in displaced steps; LayerNorm, the
# cross-attention (the same text context for every band) and the feed-forward
# act on each token alone.

def layer_norm(x: np.ndarray, gamma: np.ndarray, beta: np.ndarray, eps: float) -> np.ndarray:
    """Per token (row of x: (T, C)): (x - mean) / sqrt(var + eps) * gamma + beta."""
    m = x.mean(axis=1, keepdims=True)
    v = ((x - m) ** 2).mean(axis=1, keepdims=True)
    return (x - m) / np.sqrt(v + eps) * gamma + beta


def gelu(x: np.ndarray) -> np.ndarray:
    """Exact GELU, x * Phi(x) = x (1 + erf(x / sqrt 2)) / 2."""
    return 0.5 * x * (1.0 + torch.special.erf(torch.from_numpy(np.asarray(x, dtype=np.float64)
                                                                / math.sqrt(2.0))).numpy())


def geglu_ff(x: np.ndarray, w1: np.ndarray, b1: np.ndarray, w2: np.ndarray,
             b2: np.ndarray) -> np.ndarray:
    """Feed-forward with a GELU-gated linear unit: [a | g] = x W1^T + b1 (two halves of the
    inner width), then (a * gelu(g)) W2^T + b2."""
    h = linear(x, w1, b1)
    inner = h.shape[1] // 2
    return linear(h[:, :inner] * gelu(h[:, inner:]), w2, b2)


def transformer_layer_name(layer: int, name: str) -> str:
    """Weight name of ``name`` in basic layer ``layer`` of a transformer block: the first
    layer's weights keep their plain names, layer l >= 1 prefixes them with "l<l>."."""
    return name if layer == 0 else f"l{layer}.{name}"


def transformer_step(state: Dict, x, ctx, wts: Dict, P: int, G: int, eps: float, w: float,
                     heads: int, mode: int, storage: str, trace: Optional[Dict] = None,
                     prefix: str = "", final_storage: Optional[str] = None,
                     gn_stats: int = GN_STATS_CORRECTED, ln_eps: float = 1e-5, depth: int = 1):
    """One SDXL-shaped transformer block (R13): GroupNorm, proj_in, ``depth`` basic layers
    (self-attention, cross-attention, gated feed-forward, each with a residual), proj_out
    and the block's residual.  x: (C, H, W) image; ctx: (Tk, Cctx) text context.  Tokens
    are pixels in raster order; band p's tokens are its rows.  Each layer's
    self-attention keeps its own stale keys and values."""
    x = _a(x)
    ctx = _a(ctx)
    C, H, Wd = x.shape
    W_ = lambda n: _a(wts[prefix + n])
    gn = state.setdefault("gn", GNState())
    a, f = _gn(gn, x, W_("gn_gamma"), W_("gn_beta"), P, G, eps, w, False, mode, trace,
               prefix + "gn", gn_stats)
    a = store(a, storage)
    h = store(linear(a.reshape(C, H * Wd).T, W_("proj_in_w"), W_("proj_in_b")), storage)
    d = C // heads
    fresh_kv = []
    for layer in range(depth):
        L = lambda n: W_(transformer_layer_name(layer, n))
        kv_key = transformer_layer_name(layer, "")
        # self-attention: keys and values of other bands are the previous step's
        t = store(layer_norm(h, L("ln1_g"), L("ln1_b"), ln_eps), storage)
        q = store(linear(t, L("wq"), L("bq")), storage)
        k = store(linear(t, L("wk"), L("bk")), storage)
        v = store(linear(t, L("wv"), L("bv")), storage)
        o = store(attention_stale_kv(q, k, v, state.get(kv_key + "k_stale"),
                                     state.get(kv_key + "v_stale"), P, heads,
                                     1.0 / math.sqrt(d), mode), storage)
        h = store(h + linear(o, L("wo"), L("bo")), storage)
        # cross-attention over the text context: the same for every band
        t = store(layer_norm(h, L("ln2_g"), L("ln2_b"), ln_eps), storage)
        q2 = store(linear(t, L("cq_w"), None), storage)
        k2 = store(linear(ctx, L("ck_w"), None), storage)
        v2 = store(linear(ctx, L("cv_w"), None), storage)
        o2 = store(attention_cross(q2, k2, v2, heads, 1.0 / math.sqrt(d)), storage)
        h = store(h + linear(o2, L("co_w"), L("co_b")), storage)
        # feed-forward
        t = store(layer_norm(h, L("ln3_g"), L("ln3_b"), ln_eps), storage)
        hf = store(linear(t, L("ff1_w"), L("ff1_b")), storage)   # geglu_ff, stored where the GPU stores
        inner = hf.shape[1] // 2
        gf = store(hf[:, :inner] * gelu(hf[:, inner:]), storage)
        h = store(h + linear(gf, L("ff2_w"), L("ff2_b")), storage)
        fresh_kv.append((kv_key, k, v))
    out_tok = linear(h, W_("proj_out_w"), W_("proj_out_b")) + x.reshape(C, H * Wd).T
    out = store(out_tok.T.reshape(C, H, Wd), final_storage or storage)
    gn.refresh(f)
    for kv_key, k, v in fresh_kv:
        if trace is not None:
            trace[prefix + kv_key + "k"], trace[prefix + kv_key + "v"] = k, v
        state[kv_key + "k_stale"], state[kv_key + "v_stale"] = k, v
    return out


def unet_mini_step(state: Dict, x, wts: Dict, P: int, G: int, eps: float, w: float,
                   mode: int, storage: str, trace: Optional[Dict] = None,
                   final_storage: Optional[str] = None, gn_stats: int = GN_STATS_CORRECTED):
    """conv_in -> ResBlock(320) -> down -> ResBlock(320->640) -> Attn(640, 10 heads)
    -> down -> ResBlock(640->1280) -> Attn(1280, 20 heads)   (reading R6/R7).

    Every 3x3 conv, conv_in and the stride-2 downsamplers included, takes its
    halo rows from the previous step's copy of its own input.
    """
    x = _a(x)
    A = lambda n: _a(wts[n])
    sub = lambda n: state.setdefault(n, {})

    def conv_layer(name, inp, wname, bname, stride):
        st = sub(name)
        y = conv3x3_halo(inp, st.get("a_stale"), A(wname), A(bname), None, P, mode, stride)
        st["a_stale"] = inp
        return store(y, storage)

    h = conv_layer("conv_in", x, "conv_in_w", "conv_in_b", 1)
    h = resblock_step(sub("rb1"), h, wts, P, G, eps, w, mode, storage, trace, "rb1.",
                      gn_stats=gn_stats)
    h = conv_layer("down1", h, "down1_w", "down1_b", 2)
    h = resblock_step(sub("rb2"), h, wts, P, G, eps, w, mode, storage, trace, "rb2.",
                      gn_stats=gn_stats)
    h = attn_step(sub("at2"), h, wts, P, G, eps, w, 10, mode, storage, trace, "at2.",
                  gn_stats=gn_stats)
    h = conv_layer("down2", h, "down2_w", "down2_b", 2)
    h = resblock_step(sub("rb3"), h, wts, P, G, eps, w, mode, storage, trace, "rb3.",
                      gn_stats=gn_stats)
    h = attn_step(sub("at3"), h, wts, P, G, eps, w, 20, mode, storage, trace, "at3.",
                  final_storage, gn_stats=gn_stats)
    return h


# ---------------------------------------------------------------- SDXL-shaped U-Net step
# Reading R18: the whole denoising network of the pages' SDXL experiments
# ("DistriFusion", atlas.scime.ai summary, Key results: SDXL at 1024 px and
# above), shaped as SDXL's U-Net: conv_in; three down levels of two ResBlocks
# (level widths base, 2 base, 4 base), the ResBlocks of levels with a nonzero
# transformer depth each followed by a transformer block of that depth, levels
# 0 and 1 ending in a stride-2 conv; a middle ResBlock -> transformer ->
# ResBlock (no transformer when the deepest level's depth is 0, as no
# transformer follows a ResBlock at a level of depth 0); three up levels of
# three ResBlocks, each taking the channel
# concatenation [h, skip] of the running tensor and the latest unused skip
# (the outputs of conv_in, of every down ResBlock/transformer pair and of the
# down convs), levels 2 and 1 ending in a nearest-neighbour 2x upsample and a
# 3x3 conv; then GroupNorm -> SiLU -> conv_out to the latent's channels.
# Every ResBlock adds the step's time embedding term.  Every 3x3 conv (conv_in,
# down, up and conv_out included) takes its halo rows from the previous step's
# copy of its own input; upsampling and concatenation act on each pixel's rows
# within its band, so they need no context.

def upsample_nearest2x(x) -> np.ndarray:
    """Nearest-neighbour 2x upsampling of (C, H, W): out[:, i, j] = x[:, i // 2, j // 2]."""
    x = _a(x)
    return np.repeat(np.repeat(x, 2, axis=1), 2, axis=2)


def concat_channels(a, b) -> np.ndarray:
    """Channel concatenation [a, b] of (Ca, H, W) and (Cb, H, W)."""
    return np.concatenate([_a(a), _a(b)], axis=0)


def sdxl_unet_step(state: Dict, x, ctx, temb, wts: Dict, P: int, G: int, eps: float, w: float,
                   mode: int, storage: str, base: int = 320, depths=(0, 2, 10), head_dim: int = 64,
                   ff_mult: int = 4, trace: Optional[Dict] = None, final_storage: Optional[str] = None,
                   gn_stats: int = GN_STATS_CORRECTED) -> np.ndarray:
    """One step of the SDXL-shaped U-Net (R18).  x: (Cl, H, W) latent; ctx: (Tk, Cctx) text
    context; temb: (Ct,) the step's time embedding.  Weight names: conv_in_*; d<l>.r<i>. and
    d<l>.t<i>. (down ResBlock / transformer i of level l), d<l>.down_*; mid.r0., mid.t.,
    mid.r1.; u<l>.r<i>., u<l>.t<i>., u<l>.up_*; out. (GroupNorm + conv_out).  Transformers
    have C / head_dim heads and a feed-forward inner width ff_mult * C."""
    x = _a(x)
    A = lambda n: _a(wts[n])
    sub = lambda n: state.setdefault(n, {})
    chans = (base, 2 * base, 4 * base)

    def conv_layer(name, inp, stride):
        st = sub(name)
        y = conv3x3_halo(inp, st.get("a_stale"), A(name + "_w"), A(name + "_b"), None, P, mode, stride)
        st["a_stale"] = inp
        return store(y, storage)

    def resblock(pre, h):
        return resblock_step(sub(pre), h, wts, P, G, eps, w, mode, storage, trace, pre,
                             gn_stats=gn_stats, temb=temb)

    def transformer(pre, h, depth):
        c = h.shape[0]
        return transformer_step(sub(pre), h, ctx, wts, P, G, eps, w, c // head_dim, mode, storage,
                                trace, pre, gn_stats=gn_stats, depth=depth)

    h = conv_layer("conv_in", x, 1)
    skips = [h]
    for lvl in range(3):
        for i in range(2):
            h = resblock(f"d{lvl}.r{i}.", h)
            if depths[lvl]:
                h = transformer(f"d{lvl}.t{i}.", h, depths[lvl])
            skips.append(h)
        if lvl < 2:
            h = conv_layer(f"d{lvl}.down", h, 2)
            skips.append(h)
    h = resblock("mid.r0.", h)
    if depths[2]:
        h = transformer("mid.t.", h, depths[2])
    h = resblock("mid.r1.", h)
    for lvl in (2, 1, 0):
        for i in range(3):
            h = resblock(f"u{lvl}.r{i}.", concat_channels(h, skips.pop()))
            if depths[lvl]:
                h = transformer(f"u{lvl}.t{i}.", h, depths[lvl])
        if lvl > 0:
            h = conv_layer(f"u{lvl}.up", upsample_nearest2x(h), 1)
    assert not skips
    return gn_conv_step(sub("out."), h, wts, P, G, eps, w, True, mode, storage, trace,
                        final_storage, gn_stats, prefix="out.")


def block_step(kind: str, state: Dict, x, wts: Dict, P: int, G: int, eps: float, w: float,
               mode: int, storage: str, heads: int = 0, silu: bool = True,
               trace: Optional[Dict] = None, final_storage: Optional[str] = None,
               gn_stats: int = GN_STATS_CORRECTED, ctx=None, depth: int = 1):
    """Dispatch one block step by kind; x is (C, H, W) (a leading batch of 1 is dropped);
    ``ctx`` is a transformer block's (Tk, Cctx) text context and ``depth`` its number of
    basic layers.

    ``final_storage`` (default: ``storage``) is the rounding of the block's
    output alone; intermediates always use ``storage``.
    """
    x = _a(x)
    if x.ndim == 4:
        x = x[0]
    if kind == "gn_conv":
        return gn_conv_step(state, x, wts, P, G, eps, w, silu, mode, storage, trace,
                            final_storage, gn_stats)
    if kind == "resblock":
        return resblock_step(state, x, wts, P, G, eps, w, mode, storage, trace,
                             final_storage=final_storage, gn_stats=gn_stats)
    if kind == "attn":
        return attn_step(state, x, wts, P, G, eps, w, heads, mode, storage, trace,
                         final_storage=final_storage, gn_stats=gn_stats)
    if kind == "transformer":
        return transformer_step(state, x, ctx, wts, P, G, eps, w, heads, mode, storage, trace,
                                final_storage=final_storage, gn_stats=gn_stats, depth=depth)
    if kind == "unet_mini":
        return unet_mini_step(state, x, wts, P, G, eps, w, mode, storage, trace, final_storage,
                              gn_stats)
    raise ValueError(kind)
