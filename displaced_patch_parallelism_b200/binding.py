"""ctypes binding of ``libdp.so``: argument marshalling only.

Every function here has the name and argument order of its C counterpart in
``include/dp.h``.  Tensors are passed as device pointers (``torch.Tensor`` on a
CUDA device, an ``int`` address, or ``None`` for NULL); ``stream=None`` means
torch's current CUDA stream.  A non-zero status raises ``DPError``.  There is
no fallback: if the library is missing or a call fails, the caller sees it.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG_DIR, "libdp.so")

DP_OK, DP_ERR_INVALID_ARG, DP_ERR_UNSUPPORTED, DP_ERR_STATE, DP_ERR_CUDA, DP_ERR_TIMEOUT = 0, -1, -2, -3, -4, -5
SYNC, DISPLACED, NAIVE = 0, 1, 2
BF16, FP32 = 0, 1
GN_CONV, RESBLOCK, ATTN, UNET_MINI, TRANSFORMER, UNET_SDXL = 0, 1, 2, 3, 4, 5
GN_STATS_CORRECTED, GN_STATS_LOCAL, GN_STATS_STALE, GN_STATS_SYNC = 0, 1, 2, 3

ERR_NAMES = {DP_ERR_INVALID_ARG: "DP_ERR_INVALID_ARG", DP_ERR_UNSUPPORTED: "DP_ERR_UNSUPPORTED",
             DP_ERR_STATE: "DP_ERR_STATE", DP_ERR_CUDA: "DP_ERR_CUDA",
             DP_ERR_TIMEOUT: "DP_ERR_TIMEOUT"}


class DPError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{ERR_NAMES.get(code, code)}: {msg}")
        self.code = code


class BlockDesc(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int), ("H", ctypes.c_int), ("W", ctypes.c_int),
                ("C", ctypes.c_int), ("Cout", ctypes.c_int), ("G", ctypes.c_int),
                ("P", ctypes.c_int), ("heads", ctypes.c_int), ("dtype", ctypes.c_int),
                ("silu", ctypes.c_int), ("eps", ctypes.c_float), ("w", ctypes.c_float),
                ("gn_stats", ctypes.c_int), ("ctx_len", ctypes.c_int), ("ctx_dim", ctypes.c_int),
                ("ff_inner", ctypes.c_int), ("temb_dim", ctypes.c_int), ("gn_fuse", ctypes.c_int),
                ("depth", ctypes.c_int), ("unet_base", ctypes.c_int),
                ("unet_depth", ctypes.c_int * 3), ("ctx_fixed", ctypes.c_int)]


class BlockState(ctypes.Structure):
    _fields_ = [("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
                ("cur", ctypes.c_int), ("steps_done", ctypes.c_int)]


_V, _I, _F, _SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
_SIGS = {
    "dp_last_error": ([], ctypes.c_char_p),
    "dp_version": ([], ctypes.c_char_p),
    "dp_mode_for_step": ([_I, _I], _I),
    "dp_device_status": ([_V, ctypes.POINTER(_I)], _I),
    "dp_selftest_bounded_wait": ([_I, ctypes.c_uint, _V], _I),
    "dp_block_status": ([ctypes.POINTER(BlockDesc), ctypes.POINTER(BlockState), _V,
                         ctypes.POINTER(_I)], _I),
    "dp_groupnorm_workspace_size": ([_I, _I, _I, _I, _I], _SZ),
    "dp_groupnorm_async": ([_V, _V, _V, _V, _I, _I, _I, _I, _I, _F, _F, _I, _I, _I, _V, _V, _V, _V,
                            _V, _SZ, _V], _I),
    "dp_groupnorm_async_noalloc": ([_V, _V, _V, _V, _I, _I, _I, _I, _I, _F, _F, _I, _I, _I, _V, _V,
                                    _V, _V, _V], _I),
    "dp_gemm_workspace_size": ([], _SZ),
    "dp_groupnorm_stats": ([_V, _I, _I, _I, _I, _I, _F, _I, _I, _V, _V, _V, _V, _V, _SZ, _V], _I),
    "dp_conv3x3_halo_gn": ([_V, _V, _V, _V, _V, _V, _I, _F, _I, _V, _V, _V, _V, _I, _I, _I, _I, _I, _I,
                            _V], _I),
    "dp_conv3x3_halo": ([_V, _V, _V, _V, _V, _V, _I, _I, _I, _I, _I, _I, _I, _I, _V, _SZ, _V], _I),
    "dp_conv3x3_halo_small": ([_V, _V, _V, _V, _V, _I, _I, _I, _I, _I, _I, _V], _I),
    "dp_linear": ([_V, _V, _V, _V, _V, _V, _V, _I, _I, _I, _I, _V, _SZ, _V], _I),
    "dp_attn_workspace_size": ([], _SZ),
    "dp_attn_stale_kv": ([_V, _V, _V, _V, _V, _V, _I, _I, _I, _I, _F, _I, _V, _SZ, _V], _I),
    "dp_attn_cross": ([_V, _V, _V, _V, _I, _I, _I, _I, _F, _V, _SZ, _V], _I),
    "dp_layernorm": ([_V, _V, _V, _V, _I, _I, _F, _V], _I),
    "dp_geglu": ([_V, _V, _I, _I, _V], _I),
    "dp_concat_channels": ([_V, _V, _V, ctypes.c_size_t, _I, _I, _I, _V], _I),
    "dp_linear_geglu": ([_V, _V, _V, _V, _I, _I, _I, _V], _I),
    "dp_upsample_nearest2x": ([_V, _V, _I, _I, _I, _I, _V], _I),
    "dp_time_embedding_bias": ([_V, _V, _V, _V, _V, _I, _I, _V], _I),
    "dp_ddim_step": ([_V, _V, _V, _SZ, ctypes.c_double, ctypes.c_double, _I, _V], _I),
    "dp_dpm_solver_step": ([_V, _V, _V, _V, _SZ, ctypes.c_double, ctypes.c_double, ctypes.c_double, _I, _V],
                           _I),
    "dp_refresh_stale": ([_V, _V, _SZ, _I, _I, _I, _V], _I),
    "dp_refresh_halo": ([_V, _V, _SZ, _I, _I, _I, _I, _V], _I),
    "dp_refresh_stats": ([_V, _V, _V, _I, _I, _V], _I),
    "dp_block_desc_init": ([ctypes.POINTER(BlockDesc), _I, _I, _I, _I, _I, _I, _I, _I, _I, _I, _F, _F], _I),
    "dp_block_desc_set_gn_stats": ([ctypes.POINTER(BlockDesc), _I], _I),
    "dp_block_desc_set_gn_fusion": ([ctypes.POINTER(BlockDesc), _I], _I),
    "dp_block_desc_set_context": ([ctypes.POINTER(BlockDesc), _I, _I, _I], _I),
    "dp_block_desc_set_depth": ([ctypes.POINTER(BlockDesc), _I], _I),
    "dp_block_desc_set_unet": ([ctypes.POINTER(BlockDesc), _I, _I, _I, _I], _I),
    "dp_block_desc_set_context_fixed": ([ctypes.POINTER(BlockDesc), _I], _I),
    "dp_block_desc_set_time_embedding": ([ctypes.POINTER(BlockDesc), _I], _I),
    "dp_block_workspace_size": ([ctypes.POINTER(BlockDesc)], _SZ),
    "dp_block_state_init": ([ctypes.POINTER(BlockDesc), ctypes.POINTER(BlockState), _V, _SZ, _V], _I),
    "dp_block_graph_create": ([ctypes.POINTER(BlockDesc), ctypes.POINTER(BlockState), _V, _V,
                               ctypes.POINTER(ctypes.c_void_p), _I, _I, _V, ctypes.POINTER(ctypes.c_void_p)], _I),
    "dp_block_graph_launch": ([_V, ctypes.POINTER(BlockState), _V], _I),
    "dp_block_graph_destroy": ([_V], _I),
    "dp_block_step": ([ctypes.POINTER(BlockDesc), ctypes.POINTER(BlockState), _V, _V,
                       ctypes.POINTER(_V), _I, _I, _V], _I),
    "dp_block_flops": ([ctypes.POINTER(BlockDesc)], ctypes.c_double),
    "dp_block_launch_count": ([ctypes.POINTER(BlockDesc)], _I),
    "dp_block_weight_count": ([ctypes.POINTER(BlockDesc)], _I),
    "dp_block_launch_info": ([ctypes.POINTER(BlockDesc), _I, _I, ctypes.POINTER(_I),
                              ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double)], _I),
    "dp_block_step_timed": ([ctypes.POINTER(BlockDesc), ctypes.POINTER(BlockState), _V, _V,
                             ctypes.POINTER(_V), _I, _I, _V, ctypes.POINTER(_V), _I], _I),
}

_LIB = None


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it has not been built."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built: run `python -m displaced_patch_parallelism_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGS.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _LIB = L
    return _LIB


def _p(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _s(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(rc: int) -> int:
    if rc != DP_OK:
        raise DPError(rc, lib().dp_last_error().decode())
    return rc


def dp_version() -> str:
    return lib().dp_version().decode()


def dp_mode_for_step(step: int, warmup: int) -> int:
    rc = lib().dp_mode_for_step(step, warmup)
    if rc < 0:
        _check(rc)
    return rc


def dp_device_status(stream=None) -> int:
    st = ctypes.c_int(0)
    _check(lib().dp_device_status(_s(stream), ctypes.byref(st)))
    return st.value


SELFTEST_WAIT_MBARRIER, SELFTEST_WAIT_FLAG = 0, 1


def dp_selftest_bounded_wait(kind, limit_us, stream=None):
    return _check(lib().dp_selftest_bounded_wait(kind, limit_us, _s(stream)))


def dp_block_status(d: "BlockDesc", s: "BlockState", stream=None) -> int:
    st = ctypes.c_int(0)
    _check(lib().dp_block_status(ctypes.byref(d), ctypes.byref(s), _s(stream), ctypes.byref(st)))
    return st.value


def dp_groupnorm_workspace_size(H, W, C, G, P) -> int:
    return lib().dp_groupnorm_workspace_size(H, W, C, G, P)


def dp_groupnorm_async(x, y, gamma, beta, H, W, C, G, P, eps, w, silu, mode, dtype, stale_global,
                       stale_local, fresh_local, used_stats, workspace, workspace_bytes=None,
                       stream=None):
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    return _check(lib().dp_groupnorm_async(
        _p(x), _p(y), _p(gamma), _p(beta), H, W, C, G, P, eps, w, int(silu), mode, dtype,
        _p(stale_global), _p(stale_local), _p(fresh_local), _p(used_stats), _p(workspace),
        workspace_bytes, _s(stream)))


def dp_groupnorm_async_noalloc(x, y, gamma, beta, H, W, C, G, P, eps, w, silu, mode, dtype,
                               stale_global, stale_local, fresh_local, used_stats, stream=None):
    return _check(lib().dp_groupnorm_async_noalloc(
        _p(x), _p(y), _p(gamma), _p(beta), H, W, C, G, P, eps, w, int(silu), mode, dtype,
        _p(stale_global), _p(stale_local), _p(fresh_local), _p(used_stats), _s(stream)))


def dp_gemm_workspace_size():
    return lib().dp_gemm_workspace_size()


def dp_conv3x3_halo(a_fresh, a_stale, weight, bias, residual, out, H, W, Cin, Cout, stride, P,
                    mode, dtype, workspace=None, workspace_bytes=0, stream=None):
    return _check(lib().dp_conv3x3_halo(_p(a_fresh), _p(a_stale), _p(weight), _p(bias),
                                        _p(residual), _p(out), H, W, Cin, Cout, stride, P, mode,
                                        dtype, _p(workspace), workspace_bytes, _s(stream)))


def dp_conv3x3_halo_small(a_fresh, a_stale, weight, bias, out, H, W, Cin, Cout, P, mode,
                          stream=None):
    return _check(lib().dp_conv3x3_halo_small(_p(a_fresh), _p(a_stale), _p(weight), _p(bias),
                                              _p(out), H, W, Cin, Cout, P, mode, _s(stream)))


def dp_groupnorm_stats(x, H, W, C, G, P, w, mode, dtype, stale_global, stale_local, fresh_local,
                       used_stats, workspace, workspace_bytes=None, stream=None):
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    return _check(lib().dp_groupnorm_stats(_p(x), H, W, C, G, P, w, mode, dtype, _p(stale_global),
                                           _p(stale_local), _p(fresh_local), _p(used_stats),
                                           _p(workspace), workspace_bytes, _s(stream)))


def dp_conv3x3_halo_gn(x, a_stale, a_next, used_stats, gamma, beta, G, eps, silu, weight, bias,
                       residual, out, H, W, Cin, Cout, P, mode, stream=None):
    return _check(lib().dp_conv3x3_halo_gn(_p(x), _p(a_stale), _p(a_next), _p(used_stats), _p(gamma),
                                           _p(beta), G, eps, int(silu), _p(weight), _p(bias),
                                           _p(residual), _p(out), H, W, Cin, Cout, P, mode, _s(stream)))


def dp_linear(x, weight, bias, residual, out0, out1, out2, M, N, K, split, workspace=None,
              workspace_bytes=0, stream=None):
    return _check(lib().dp_linear(_p(x), _p(weight), _p(bias), _p(residual), _p(out0), _p(out1),
                                  _p(out2), M, N, K, split, _p(workspace), workspace_bytes,
                                  _s(stream)))


def dp_attn_workspace_size():
    return lib().dp_attn_workspace_size()


def dp_attn_stale_kv(q, k_fresh, v_fresh, k_stale, v_stale, o, T, heads, head_dim, P, scale,
                     mode, workspace=None, workspace_bytes=0, stream=None):
    return _check(lib().dp_attn_stale_kv(_p(q), _p(k_fresh), _p(v_fresh), _p(k_stale),
                                         _p(v_stale), _p(o), T, heads, head_dim, P, scale, mode,
                                         _p(workspace), workspace_bytes, _s(stream)))


def dp_attn_cross(q, k, v, o, Tq, Tk, heads, head_dim, scale, workspace=None, workspace_bytes=0,
                  stream=None):
    return _check(lib().dp_attn_cross(_p(q), _p(k), _p(v), _p(o), Tq, Tk, heads, head_dim, scale,
                                      _p(workspace), workspace_bytes, _s(stream)))


def dp_layernorm(x, y, gamma, beta, T, C, eps, stream=None):
    return _check(lib().dp_layernorm(_p(x), _p(y), _p(gamma), _p(beta), T, C, eps, _s(stream)))


def dp_geglu(h, y, T, F, stream=None):
    return _check(lib().dp_geglu(_p(h), _p(y), T, F, _s(stream)))


def dp_linear_geglu(x, weight, bias, y, M, F, K, stream=None):
    return _check(lib().dp_linear_geglu(_p(x), _p(weight), _p(bias), _p(y), M, F, K, _s(stream)))


def dp_concat_channels(a, b, out, npix, Ca, Cb, dtype=BF16, stream=None):
    return _check(lib().dp_concat_channels(_p(a), _p(b), _p(out), npix, Ca, Cb, dtype, _s(stream)))


def dp_upsample_nearest2x(x, out, H, W, C, dtype=BF16, stream=None):
    return _check(lib().dp_upsample_nearest2x(_p(x), _p(out), H, W, C, dtype, _s(stream)))


def dp_time_embedding_bias(temb, temb_w, temb_b, conv_b, bias, Ct, Cout, stream=None):
    return _check(lib().dp_time_embedding_bias(_p(temb), _p(temb_w), _p(temb_b), _p(conv_b),
                                               _p(bias), Ct, Cout, _s(stream)))


def dp_ddim_step(x, eps, x_prev, n, abar_t, abar_prev, dtype, stream=None):
    return _check(lib().dp_ddim_step(_p(x), _p(eps), _p(x_prev), n, abar_t, abar_prev, dtype,
                                     _s(stream)))


def dp_dpm_solver_step(x, eps, x0_buf, x_next, n, abar_prev, abar_s, abar_t, dtype, stream=None):
    return _check(lib().dp_dpm_solver_step(_p(x), _p(eps), _p(x0_buf), _p(x_next), n, abar_prev, abar_s,
                                           abar_t, dtype, _s(stream)))


def dp_refresh_stale(fresh, stale, row_bytes, rows, P, band=-1, stream=None):
    return _check(lib().dp_refresh_stale(_p(fresh), _p(stale), row_bytes, rows, P, band,
                                         _s(stream)))


def dp_refresh_halo(fresh, stale, row_bytes, rows, P, above, below, stream=None):
    return _check(lib().dp_refresh_halo(_p(fresh), _p(stale), row_bytes, rows, P, above, below,
                                        _s(stream)))


def dp_refresh_stats(fresh_local, stale_local, stale_global, P, G, stream=None):
    return _check(lib().dp_refresh_stats(_p(fresh_local), _p(stale_local), _p(stale_global), P, G,
                                         _s(stream)))


def dp_block_desc_init(kind, H, W, C, Cout, G, P, heads, dtype, silu, eps, w) -> BlockDesc:
    d = BlockDesc()
    _check(lib().dp_block_desc_init(ctypes.byref(d), kind, H, W, C, Cout, G, P, heads, dtype,
                                    int(silu), eps, w))
    return d


def dp_block_desc_set_gn_stats(d: BlockDesc, variant: int):
    return _check(lib().dp_block_desc_set_gn_stats(ctypes.byref(d), variant))


def dp_block_desc_set_gn_fusion(d: BlockDesc, on: int):
    return _check(lib().dp_block_desc_set_gn_fusion(ctypes.byref(d), int(on)))


def dp_block_desc_set_context(d: BlockDesc, ctx_len: int, ctx_dim: int, ff_inner: int):
    return _check(lib().dp_block_desc_set_context(ctypes.byref(d), ctx_len, ctx_dim, ff_inner))


def dp_block_desc_set_depth(d: BlockDesc, depth: int):
    return _check(lib().dp_block_desc_set_depth(ctypes.byref(d), depth))


def dp_block_desc_set_context_fixed(d: BlockDesc, on: bool):
    return _check(lib().dp_block_desc_set_context_fixed(ctypes.byref(d), int(on)))


def dp_block_desc_set_unet(d: BlockDesc, base: int, depth0: int, depth1: int, depth2: int):
    return _check(lib().dp_block_desc_set_unet(ctypes.byref(d), base, depth0, depth1, depth2))


def dp_block_desc_set_time_embedding(d: BlockDesc, temb_dim: int):
    return _check(lib().dp_block_desc_set_time_embedding(ctypes.byref(d), temb_dim))


def dp_block_workspace_size(d: BlockDesc) -> int:
    n = lib().dp_block_workspace_size(ctypes.byref(d))
    if n == 0:
        raise DPError(DP_ERR_INVALID_ARG, lib().dp_last_error().decode())
    return n


def dp_block_state_init(d: BlockDesc, workspace, workspace_bytes=None, stream=None) -> BlockState:
    s = BlockState()
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    _check(lib().dp_block_state_init(ctypes.byref(d), ctypes.byref(s), _p(workspace),
                                     workspace_bytes, _s(stream)))
    return s


def dp_block_step(d: BlockDesc, s: BlockState, x, out, weights: Sequence, mode: int, stream=None):
    arr = (ctypes.c_void_p * len(weights))(*[_p(w) for w in weights])
    return _check(lib().dp_block_step(ctypes.byref(d), ctypes.byref(s), _p(x), _p(out), arr,
                                      len(weights), mode, _s(stream)))


def dp_block_graph_create(d: BlockDesc, s: BlockState, x, out, weights: Sequence, mode: int,
                          stream=None) -> int:
    """The opaque graph handle (an address) of one captured step per ping-pong parity."""
    arr = (ctypes.c_void_p * len(weights))(*[_p(w) for w in weights])
    h = ctypes.c_void_p(0)
    _check(lib().dp_block_graph_create(ctypes.byref(d), ctypes.byref(s), _p(x), _p(out), arr, len(weights),
                                       mode, _s(stream), ctypes.byref(h)))
    return h.value


def dp_block_graph_launch(graph: int, s: BlockState, stream=None):
    return _check(lib().dp_block_graph_launch(graph, ctypes.byref(s), _s(stream)))


def dp_block_graph_destroy(graph: int):
    return _check(lib().dp_block_graph_destroy(graph))


def dp_block_launch_count(d: BlockDesc) -> int:
    n = lib().dp_block_launch_count(ctypes.byref(d))
    if n < 0:
        _check(n)
    return n


def dp_block_step_timed(d: BlockDesc, s: BlockState, x, out, weights: Sequence, mode: int, events,
                        stream=None):
    """``events``: torch.cuda.Event objects (timing enabled), at least launches + 1."""
    arr = (ctypes.c_void_p * len(weights))(*[_p(w) for w in weights])
    handles = [e.cuda_event for e in events]
    if not all(handles):
        raise ValueError("events must be created before use (record each once first)")
    ev = (ctypes.c_void_p * len(events))(*handles)
    return _check(lib().dp_block_step_timed(ctypes.byref(d), ctypes.byref(s), _p(x), _p(out), arr,
                                            len(weights), mode, _s(stream), ev, len(events)))


KERNEL_NAMES = {0: "gn_stats", 1: "gn_apply", 2: "gn_fused", 3: "conv", 4: "linear", 5: "attn",
                6: "copy", 7: "conv_small", 8: "splitk_finish",
                9: "gn_cluster", 10: "layernorm", 11: "geglu", 12: "temb", 13: "conv_gn", 14: "conv_f32",
                15: "conv_narrow", 16: "concat", 17: "upsample"}


def dp_block_launch_info(d: BlockDesc, mode: int, i: int):
    """(kernel name, algorithmic flops, algorithmic bytes) of launch i."""
    k, f, b = ctypes.c_int(0), ctypes.c_double(0), ctypes.c_double(0)
    _check(lib().dp_block_launch_info(ctypes.byref(d), mode, i, ctypes.byref(k), ctypes.byref(f),
                                      ctypes.byref(b)))
    return KERNEL_NAMES[k.value], f.value, b.value


def dp_block_weight_count(d: BlockDesc) -> int:
    n = lib().dp_block_weight_count(ctypes.byref(d))
    if n < 0:
        _check(n)
    return n


def dp_block_flops(d: BlockDesc) -> float:
    return lib().dp_block_flops(ctypes.byref(d))


class Block:
    """A block descriptor, its device workspace (a torch uint8 tensor) and its state."""

    def __init__(self, kind, H, W, C, Cout=0, G=32, P=4, heads=0, dtype=BF16, silu=True,
                 eps=1e-5, w=1.0, device="cuda", stream=None, gn_stats=GN_STATS_CORRECTED,
                 context=None, temb_dim=0, gn_fuse=False, depth=1, unet=None, context_fixed=False):
        """``context`` = (ctx_len, ctx_dim, ff_inner) for TRANSFORMER and UNET_SDXL blocks;
        ``temb_dim`` the time-embedding width of a RESBLOCK or UNET_SDXL (0: none); ``unet`` =
        (base, depth0, depth1, depth2) of a UNET_SDXL block."""
        import torch
        self.desc = dp_block_desc_init(kind, H, W, C, Cout, G, P, heads, dtype, silu, eps, w)
        if unet is not None:
            dp_block_desc_set_unet(self.desc, *unet)
        if context is not None:
            dp_block_desc_set_context(self.desc, *context)
        if depth != 1:
            dp_block_desc_set_depth(self.desc, depth)
        if context_fixed:
            dp_block_desc_set_context_fixed(self.desc, True)
        if temb_dim:
            dp_block_desc_set_time_embedding(self.desc, temb_dim)
        if gn_stats != GN_STATS_CORRECTED:
            dp_block_desc_set_gn_stats(self.desc, gn_stats)
        if gn_fuse:
            dp_block_desc_set_gn_fusion(self.desc, 1)
        self.ws_bytes = dp_block_workspace_size(self.desc)
        self.workspace = torch.empty(self.ws_bytes, dtype=torch.uint8, device=device)
        self.state = dp_block_state_init(self.desc, self.workspace, self.ws_bytes, stream)

    def step(self, x, out, weights, mode, stream=None):
        return dp_block_step(self.desc, self.state, x, out, weights, mode, stream)

    def graph(self, x, out, weights, mode, stream):
        """One captured step per ping-pong parity with these arguments; launch() runs the
        state's next step from it (see dp_block_graph_create)."""
        return BlockGraph(self, dp_block_graph_create(self.desc, self.state, x, out, weights, mode, stream))

    def step_timed(self, x, out, weights, mode, events, stream=None):
        return dp_block_step_timed(self.desc, self.state, x, out, weights, mode, events, stream)

    def status(self, stream=None) -> int:
        """Reads and clears this block's own device status word (DP_OK or DP_ERR_TIMEOUT)."""
        return dp_block_status(self.desc, self.state, stream)

    @property
    def launches(self) -> int:
        return dp_block_launch_count(self.desc)

    @property
    def flops(self) -> float:
        return dp_block_flops(self.desc)


class BlockGraph:
    """A block's captured steps; launch() replays the state's next one."""

    def __init__(self, block: Block, handle: int):
        self.block, self.handle = block, handle

    def launch(self, stream=None):
        return dp_block_graph_launch(self.handle, self.block.state, stream)

    def close(self):
        if self.handle:
            dp_block_graph_destroy(self.handle)
            self.handle = 0

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
