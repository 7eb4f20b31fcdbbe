"""C-ABI checks that need no GPU: the library loads, exports every declared
symbol, and rejects bad arguments on the host before touching CUDA."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def B():
    from displaced_patch_parallelism_b200 import binding
    if not os.path.exists(binding.LIB_PATH):
        from displaced_patch_parallelism_b200 import build
        build.build()
    binding.lib()
    return binding


def declared_symbols():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            text = open(os.path.join(ROOT, "include", h)).read()
            names += re.findall(r"^DP_API\s+[\w\s\*]+?\b(dp_\w+)\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_block_calls():
    names = declared_symbols()
    for n in ("dp_groupnorm_async", "dp_conv3x3_halo", "dp_attn_stale_kv", "dp_refresh_stale",
              "dp_block_step"):
        assert n in names


def test_every_declared_symbol_is_exported(B):
    lib = ctypes.CDLL(B.LIB_PATH)
    missing = [n for n in declared_symbols() if not hasattr(lib, n)]
    assert not missing, missing


def test_mode_for_step(B):
    assert B.dp_mode_for_step(0, 0) == B.NAIVE
    assert B.dp_mode_for_step(0, 4) == B.SYNC
    assert B.dp_mode_for_step(3, 4) == B.SYNC
    assert B.dp_mode_for_step(4, 4) == B.DISPLACED
    assert B.dp_mode_for_step(1, 0) == B.DISPLACED
    with pytest.raises(B.DPError):
        B.dp_mode_for_step(-1, 0)


def test_mode_for_step_matches_input_module(B):
    from displaced_patch_parallelism_b200 import synth
    for w in range(4):
        for s in range(8):
            assert B.dp_mode_for_step(s, w) == synth.mode_for_step(s, w)


def test_block_desc_validation(B):
    d = B.dp_block_desc_init(B.RESBLOCK, 128, 128, 320, 320, 32, 4, 0, B.BF16, 1, 1e-5, 1.0)
    assert B.dp_block_workspace_size(d) > 4 * 128 * 128 * 320 * 2
    # a GroupNorm whose tensor fits in shared memory is one launch: one cluster
    # per band in displaced steps, a grid-wide single pass in sync steps
    assert [B.dp_block_launch_info(d, B.DISPLACED, i)[0] for i in range(B.dp_block_launch_count(d))] \
        == ["gn_cluster", "conv", "gn_cluster", "conv"]
    assert [B.dp_block_launch_info(d, B.SYNC, i)[0] for i in range(B.dp_block_launch_count(d))] \
        == ["gn_fused", "conv", "gn_fused", "conv"]
    assert abs(B.dp_block_flops(d) - 2 * 2 * 128 * 128 * 320 * 9 * 320) < 1
    assert abs(sum(B.dp_block_launch_info(d, B.DISPLACED, i)[1] for i in range(4))
               - B.dp_block_flops(d)) < 1
    d2 = B.dp_block_desc_init(B.RESBLOCK, 64, 64, 320, 640, 32, 4, 0, B.BF16, 1, 1e-5, 1.0)
    assert [B.dp_block_launch_info(d2, B.SYNC, i)[0] for i in range(B.dp_block_launch_count(d2))] \
        == ["gn_fused", "conv", "gn_fused", "linear", "conv"]
    da = B.dp_block_desc_init(B.ATTN, 64, 64, 640, 640, 32, 4, 10, B.BF16, 0, 1e-5, 1.0)
    assert [B.dp_block_launch_info(da, B.DISPLACED, i)[0] for i in range(B.dp_block_launch_count(da))] \
        == ["gn_cluster", "linear", "attn", "linear"]
    # naive attention sees only its own band's keys
    assert B.dp_block_launch_info(da, B.NAIVE, 2)[1] * 4 == B.dp_block_launch_info(da, B.DISPLACED, 2)[1]
    # the 480x480 tensor does not fit on chip: two GroupNorm passes
    d4 = B.dp_block_desc_init(B.GN_CONV, 480, 480, 320, 320, 32, 8, 0, B.BF16, 1, 1e-5, 1.0)
    assert [B.dp_block_launch_info(d4, B.DISPLACED, i)[0] for i in range(B.dp_block_launch_count(d4))] \
        == ["gn_stats", "gn_apply", "conv"]
    # the 1280-channel convs at 32x32 have 16 output tiles for 74 SM pairs: K is
    # split into runs and a finish kernel adds them
    d5 = B.dp_block_desc_init(B.RESBLOCK, 32, 32, 640, 1280, 32, 4, 0, B.BF16, 1, 1e-5, 1.0)
    assert [B.dp_block_launch_info(d5, B.DISPLACED, i)[0] for i in range(B.dp_block_launch_count(d5))] \
        == ["gn_cluster", "conv", "splitk_finish", "gn_cluster", "linear", "conv", "splitk_finish"]
    du = B.dp_block_desc_init(B.UNET_MINI, 128, 128, 4, 0, 32, 4, 0, B.BF16, 1, 1e-5, 1.0)
    assert B.dp_block_weight_count(du) == 46
    assert abs(B.dp_block_flops(du) - sum(B.dp_block_launch_info(du, B.DISPLACED, i)[1]
                                          for i in range(B.dp_block_launch_count(du)))) < 1
    bad = [
        (B.RESBLOCK, 130, 128, 320, 320, 32, 4, 0, B.BF16, B.DP_ERR_UNSUPPORTED),   # H % P
        (B.RESBLOCK, 128, 128, 320, 320, 33, 4, 0, B.BF16, B.DP_ERR_UNSUPPORTED),   # C % G
        (B.ATTN, 64, 64, 640, 640, 32, 4, 9, B.BF16, B.DP_ERR_UNSUPPORTED),         # heads*64 != C
        (B.ATTN, 8, 8, 128, 128, 32, 4, 2, B.BF16, B.DP_ERR_UNSUPPORTED),           # 16 tokens/band
        (B.RESBLOCK, 64, 64, 64, 64, 32, 4, 0, B.FP32, B.DP_ERR_UNSUPPORTED),       # fp32 resblock
        (7, 64, 64, 64, 64, 32, 4, 0, B.BF16, B.DP_ERR_INVALID_ARG),                # kind
        (B.GN_CONV, 0, 64, 64, 64, 32, 4, 0, B.BF16, B.DP_ERR_INVALID_ARG),         # H = 0
    ]
    for kind, H, W, C, Co, G, P, heads, dt, code in bad:
        with pytest.raises(B.DPError) as e:
            B.dp_block_desc_init(kind, H, W, C, Co, G, P, heads, dt, 1, 1e-5, 1.0)
        assert e.value.code == code, (kind, H, W, C, G, P, heads)


def test_kernel_calls_reject_bad_arguments_on_the_host(B):
    # null pointers and unsupported shapes return before any CUDA call
    with pytest.raises(B.DPError) as e:
        B.dp_conv3x3_halo(None, None, None, None, None, None, 8, 8, 64, 64, 1, 2, B.SYNC, B.BF16, stream=0)
    assert e.value.code == B.DP_ERR_INVALID_ARG
    with pytest.raises(B.DPError) as e:   # Cin not a multiple of 64
        B.dp_conv3x3_halo(16, 16, 16, None, None, 32, 8, 8, 48, 64, 1, 2, B.SYNC, B.BF16, stream=0)
    assert e.value.code == B.DP_ERR_UNSUPPORTED
    with pytest.raises(B.DPError) as e:   # stride 3
        B.dp_conv3x3_halo(16, 16, 16, None, None, 32, 8, 8, 64, 64, 3, 2, B.SYNC, B.BF16, stream=0)
    assert e.value.code == B.DP_ERR_UNSUPPORTED
    with pytest.raises(B.DPError) as e:   # displaced without the stale buffer
        B.dp_conv3x3_halo(16, None, 16, None, None, 32, 8, 8, 64, 64, 1, 2, B.DISPLACED, B.BF16, stream=0)
    assert e.value.code == B.DP_ERR_INVALID_ARG
    with pytest.raises(B.DPError) as e:   # misaligned pointer
        B.dp_conv3x3_halo(18, 16, 16, None, None, 32, 8, 8, 64, 64, 1, 2, B.SYNC, B.BF16, stream=0)
    assert e.value.code == B.DP_ERR_UNSUPPORTED
    with pytest.raises(B.DPError) as e:   # head_dim 128
        B.dp_attn_stale_kv(16, 16, 16, 16, 16, 32, 256, 2, 128, 2, 0.1, B.SYNC, stream=0)
    assert e.value.code == B.DP_ERR_UNSUPPORTED
    with pytest.raises(B.DPError) as e:   # band of 96 tokens
        B.dp_attn_stale_kv(16, 16, 16, 16, 16, 32, 192, 2, 64, 2, 0.1, B.SYNC, stream=0)
    assert e.value.code == B.DP_ERR_UNSUPPORTED
    with pytest.raises(B.DPError) as e:   # o aliases q
        B.dp_attn_stale_kv(16, 32, 48, 64, 80, 16, 256, 2, 64, 2, 0.1, B.SYNC, stream=0)
    assert e.value.code == B.DP_ERR_INVALID_ARG
    with pytest.raises(B.DPError) as e:   # linear K % 64
        B.dp_linear(16, 16, None, None, 32, None, None, 10, 64, 48, 64, stream=0)
    assert e.value.code == B.DP_ERR_UNSUPPORTED
    with pytest.raises(B.DPError) as e:   # groupnorm: C % G
        B.dp_groupnorm_async(16, 32, 16, 16, 8, 8, 30, 32, 2, 1e-5, 1.0, 1, B.SYNC, B.BF16, None, None,
                             16, 16, 16, 1 << 20, 0)
    assert e.value.code == B.DP_ERR_UNSUPPORTED
    with pytest.raises(B.DPError) as e:   # groupnorm: workspace too small
        B.dp_groupnorm_async(16, 32, 16, 16, 8, 8, 64, 32, 2, 1e-5, 1.0, 1, B.SYNC, B.BF16, None, None,
                             16, 16, 16, 8, 0)
    assert e.value.code == B.DP_ERR_INVALID_ARG
    with pytest.raises(B.DPError) as e:   # groupnorm: displaced without stale statistics
        B.dp_groupnorm_async(16, 32, 16, 16, 8, 8, 64, 32, 2, 1e-5, 1.0, 1, B.DISPLACED, B.BF16, None,
                             None, 16, 16, 16, 1 << 20, 0)
    assert e.value.code == B.DP_ERR_INVALID_ARG
    with pytest.raises(B.DPError) as e:   # refresh: overlapping buffers
        B.dp_refresh_stale(1024, 1024 + 256, 256, 8, 2, -1, 0)
    assert e.value.code == B.DP_ERR_INVALID_ARG
    with pytest.raises(B.DPError) as e:   # refresh: bad band
        B.dp_refresh_stale(1024, 1 << 20, 256, 8, 2, 5, 0)
    assert e.value.code == B.DP_ERR_INVALID_ARG
    assert "refresh" in B.lib().dp_last_error().decode()


def test_groupnorm_workspace_size(B):
    assert B.dp_groupnorm_workspace_size(128, 128, 320, 32, 4) >= 256 + 4 * 32 * 2 * 8
    assert B.dp_groupnorm_workspace_size(128, 128, 320, 32, 0) == 0


def test_gn_stats_variants_on_the_host(B):
    """GroupNorm statistics variants of displaced steps: the default is the corrected statistics;
    the exact variant needs the whole image, so its GroupNorms take the grid-wide pass even in a
    displaced step; unknown variants are refused before any launch."""
    kinds = lambda d, m: [B.dp_block_launch_info(d, m, i)[0] for i in range(B.dp_block_launch_count(d))]
    d = B.dp_block_desc_init(B.RESBLOCK, 128, 128, 320, 320, 32, 4, 0, B.BF16, 1, 1e-5, 1.0)
    assert d.gn_stats == B.GN_STATS_CORRECTED
    B.dp_block_desc_set_gn_stats(d, B.GN_STATS_SYNC)
    assert kinds(d, B.DISPLACED) == ["gn_fused", "conv", "gn_fused", "conv"]
    for v in (B.GN_STATS_LOCAL, B.GN_STATS_STALE, B.GN_STATS_CORRECTED):
        B.dp_block_desc_set_gn_stats(d, v)
        assert kinds(d, B.DISPLACED) == ["gn_cluster", "conv", "gn_cluster", "conv"]
    # with fusion on, the conv normalises its own input under every variant
    d1 = B.dp_block_desc_init(B.RESBLOCK, 128, 128, 320, 320, 32, 4, 0, B.BF16, 1, 1e-5, 1.0)
    B.dp_block_desc_set_gn_fusion(d1, 1)
    for v in (B.GN_STATS_SYNC, B.GN_STATS_LOCAL, B.GN_STATS_STALE, B.GN_STATS_CORRECTED):
        B.dp_block_desc_set_gn_stats(d1, v)
        assert kinds(d1, B.DISPLACED) == ["gn_stats", "conv_gn", "gn_stats", "conv_gn"]
    with pytest.raises(B.DPError):
        B.dp_block_desc_set_gn_stats(d, 4)
    with pytest.raises(B.DPError):
        B.dp_block_desc_set_gn_stats(d, -1)
    d.gn_stats = 7                      # a descriptor edited by hand is checked too
    with pytest.raises(B.DPError, match="statistics variant"):
        B.dp_block_workspace_size(d)
    assert B.lib().dp_block_desc_set_gn_stats(None, 0) == -1


def test_refresh_halo_rejects_bad_arguments_on_the_host(B):
    with pytest.raises(B.DPError) as e:   # halo deeper than a band
        B.dp_refresh_halo(16, 4096, 64, 8, 4, 3, 0, stream=0)
    assert e.value.code == B.DP_ERR_INVALID_ARG
    with pytest.raises(B.DPError) as e:   # rows not a multiple of P
        B.dp_refresh_halo(16, 4096, 64, 9, 4, 1, 1, stream=0)
    assert e.value.code == B.DP_ERR_UNSUPPORTED
    with pytest.raises(B.DPError) as e:   # overlapping buffers
        B.dp_refresh_halo(16, 32, 64, 8, 4, 1, 1, stream=0)
    assert e.value.code == B.DP_ERR_INVALID_ARG
    with pytest.raises(B.DPError) as e:   # row bytes not a multiple of 16
        B.dp_refresh_halo(16, 4096, 40, 8, 4, 1, 1, stream=0)
    assert e.value.code == B.DP_ERR_UNSUPPORTED
    assert B.dp_refresh_halo(16, 4096, 64, 8, 1, 1, 1, stream=0) == B.DP_OK   # one band: nothing to do


def test_plain_c_caller(B, tmp_path):
    """The header is plain C99, and a C program links against libdp and uses the host-side
    calls (descriptor set-up, validation, the step-mode helper) with no Python in between."""
    import shutil
    import subprocess
    if not shutil.which("gcc"):
        pytest.skip("no C compiler")
    src = tmp_path / "caller.c"
    src.write_text(r'''
#include <stdio.h>
#include <string.h>
#include "dp.h"
int main(void) {
  dp_block_desc d;
  if (dp_block_desc_init(&d, DP_BLOCK_RESBLOCK, 128, 128, 320, 320, 32, 4, 0, DP_BF16, 1,
                         1e-5f, 1.0f) != DP_OK) return 1;
  if (d.gn_stats != DP_GN_STATS_CORRECTED) return 2;
  if (dp_block_desc_set_gn_stats(&d, DP_GN_STATS_SYNC) != DP_OK) return 3;
  if (dp_block_desc_set_gn_stats(&d, 9) != DP_ERR_INVALID_ARG) return 4;
  if (strstr(dp_last_error(), "variant") == NULL) return 5;
  if (dp_block_workspace_size(&d) == 0) return 6;
  if (dp_mode_for_step(0, 0) != DP_MODE_NAIVE || dp_mode_for_step(3, 4) != DP_MODE_SYNC ||
      dp_mode_for_step(4, 4) != DP_MODE_DISPLACED) return 7;
  if (dp_block_desc_init(&d, DP_BLOCK_RESBLOCK, 130, 128, 320, 320, 32, 4, 0, DP_BF16, 1,
                         1e-5f, 1.0f) != DP_ERR_UNSUPPORTED) return 8;
  printf("%s\n", dp_version());
  return 0;
}
''')
    exe = tmp_path / "caller"
    libdir = os.path.dirname(B.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                    "-I" + os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                    "-L" + libdir, "-l:libdp.so", "-Wl,-rpath," + libdir], check=True)
    run = subprocess.run([str(exe)], capture_output=True, text=True)
    assert run.returncode == 0, (run.returncode, run.stdout, run.stderr)
    assert run.stdout.strip()


def test_cross_attention_rejects_bad_arguments_on_the_host(B):
    with pytest.raises(B.DPError) as e:   # query count not a multiple of 256
        B.dp_attn_cross(16, 32, 48, 64, 300, 77, 2, 64, 0.125, stream=0)
    assert e.value.code == B.DP_ERR_UNSUPPORTED
    with pytest.raises(B.DPError) as e:   # head_dim 128
        B.dp_attn_cross(16, 32, 48, 64, 256, 77, 2, 128, 0.125, stream=0)
    assert e.value.code == B.DP_ERR_UNSUPPORTED
    with pytest.raises(B.DPError) as e:   # output aliases the queries
        B.dp_attn_cross(16, 32, 48, 16, 256, 77, 2, 64, 0.125, stream=0)
    assert e.value.code == B.DP_ERR_INVALID_ARG
    with pytest.raises(B.DPError) as e:
        B.dp_attn_cross(None, 32, 48, 64, 256, 77, 2, 64, 0.125, stream=0)
    assert e.value.code == B.DP_ERR_INVALID_ARG


def test_token_operators_reject_bad_arguments_on_the_host(B):
    with pytest.raises(B.DPError) as e:   # C not a multiple of 8
        B.dp_layernorm(16, 4096, 32, 48, 4, 12, 1e-5, stream=0)
    assert e.value.code == B.DP_ERR_UNSUPPORTED
    with pytest.raises(B.DPError) as e:   # C too large for one warp's registers
        B.dp_layernorm(16, 1 << 20, 32, 48, 4, 4096, 1e-5, stream=0)
    assert e.value.code == B.DP_ERR_UNSUPPORTED
    with pytest.raises(B.DPError) as e:   # y aliases x
        B.dp_layernorm(16, 16, 32, 48, 4, 64, 1e-5, stream=0)
    assert e.value.code == B.DP_ERR_INVALID_ARG
    with pytest.raises(B.DPError) as e:   # y overlaps x in part (4 tokens x 64 x 2 bytes = 512)
        B.dp_layernorm(4096, 4096 + 256, 32, 48, 4, 64, 1e-5, stream=0)
    assert e.value.code == B.DP_ERR_INVALID_ARG
    with pytest.raises(B.DPError) as e:   # F not a multiple of 8
        B.dp_geglu(16, 4096, 4, 12, stream=0)
    assert e.value.code == B.DP_ERR_UNSUPPORTED
    with pytest.raises(B.DPError) as e:   # y overlaps h
        B.dp_geglu(16, 32, 4, 64, stream=0)
    assert e.value.code == B.DP_ERR_INVALID_ARG


def test_transformer_block_plan_on_the_host(B):
    """An SDXL-shaped transformer block: it needs its context sizes, takes 25 pointers, and its
    launches follow the documented order; the launches' flops add up to the block's."""
    d = B.dp_block_desc_init(B.TRANSFORMER, 64, 64, 640, 640, 32, 4, 10, B.BF16, 0, 1e-5, 1.0)
    with pytest.raises(B.DPError, match="set_context"):
        B.dp_block_workspace_size(d)
    with pytest.raises(B.DPError):
        B.dp_block_desc_set_context(d, 77, 100, 2560)     # context width not a multiple of 64
    B.dp_block_desc_set_context(d, 77, 2048, 2560)
    assert B.dp_block_weight_count(d) == 25
    kinds = [B.dp_block_launch_info(d, B.DISPLACED, i)[0] for i in range(B.dp_block_launch_count(d))]
    # ff1 carries the gated GELU in its epilogue (2F = 5120 is a whole number of pair tiles)
    assert [k for k in kinds if k != "splitk_finish"] == [
        "gn_cluster", "linear", "layernorm", "linear", "attn", "linear", "layernorm", "linear", "linear",
        "attn", "linear", "layernorm", "linear", "linear", "linear"]
    fl = sum(B.dp_block_launch_info(d, B.DISPLACED, i)[1] for i in range(B.dp_block_launch_count(d)))
    assert abs(fl - B.dp_block_flops(d)) < 1e-6 * fl
    assert B.dp_block_workspace_size(d) > 64 * 64 * 2560 * 2 * 2
    # tokens wider than one LayerNorm warp holds are rejected before any step runs
    dw = B.dp_block_desc_init(B.TRANSFORMER, 32, 32, 2112, 2112, 32, 4, 33, B.BF16, 0, 1e-5, 1.0)
    with pytest.raises(B.DPError, match="LayerNorm width") as e:
        B.dp_block_desc_set_context(dw, 77, 2048, 4 * 2112)
        B.dp_block_workspace_size(dw)
    assert e.value.code in (B.DP_ERR_UNSUPPORTED, B.DP_ERR_INVALID_ARG)
    dr = B.dp_block_desc_init(B.RESBLOCK, 64, 64, 320, 320, 32, 4, 0, B.BF16, 1, 1e-5, 1.0)
    with pytest.raises(B.DPError, match="only for TRANSFORMER"):
        B.dp_block_desc_set_context(dr, 77, 2048, 1280)


def test_time_embedding_rejects_bad_arguments_on_the_host(B):
    A = 1 << 20                                   # fake, never dereferenced: checks run first
    for args in [(0, A, 0, 0, 2 * A, 8, 4),      # null temb
                 (A, A, 0, 0, 0, 8, 4),           # null bias
                 (A, 2 * A, 0, 0, 3 * A, 0, 4),   # Ct = 0
                 (A, 2 * A, 0, 0, 3 * A, 8193, 4),
                 (A, 2 * A, 0, 0, 3 * A, 8, 0),   # Cout = 0
                 (A, 2 * A, 0, 0, A + 16, 8, 4),  # bias overlaps temb
                 (A, 2 * A, 0, 3 * A, 3 * A + 8, 8, 4)]:   # bias overlaps conv_b
        with pytest.raises(B.DPError) as e:
            B.dp_time_embedding_bias(*args, stream=0)
        assert e.value.code == B.DP_ERR_INVALID_ARG, args


def test_resblock_time_embedding_plan_on_the_host(B):
    """A RESBLOCK with a time embedding takes temb_w, temb_b and temb after its other
    weights, launches the bias kernel first, and counts its flops."""
    d = B.dp_block_desc_init(B.RESBLOCK, 64, 64, 320, 640, 32, 4, 0, B.BF16, 1, 1e-5, 1.0)
    n0, f0, w0 = B.dp_block_launch_count(d), B.dp_block_flops(d), B.dp_block_workspace_size(d)
    assert B.dp_block_weight_count(d) == 10
    B.dp_block_desc_set_time_embedding(d, 1280)
    assert B.dp_block_weight_count(d) == 13
    assert B.dp_block_launch_count(d) == n0 + 1
    assert B.dp_block_launch_info(d, B.DISPLACED, 0)[:2] == ("temb", 2.0 * 640 * 1280)
    assert B.dp_block_flops(d) == f0 + 2.0 * 640 * 1280
    fl = sum(B.dp_block_launch_info(d, B.DISPLACED, i)[1] for i in range(B.dp_block_launch_count(d)))
    assert abs(fl - B.dp_block_flops(d)) < 1e-6 * fl
    assert B.dp_block_workspace_size(d) >= w0 + 640 * 4
    B.dp_block_desc_set_time_embedding(d, 0)       # off again: the plain ResBlock
    assert B.dp_block_weight_count(d) == 10 and B.dp_block_launch_count(d) == n0
    for bad in (-1, 8193):
        with pytest.raises(B.DPError):
            B.dp_block_desc_set_time_embedding(d, bad)
    da = B.dp_block_desc_init(B.ATTN, 64, 64, 640, 640, 32, 4, 10, B.BF16, 0, 1e-5, 1.0)
    with pytest.raises(B.DPError, match="only for RESBLOCK"):
        B.dp_block_desc_set_time_embedding(da, 1280)
    da.temb_dim = 1280                              # set behind the setter's back
    with pytest.raises(B.DPError, match="only for RESBLOCK"):
        B.dp_block_workspace_size(da)


def test_ddim_step_rejects_bad_arguments_on_the_host(B):
    A = 1 << 20                                   # fake, never dereferenced: checks run first
    bad = [((0, 2 * A, 3 * A, 64, 0.5, 0.6, B.BF16), B.DP_ERR_INVALID_ARG),    # null x
           ((A, 2 * A, 3 * A, 64, 0.5, 0.6, 7), B.DP_ERR_INVALID_ARG),         # dtype
           ((A, 2 * A, 3 * A, 64, 0.0, 0.6, B.BF16), B.DP_ERR_INVALID_ARG),    # abar_t = 0
           ((A, 2 * A, 3 * A, 64, 0.5, 1.5, B.BF16), B.DP_ERR_INVALID_ARG),    # abar_prev > 1
           ((A, 2 * A, 3 * A, 64, float("nan"), 0.6, B.BF16), B.DP_ERR_INVALID_ARG),
           ((A, 2 * A, 3 * A + 8, 64, 0.5, 0.6, B.BF16), B.DP_ERR_UNSUPPORTED),  # misaligned
           ((A, 2 * A, 2 * A + 64, 64, 0.5, 0.6, B.BF16), B.DP_ERR_INVALID_ARG),  # overlaps eps
           ((A, 2 * A, A + 64, 64, 0.5, 0.6, B.FP32), B.DP_ERR_INVALID_ARG),      # partly overlaps x
           ((A, 2 * A, 3 * A, 1 << 62, 0.5, 0.6, B.FP32), B.DP_ERR_INVALID_ARG)]  # byte count overflows
    for args, code in bad:
        with pytest.raises(B.DPError) as e:
            B.dp_ddim_step(*args, stream=0)
        assert e.value.code == code, args
    B.dp_ddim_step(A, 2 * A, A, 0, 0.5, 0.6, B.BF16, stream=0)   # in place, n = 0: nothing to do


def test_binding_structs_match_the_header(B, tmp_path):
    """Every field of dp_block_desc and dp_block_state sits at the same offset, and each struct
    has the same size, in the C header (compiled by gcc) and in the ctypes binding."""
    import shutil
    import subprocess
    if not shutil.which("gcc"):
        pytest.skip("no C compiler")
    structs = {"dp_block_desc": B.BlockDesc, "dp_block_state": B.BlockState}
    lines = []
    for cname, py in structs.items():
        lines.append(f'  printf("{cname} sizeof %zu\\n", sizeof({cname}));')
        for field, _ in py._fields_:
            lines.append(f'  printf("{cname} {field} %zu\\n", offsetof({cname}, {field}));')
    src = tmp_path / "layout.c"
    src.write_text("#include <stddef.h>\n#include <stdio.h>\n#include \"dp.h\"\nint main(void) {\n" +
                   "\n".join(lines) + "\n  return 0;\n}\n")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I" + os.path.join(ROOT, "include"),
                    str(src), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split("\n")
    for row in filter(None, out):
        cname, field, value = row.split()
        py = structs[cname]
        want = ctypes.sizeof(py) if field == "sizeof" else getattr(py, field).offset
        assert int(value) == want, (cname, field, int(value), want)


def test_transformer_depth_on_the_host(B):
    """A transformer block of depth 3: 7 + 18 * 3 pointers, the layer launches three times
    between proj_in and proj_out, flops three layers' worth; a depth is for TRANSFORMER
    blocks only and lies in [1, 16]."""
    d = B.dp_block_desc_init(B.TRANSFORMER, 32, 32, 320, 320, 32, 4, 5, B.BF16, 0, 1e-5, 1.0)
    B.dp_block_desc_set_context(d, 77, 128, 1280)
    one = B.dp_block_flops(d)
    ws1 = B.dp_block_workspace_size(d)
    for bad in (0, 17, -1):
        with pytest.raises(B.DPError):
            B.dp_block_desc_set_depth(d, bad)
    B.dp_block_desc_set_depth(d, 3)
    assert B.dp_block_weight_count(d) == 7 + 18 * 3
    kinds = [B.dp_block_launch_info(d, B.DISPLACED, i)[0] for i in range(B.dp_block_launch_count(d))]
    layer = ["layernorm", "linear", "attn", "linear", "layernorm", "linear", "linear", "attn", "linear",
             "layernorm", "linear", "linear"]
    assert [k for k in kinds if k != "splitk_finish"] == ["gn_cluster", "linear"] + 3 * layer + ["linear"]
    T, C = 32 * 32, 320
    proj = 2 * 2.0 * T * C * C
    assert abs(B.dp_block_flops(d) - (proj + 3 * (one - proj))) < 1e-9 * one
    # two more layers' stale key/value ping-pong pairs
    assert B.dp_block_workspace_size(d) - ws1 >= 2 * 4 * T * C * 2
    r = B.dp_block_desc_init(B.RESBLOCK, 32, 32, 320, 320, 32, 4, 0, B.BF16, 1, 1e-5, 1.0)
    with pytest.raises(B.DPError, match="TRANSFORMER"):
        B.dp_block_desc_set_depth(r, 2)
    r.depth = 2                                     # written past the setter: rejected at use
    with pytest.raises(B.DPError, match="depth"):
        B.dp_block_workspace_size(r)


def test_feed_forward_fusion_rule_on_the_host(B):
    """The gated GELU rides in ff1's epilogue when 2F is a whole number of 160-column pair
    tiles (SDXL: F = 4C, C a multiple of 320 here); otherwise ff1 and a GEGLU pass run; the
    fused call rejects other shapes before any launch."""
    def kinds(C, F):
        d = B.dp_block_desc_init(B.TRANSFORMER, 32, 32, C, C, 32, 2, C // 64, B.BF16, 0, 1e-5, 1.0)
        B.dp_block_desc_set_context(d, 77, 128, F)
        return [B.dp_block_launch_info(d, B.DISPLACED, i)[0] for i in range(B.dp_block_launch_count(d))]
    assert "geglu" not in kinds(640, 2560) and "geglu" not in kinds(320, 1280)
    assert kinds(128, 512).count("geglu") == 1 and kinds(256, 1024).count("geglu") == 1
    A = 1 << 20
    for args, code in [((0, 2 * A, 0, 3 * A, 128, 1280, 320), B.DP_ERR_INVALID_ARG),   # null x
                       ((A, 2 * A, 0, 3 * A, 128, 512, 320), B.DP_ERR_UNSUPPORTED),   # 2F % 160
                       ((A, 2 * A, 0, 3 * A, 128, 1280, 96), B.DP_ERR_UNSUPPORTED),   # K % 64
                       ((A, 2 * A, 0, A + 64, 128, 1280, 320), B.DP_ERR_INVALID_ARG)]:  # y overlaps x
        with pytest.raises(B.DPError) as e:
            B.dp_linear_geglu(*args, stream=0)
        assert e.value.code == code, args


def test_block_graph_rejects_bad_arguments_on_the_host(B):
    """Graph capture checks its arguments before any CUDA call: a state before its first
    step, the default stream, a null handle pointer; launch and destroy of a null handle."""
    import ctypes
    d = B.dp_block_desc_init(B.RESBLOCK, 32, 32, 320, 320, 32, 4, 0, B.BF16, 1, 1e-5, 1.0)
    A = 1 << 20
    st = B.BlockState(A, B.dp_block_workspace_size(d), 0, 0)
    w = (ctypes.c_void_p * 8)(*([A] * 8))
    h = ctypes.c_void_p(0)
    L = B.lib()
    assert L.dp_block_graph_create(ctypes.byref(d), ctypes.byref(st), A, 2 * A, w, 8, B.DISPLACED, A,
                                   ctypes.byref(h)) == B.DP_ERR_STATE
    st.steps_done = 1
    assert L.dp_block_graph_create(ctypes.byref(d), ctypes.byref(st), A, 2 * A, w, 8, B.DISPLACED, None,
                                   ctypes.byref(h)) == B.DP_ERR_INVALID_ARG       # default stream
    assert L.dp_block_graph_create(ctypes.byref(d), ctypes.byref(st), A, 2 * A, w, 8, B.DISPLACED, A,
                                   None) == B.DP_ERR_INVALID_ARG                  # no handle pointer
    assert L.dp_block_graph_create(ctypes.byref(d), ctypes.byref(st), A, 2 * A, w, 7, B.DISPLACED, A,
                                   ctypes.byref(h)) == B.DP_ERR_INVALID_ARG       # too few weights
    assert L.dp_block_graph_launch(None, ctypes.byref(st), A) == B.DP_ERR_INVALID_ARG
    assert L.dp_block_graph_destroy(None) == B.DP_OK


def test_fixed_context_on_the_host(B):
    """A fixed context drops each layer's context k/v projection from the (later) steps' plan
    and flops, and is only for TRANSFORMER and UNET_SDXL blocks."""
    d = B.dp_block_desc_init(B.TRANSFORMER, 32, 32, 320, 320, 32, 4, 5, B.BF16, 0, 1e-5, 1.0)
    B.dp_block_desc_set_context(d, 77, 128, 1280)
    B.dp_block_desc_set_depth(d, 3)
    n, fl = B.dp_block_launch_count(d), B.dp_block_flops(d)
    B.dp_block_desc_set_context_fixed(d, True)
    assert B.dp_block_launch_count(d) == n - 3
    assert abs(fl - B.dp_block_flops(d) - 3 * 2.0 * 77 * 2 * 320 * 128) < 1e-6 * fl
    with pytest.raises(B.DPError):
        B.dp_block_desc_set_context_fixed(d, 2)
    r = B.dp_block_desc_init(B.RESBLOCK, 32, 32, 320, 320, 32, 4, 0, B.BF16, 1, 1e-5, 1.0)
    with pytest.raises(B.DPError, match="TRANSFORMER"):
        B.dp_block_desc_set_context_fixed(r, True)


def test_transformer_depth_workload_marshals(B):
    """Seeded weights of a depth-2 transformer workload marshal into 7 + 18 * 2 pointers (the
    context last), and its first layer's weights are those of the depth-1 workload."""
    import dataclasses

    import torch

    from displaced_patch_parallelism_b200 import synth
    from displaced_patch_parallelism_b200.weights import block_weights
    wl1 = dataclasses.replace(synth.WORKLOADS["transformer_640x64x64"], C=64, ctx_dim=64, ff_inner=256, heads=1)
    wl2 = dataclasses.replace(wl1, depth=2)
    w1 = block_weights("transformer", synth.make_weights(wl1, True), torch.bfloat16, "cpu")
    w2 = block_weights("transformer", synth.make_weights(wl2, True), torch.bfloat16, "cpu", depth=2)
    assert len(w2) + 1 == 7 + 18 * 2
    for a, b in zip(w1[:22], w2[:22]):
        assert torch.equal(a, b)
    assert torch.equal(w1[22], w2[40]) and torch.equal(w1[23], w2[41])   # proj_out
    assert not torch.equal(w2[6], w2[24])                                 # the layers' wqkv differ


def test_unet_sdxl_descriptor_on_the_host(B):
    """An SDXL-shaped U-Net step: it needs its context and time embedding; at SDXL's own sizes
    (latent 4x128x128, base 320, depths 0 / 2 / 10) it takes 1534 pointers and 6.76 TFLOP;
    its launches follow the stage order and add up to its flops; the seeded small workload's
    marshalled weights fill its list."""
    import torch

    from displaced_patch_parallelism_b200 import synth
    from displaced_patch_parallelism_b200.weights import unet_sdxl_weights
    d = B.dp_block_desc_init(B.UNET_SDXL, 128, 128, 4, 0, 32, 8, 0, B.BF16, 1, 1e-5, 1.0)
    assert d.Cout == 4 and d.unet_base == 320 and list(d.unet_depth) == [0, 2, 10]
    with pytest.raises(B.DPError, match="set_context"):
        B.dp_block_workspace_size(d)
    B.dp_block_desc_set_context(d, 77, 2048, 0)
    with pytest.raises(B.DPError, match="set_time_embedding"):
        B.dp_block_workspace_size(d)
    B.dp_block_desc_set_time_embedding(d, 1280)
    assert B.dp_block_weight_count(d) == 1534
    assert abs(B.dp_block_flops(d) - 6.7612e12) < 1e-3 * 6.76e12
    kinds = [B.dp_block_launch_info(d, B.DISPLACED, i)[0] for i in range(B.dp_block_launch_count(d))]
    assert kinds[:2] == ["copy", "conv_small"] and kinds[-1] == "conv_narrow"
    assert kinds.count("concat") == 9 and kinds.count("upsample") == 2
    fl = sum(B.dp_block_launch_info(d, B.DISPLACED, i)[1] for i in range(len(kinds)))
    assert abs(fl - B.dp_block_flops(d)) < 1e-9 * fl
    for bad in [(320, -1, 2, 10), (96, 0, 2, 10), (320, 0, 17, 10), (1024, 0, 2, 10)]:
        with pytest.raises(B.DPError):
            B.dp_block_desc_set_unet(d, *bad)
    with pytest.raises(B.DPError):
        B.dp_block_desc_set_context(d, 77, 2048, 5120)   # the inner width is 4C per level
    r = B.dp_block_desc_init(B.RESBLOCK, 32, 32, 320, 320, 32, 4, 0, B.BF16, 1, 1e-5, 1.0)
    with pytest.raises(B.DPError, match="UNET_SDXL"):
        B.dp_block_desc_set_unet(r, 320, 0, 2, 10)
    # a small U-Net: the marshalled seeded weights fill the list, the context and temb follow
    wl = synth.Workload(name="u", kind="unet_sdxl", C=4, H=64, W=64, P=2, base=64, depths=(0, 1, 1),
                        ctx_len=77, ctx_dim=128, temb_dim=128)
    s = B.dp_block_desc_init(B.UNET_SDXL, 64, 64, 4, 4, 32, 2, 0, B.BF16, 1, 1e-5, 1.0)
    B.dp_block_desc_set_unet(s, 64, 0, 1, 1)
    B.dp_block_desc_set_context(s, 77, 128, 0)
    B.dp_block_desc_set_time_embedding(s, 128)
    w = unet_sdxl_weights(synth.make_weights(wl), synth.sdxl_unet_stages(64, (0, 1, 1)), (0, 1, 1),
                          torch.bfloat16, "cpu")
    assert len(w) + 2 == B.dp_block_weight_count(s)
    # too few tokens per band at the deepest level for its transformer
    with pytest.raises(B.DPError):
        B.dp_block_desc_set_unet(d, 320, 0, 2, 10)
        t = B.dp_block_desc_init(B.UNET_SDXL, 32, 32, 4, 4, 32, 2, 0, B.BF16, 1, 1e-5, 1.0)
        B.dp_block_desc_set_context(t, 77, 2048, 0)
        B.dp_block_desc_set_time_embedding(t, 1280)


def test_concat_upsample_reject_bad_arguments_on_the_host(B):
    """Argument checks run before any launch: null pointers, channel counts that are not whole
    16-byte vectors, overlapping output, misalignment, bad sizes."""
    A = 1 << 20                                   # fake, never dereferenced: checks run first
    for args, code in [((0, 2 * A, 3 * A, 4, 64, 64), B.DP_ERR_INVALID_ARG),            # null a
                       ((A, 2 * A, 3 * A, 4, 60, 68), B.DP_ERR_UNSUPPORTED),           # channels
                       ((3 * A, 2 * A, 3 * A, 4, 64, 64), B.DP_ERR_INVALID_ARG),       # out overlaps a
                       ((A, 2 * A, 3 * A + 8, 4, 64, 64), B.DP_ERR_UNSUPPORTED),       # misaligned
                       ((A, 2 * A, 3 * A, 4, 0, 64), B.DP_ERR_INVALID_ARG)]:           # empty channels
        with pytest.raises(B.DPError) as e:
            B.dp_concat_channels(*args, stream=0)
        assert e.value.code == code, args
    for args, code in [((0, 2 * A, 2, 2, 64), B.DP_ERR_INVALID_ARG),                   # null x
                       ((A, 2 * A, 2, 2, 12), B.DP_ERR_UNSUPPORTED),                   # C not whole vectors
                       ((A, A + 64, 1, 1, 64), B.DP_ERR_INVALID_ARG),                  # out overlaps x
                       ((A, 2 * A, 0, 2, 64), B.DP_ERR_INVALID_ARG)]:                  # empty image
        with pytest.raises(B.DPError) as e:
            B.dp_upsample_nearest2x(*args, stream=0)
        assert e.value.code == code, args


def test_transformer_workload_marshals_to_the_block(B):
    """The benchmark's SDXL transformer workload: its seeded weights marshal into the 24
    pointers the block documents (the context is the 25th), with the documented shapes."""
    import torch

    from displaced_patch_parallelism_b200 import synth
    from displaced_patch_parallelism_b200.weights import block_weights
    wl = synth.WORKLOADS["transformer_640x64x64"]
    C, F, Cc, Tk = wl.C, wl.ff_inner, wl.ctx_dim, wl.ctx_len
    d = B.dp_block_desc_init(B.TRANSFORMER, wl.H, wl.W, C, C, wl.G, wl.P, wl.heads, B.BF16, 0,
                             wl.eps, 1.0)
    B.dp_block_desc_set_context(d, Tk, Cc, F)
    w = block_weights("transformer", synth.make_weights(wl), torch.bfloat16, "cpu")
    assert len(w) + 1 == B.dp_block_weight_count(d)
    shapes = [(C,), (C,), (C, C), (C,), (C,), (C,), (3 * C, C), (3 * C,), (C, C), (C,), (C,), (C,),
              (C, C), (2 * C, Cc), (C, C), (C,), (C,), (C,), (2 * F, C), (2 * F,), (C, F), (C,),
              (C, C), (C,)]
    assert [tuple(t.shape) for t in w] == shapes
    assert tuple(synth.context(wl).shape) == (Tk, Cc)


def test_selftest_and_block_status_reject_bad_arguments_on_the_host(B):
    for kind, limit in [(2, 100), (-1, 100), (0, 0), (1, 2000000)]:
        with pytest.raises(B.DPError) as e:
            B.dp_selftest_bounded_wait(kind, limit, stream=0)
        assert e.value.code == B.DP_ERR_INVALID_ARG
    d = B.dp_block_desc_init(B.GN_CONV, 16, 16, 64, 64, 32, 2, 0, B.BF16, 1, 1e-5, 1.0)
    with pytest.raises(B.DPError) as e:   # a state never initialised has no workspace
        B.dp_block_status(d, B.BlockState(), stream=0)
    assert e.value.code == B.DP_ERR_INVALID_ARG


def test_groupnorm_fusion_plan(B):
    """dp_block_desc_set_gn_fusion(d, 1): every GroupNorm -> conv pair the fused conv takes is a
    statistics pass plus a conv that normalises its own input; others stay as they are; the
    flag reaches the mini U-Net's ResBlocks; it is checked."""
    kinds = lambda d, m: [B.dp_block_launch_info(d, m, i)[0] for i in range(B.dp_block_launch_count(d))]
    d = B.dp_block_desc_init(B.RESBLOCK, 128, 128, 320, 320, 32, 4, 0, B.BF16, 1, 1e-5, 1.0)
    B.dp_block_desc_set_gn_fusion(d, 1)
    assert kinds(d, B.DISPLACED) == ["gn_stats", "conv_gn", "gn_stats", "conv_gn"]
    assert kinds(d, B.SYNC) == ["gn_stats", "conv_gn", "gn_stats", "conv_gn"]
    fl = sum(B.dp_block_launch_info(d, B.DISPLACED, i)[1] for i in range(4))
    assert abs(fl - B.dp_block_flops(d)) < 1
    d4 = B.dp_block_desc_init(B.GN_CONV, 480, 480, 320, 320, 32, 8, 0, B.BF16, 1, 1e-5, 1.0)
    B.dp_block_desc_set_gn_fusion(d4, 1)
    assert kinds(d4, B.DISPLACED) == ["gn_stats", "conv_gn"]
    d2 = B.dp_block_desc_init(B.RESBLOCK, 64, 64, 320, 640, 32, 4, 0, B.BF16, 1, 1e-5, 1.0)
    B.dp_block_desc_set_gn_fusion(d2, 1)                  # 64 columns: not eligible
    assert kinds(d2, B.DISPLACED) == ["gn_cluster", "conv", "gn_cluster", "linear", "conv"]
    du = B.dp_block_desc_init(B.UNET_MINI, 128, 128, 4, 0, 32, 4, 0, B.BF16, 1, 1e-5, 1.0)
    B.dp_block_desc_set_gn_fusion(du, 1)
    assert kinds(du, B.DISPLACED).count("conv_gn") == 2   # the 128x128 ResBlock's two convs
    with pytest.raises(B.DPError):
        B.dp_block_desc_set_gn_fusion(d, 2)
    d.gn_fuse = 5                                         # edited by hand: checked too
    with pytest.raises(B.DPError, match="fusion"):
        B.dp_block_workspace_size(d)


def test_groupnorm_conv_rejects_bad_arguments_on_the_host(B):
    A = 1 << 20                                   # fake, never dereferenced: checks run first
    base = dict(x=A, a_stale=2 * A, a_next=0, used=3 * A, gamma=4 * A, beta=5 * A, G=32, eps=1e-5,
                silu=1, weight=6 * A, bias=0, residual=0, out=7 * A, H=16, W=128, Cin=64, Cout=160,
                P=2, mode=B.DISPLACED)

    def call(**kw):
        a = dict(base, **kw)
        B.dp_conv3x3_halo_gn(a["x"], a["a_stale"], a["a_next"], a["used"], a["gamma"], a["beta"],
                             a["G"], a["eps"], a["silu"], a["weight"], a["bias"], a["residual"],
                             a["out"], a["H"], a["W"], a["Cin"], a["Cout"], a["P"], a["mode"], stream=0)

    for kw, code in [(dict(W=64), B.DP_ERR_UNSUPPORTED),          # tiles need 128 columns
                     (dict(Cout=96), B.DP_ERR_UNSUPPORTED),       # Cout % 160
                     (dict(used=0), B.DP_ERR_INVALID_ARG),
                     (dict(eps=0.0), B.DP_ERR_INVALID_ARG),
                     (dict(a_stale=0), B.DP_ERR_INVALID_ARG),     # displaced needs a_stale
                     (dict(a_next=A + 64), B.DP_ERR_INVALID_ARG),  # a_next overlaps x
                     (dict(H=15), B.DP_ERR_UNSUPPORTED)]:         # H % P
        with pytest.raises(B.DPError) as e:
            call(**kw)
        assert e.value.code == code, kw
    with pytest.raises(B.DPError) as e:                           # stats: displaced needs stale moments
        B.dp_groupnorm_stats(A, 16, 128, 64, 32, 2, 1.0, B.DISPLACED, B.BF16, 0, 0, 2 * A, 3 * A, 4 * A,
                             1 << 16, stream=0)
    assert e.value.code == B.DP_ERR_INVALID_ARG


def test_dpm_solver_rejects_bad_arguments_on_the_host(B):
    A = 1 << 20                                   # fake, never dereferenced: checks run first
    good = (A, 2 * A, 3 * A, 4 * A, 64, 0.1, 0.2, 0.3, B.FP32)
    for args, code in [((0,) + good[1:], B.DP_ERR_INVALID_ARG),                       # null x
                       (good[:5] + (0.1, 0.3, 0.2, B.FP32), B.DP_ERR_INVALID_ARG),   # abar_t < abar_s
                       (good[:5] + (0.25, 0.2, 0.3, B.FP32), B.DP_ERR_INVALID_ARG),  # abar_prev > abar_s
                       (good[:8] + (7,), B.DP_ERR_INVALID_ARG),                       # dtype
                       ((A, 2 * A, A + 64, 4 * A) + good[4:], B.DP_ERR_INVALID_ARG),  # x0_buf overlaps x
                       ((A + 8,) + good[1:], B.DP_ERR_UNSUPPORTED)]:                  # misaligned
        with pytest.raises(B.DPError) as e:
            B.dp_dpm_solver_step(*args, stream=0)
        assert e.value.code == code, args
