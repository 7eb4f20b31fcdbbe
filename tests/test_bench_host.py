"""bench.py's host-side bookkeeping: the flop count both arms use, and the rule
that the oracle arm never loads the CUDA library."""
import os
import subprocess
import sys

import pytest

import bench
from displaced_patch_parallelism_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("name", sorted(synth.WORKLOADS))
def test_python_flop_count_matches_the_library(name):
    """wl_flops (shapes only, no library) equals dp_block_flops for every workload, so the
    oracle arm's TFLOP/s and ours count the same work."""
    from displaced_patch_parallelism_b200 import binding as B
    B.lib()
    wl = synth.WORKLOADS[name]
    assert bench.wl_flops(wl) == pytest.approx(B.dp_block_flops(bench.block_desc(B, wl)), rel=1e-12)


def test_flop_count_of_a_row_crop():
    wl = synth.WORKLOADS["gn_conv_320x480x480"]
    assert bench.wl_flops(wl, 16) == pytest.approx(2.0 * 16 * 480 * 320 * 9 * 320)


def test_headline_workload_is_the_largest_single_gpu_one():
    src = open(os.path.join(ROOT, "bench.py")).read()
    assert 'default="gn_conv_320x480x480"' in src
    big = max((synth.WORKLOADS[n] for n in synth.CONFIG_WORKLOADS), key=lambda w: bench.wl_flops(w))
    assert big.name == "gn_conv_320x480x480"


def test_l2_policy():
    assert bench.l2_policy(synth.WORKLOADS["gn_conv_320x480x480"])[0] is False
    assert bench.l2_policy(synth.WORKLOADS["resblock_320x128x128"])[0] is True


def test_reference_arm_code_path_loads_no_library():
    """The oracle arm's helpers (flop count, row crop, one oracle step) run in a fresh
    process that never maps libdp.so."""
    code = (
        "import dataclasses, bench\n"
        "from displaced_patch_parallelism_b200 import synth\n"
        "wl = synth.WORKLOADS['gn_conv_320x480x480']\n"
        "bench.wl_flops(wl, 16)\n"
        "bench.oracle_step_time(dataclasses.replace(synth.WORKLOADS['tiny_fp32_gn_conv'], H=4))\n"
        "maps = open('/proc/self/maps').read()\n"
        "assert 'libdp.so' not in maps, 'libdp.so mapped'\n"
        "print('clean')\n")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert "clean" in r.stdout
