"""Error of each GroupNorm statistics variant against the exact synchronous
block, on synthetic inputs, computed with the oracle alone.

"DistriFusion" (atlas.scime.ai summary, the GroupNorm ablation rows) compares
the corrected asynchronous statistics with statistics of the device's own
patch only, stale statistics only, and a synchronous exact pass.  This script
runs a ResBlock chain (one synchronous warm-up step, then displaced steps, the
input drifting by N(0, drift^2) per step) for each variant, and reports the
relative L2 distance of every displaced step's output from the same step
computed synchronously (exact statistics and fresh context everywhere).  The
naive chain (every band alone) is the no-context baseline.

Test infrastructure like the rest of ``oracle/``: fp64 numpy, slow.

    python -m oracle.gn_stats_ablation [--size 64] [--steps 4] [--drift 0.05]
"""
import argparse
import dataclasses
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
from displaced_patch_parallelism_b200 import synth  # noqa: E402  (seeded inputs only)
from oracle import dp_oracle as O  # noqa: E402

VARIANTS = [("corrected", O.GN_STATS_CORRECTED), ("band-local", O.GN_STATS_LOCAL),
            ("stale-only", O.GN_STATS_STALE), ("exact stats", O.GN_STATS_SYNC)]


def chain(wl, wts, modes, gn_stats=O.GN_STATS_CORRECTED):
    xs = synth.InputStream(wl)
    st, outs = {}, []
    for k, m in enumerate(modes):
        outs.append(O.block_step(wl.kind, st, xs.x(k)[0].double().numpy(), wts, wl.P, wl.G, wl.eps,
                                 1.0, m, wl.dtype, heads=wl.heads, silu=wl.silu, gn_stats=gn_stats,
                                 final_storage="none"))
    return outs


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--size", type=int, default=64, help="latent rows and columns")
    ap.add_argument("--steps", type=int, default=4, help="displaced steps after one warm-up step")
    ap.add_argument("--drift", type=float, default=0.05)
    args = ap.parse_args()
    wl = dataclasses.replace(synth.WORKLOADS["resblock_320x128x128"], H=args.size, W=args.size,
                             drift=args.drift, name=f"resblock_320x{args.size}x{args.size}")
    wts = {n: v.double().numpy() for n, v in synth.make_weights(wl).items()}
    n = args.steps + 1
    exact = chain(wl, wts, [O.SYNC] * n)
    rows = [("naive (no context)", chain(wl, wts, [O.NAIVE] * n))]
    for name, v in VARIANTS:
        rows.append((name, chain(wl, wts, [O.SYNC] + [O.DISPLACED] * args.steps, v)))
    print(f"{wl.name}, P={wl.P}, drift {args.drift}: rel-L2 of displaced steps 1..{args.steps} "
          f"against the synchronous block")
    for name, outs in rows:
        errs = [np.linalg.norm(outs[k] - exact[k]) / np.linalg.norm(exact[k]) for k in range(1, n)]
        print(f"  {name:20s} " + " ".join(f"{e:.3e}" for e in errs))


if __name__ == "__main__":
    main()
