"""Write the decoder golden files: oracle outputs at sampled positions of the
full-size synthetic decoders (the oracle takes minutes per decode, too long
for a test run).

Calls only ``oracle`` and the seeded input generator.  Each side (batch row)
and tile range is one job; jobs run in a spawn process pool.

    python tests/golden/make_decoder_goldens.py [--jobs 8]

Writes tests/golden/<workload>.npz with
  idx    int64 [n]        sample positions (the same for every row)
  value  float32 [B, n]   oracle waveform at those positions
  count  float32 [n]      tiles covering the position (tiled workload only)
  meta   str              workload, seed, positions recipe
"""
import argparse
import multiprocessing as mp
import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def positions(L, exact_ranges, n_random, seed):
    """Windows at the start, the middle and the end of each exact range, the
    edges of the tile overlaps inside it, and n_random uniform positions."""
    rng = np.random.default_rng(seed)
    picks = []
    for lo, hi, edges in exact_ranges:
        w = min(2048, (hi - lo) // 4)
        for c in [lo + w // 2, (lo + hi) // 2, hi - w // 2] + list(edges):
            a = max(lo, min(hi - w, c - w // 2))
            picks.append(np.arange(a, a + w))
        span = np.concatenate([np.arange(lo, hi)])
        picks.append(rng.choice(span, size=min(n_random, hi - lo), replace=False))
    idx = np.unique(np.concatenate(picks)).astype(np.int64)
    assert idx.min() >= 0 and idx.max() < L
    return idx


def _job(args):
    name, b, tiles = args
    import oracle
    from bigvgan_waveform_decoder_alias_b200 import synth
    w = synth.DECODER_WORKLOADS[name]
    z, params = w.make()
    t = time.time()
    if tiles is None:
        y = oracle.decode(w.geometry, params, z[b:b + 1])
        cnt = None
    else:
        y, cnt = oracle.decode_tiled(w.geometry, params, z[b:b + 1], w.tile_frames,
                                     w.overlap_frames, tiles=tiles)
    return name, b, tiles, y[0, 0], cnt, time.time() - t


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--jobs", type=int, default=os.cpu_count())
    ap.add_argument("--only", default=None)
    args = ap.parse_args()
    from bigvgan_waveform_decoder_alias_b200 import synth
    import oracle

    plans = {}
    for name, w in synth.DECODER_WORKLOADS.items():
        if args.only and name != args.only:
            continue
        hop = w.geometry.hop
        L = w.frames * hop
        if w.tile_frames:
            step = w.tile_frames - w.overlap_frames
            nt = oracle.tile_count(w.frames, w.tile_frames, w.overlap_frames)
            starts = [k * step for k in range(nt)]
            # tiles 0-1 fix every sample before tile 2 starts; the last two
            # tiles fix every sample after tile nt-3 ends; two middle tiles m,
            # m+1 fix every sample between the end of tile m-1 and the start
            # of tile m+2
            head = (0, starts[2] * hop, [starts[1] * hop, w.tile_frames * hop])
            tail_lo = (starts[nt - 3] + w.tile_frames) * hop
            tail = (tail_lo, L, [starts[nt - 1] * hop, (starts[nt - 2] + w.tile_frames) * hop])
            m = nt // 2
            mid = ((starts[m - 1] + w.tile_frames) * hop, starts[m + 2] * hop,
                   [starts[m + 1] * hop, (starts[m] + w.tile_frames) * hop])
            plans[name] = (positions(L, [head, mid, tail], 4096, w.seed),
                           [(0, 2), (m, m + 2), (nt - 2, nt)])
        else:
            plans[name] = (positions(L, [(0, L, [])], 4096, w.seed), [None])

    jobs = [(name, b, tiles) for name, (_, tl) in plans.items()
            for b in range(synth.DECODER_WORKLOADS[name].batch) for tiles in tl]
    print(f"{len(jobs)} jobs on {args.jobs} processes", flush=True)
    ctx = mp.get_context("spawn")
    results = {}
    with ctx.Pool(args.jobs) as pool:
        for name, b, tiles, y, cnt, dt in pool.imap_unordered(_job, jobs):
            print(f"  {name} side {b} tiles {tiles}: {dt:.0f} s", flush=True)
            results[(name, b, tiles)] = (y, cnt)

    for name, (idx, tl) in plans.items():
        w = synth.DECODER_WORKLOADS[name]
        vals = np.zeros((w.batch, idx.size), np.float32)
        count = np.zeros(idx.size, np.float32)
        for b in range(w.batch):
            full = np.full(w.frames * w.geometry.hop, np.nan, np.float32)
            cov = np.zeros(w.frames * w.geometry.hop, np.float32)
            for tiles in tl:
                y, cnt = results[(name, b, tiles)]
                ok = ~np.isnan(y)
                full[ok] = y[ok]
                if cnt is not None:
                    cov = np.maximum(cov, cnt)
            assert not np.isnan(full[idx]).any(), name
            vals[b] = full[idx]
            if w.tile_frames:
                count = cov[idx]
        meta = (f"workload={name} seed={w.seed} batch={w.batch} frames={w.frames} "
                f"tile={w.tile_frames} overlap={w.overlap_frames}; oracle decode, float "
                f"stores; positions: windows + uniform picks (seed {w.seed})")
        out = os.path.join(HERE, f"{name}.npz")
        np.savez_compressed(out, idx=idx, value=vals, count=count, meta=np.array(meta))
        print(f"wrote {out}: {idx.size} positions x {w.batch} rows")


if __name__ == "__main__":
    main()
