"""One decode sharded over the ranks of a process group (one GPU per rank).

A long or stereo decode splits into independent units -- unit u = k B + b is
time tile k of side b (the stereo sides are independent mono passes, as both
decoders run them, and the tiles of a tiled decode are independent decodes,
as in docs.rs cortiq-engine music3.rs `Music3Dit::forward_windowed`).  The
units are partitioned into contiguous ranges, ceil(units / world) per rank
(the last non-empty rank may hold fewer, later ranks none); every rank decodes
its range with the library's unit decode, one all-gather brings every unit
row to every rank (collective over NCCL between GPUs, gloo in the CPU
tests), and the root stitches them with the library's overlap average.
Because the ranges are contiguous and all but the last are full, the
gathered rows are already in unit order.  The result equals the one-GPU
decode bit for bit: the same kernels decode each unit, rows independently.

The decoder object needs ``tile_count(frames)``, ``unit_length(frames)``,
``decode_units(z, u0, u1, y_units=...)``, ``stitch_units(rows, B, frames)``
and ``cfg.out_channels`` -- ``native.Decoder`` has them.
"""
from __future__ import annotations

from typing import List, Tuple

import torch


def unit_ranges(n_units: int, world: int) -> Tuple[List[Tuple[int, int]], int]:
    """Contiguous unit ranges of every rank and the rows each rank sends."""
    if n_units < 1 or world < 1:
        raise ValueError(f"{n_units} units over {world} ranks")
    per = -(-n_units // world)
    ranges = [(min(r * per, n_units), min((r + 1) * per, n_units)) for r in range(world)]
    return ranges, per


def decode_sharded(dec, z: torch.Tensor, group=None, root: int = 0):
    """Decode z [B, in_channels, frames] over the ranks of `group`; returns
    y [B, out_channels, frames hop] on `root` and None elsewhere.  Every
    rank passes the whole latent (it reads only its units' frames)."""
    import torch.distributed as dist
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    B, F = dec._bf(z) if hasattr(dec, "_bf") else (z.shape[0], z.shape[2])
    n_units = dec.tile_count(F) * B
    ranges, per = unit_ranges(n_units, world)
    u0, u1 = ranges[rank]
    O, P = dec.cfg.out_channels, dec.unit_length(F)
    rows = torch.empty((per, O, P), device=z.device, dtype=torch.float32)
    if u1 > u0:
        dec.decode_units(z, u0, u1, y_units=rows[: u1 - u0])
    gathered = torch.empty((world * per, O, P), device=z.device, dtype=torch.float32)
    dist.all_gather_into_tensor(gathered, rows, group=group)
    if rank != root:
        return None
    return dec.stitch_units(gathered[:n_units], B, F)
