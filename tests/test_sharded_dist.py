"""One decode sharded over ranks: the host logic on CPU with gloo ranks.

Each rank decodes a contiguous range of (tile, side) units, one all-gather
brings every unit row to every rank, and the root stitches.  Here the unit
decode is the oracle's decode of the unit's latent frames and the stitch a
coverage average written in the test, so what is checked is the partition,
the gather and the reassembly: the root's waveform must equal the oracle's
own tiled decode (``oracle.decode_tiled``).  The GPU kernels behind the same
steps are checked in tests/test_gpu_parity.py.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from bigvgan_waveform_decoder_alias_b200 import sharded, synth  # noqa: E402

TILE, OVERLAP, FRAMES, SIDES = 6, 2, 23, 2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_unit_ranges_cover_every_unit_once():
    for n in (1, 2, 7, 26, 100):
        for world in (1, 2, 3, 4, 8, 30):
            ranges, per = sharded.unit_ranges(n, world)
            assert len(ranges) == world and per == -(-n // world)
            got = [u for a, b in ranges for u in range(a, b)]
            assert got == list(range(n))
            # every non-empty range but the last is full, so rank r's rows
            # start at unit r * per
            for r, (a, b) in enumerate(ranges):
                assert b - a <= per and (a == b or a == r * per)
    with pytest.raises(ValueError):
        sharded.unit_ranges(0, 2)


class OracleUnits:
    """The unit-level decoder interface, computed by the oracle on the CPU."""

    class _Cfg:
        out_channels = 1

    def __init__(self, geo, params, tile, overlap):
        import oracle
        self.o, self.geo, self.params = oracle, geo, params
        self.tile, self.overlap = tile, overlap
        self.cfg = self._Cfg()

    def tile_count(self, F):
        return self.o.tile_count(F, self.tile, self.overlap)

    def unit_length(self, F):
        return self.tile * self.geo.hop

    def decode_units(self, z, u0, u1, y_units):
        import torch
        B, _, F = z.shape
        step = self.tile - self.overlap
        zn = z.numpy()
        for u in range(u0, u1):
            k, b = divmod(u, B)
            n = min(self.tile, F - k * step)
            y = self.o.decode(self.geo, self.params, zn[b:b + 1, :, k * step:k * step + n])
            y_units[u - u0, :, :n * self.geo.hop] = torch.from_numpy(y[0])
        return y_units

    def stitch_units(self, rows, B, F):
        import torch
        step, hop = self.tile - self.overlap, self.geo.hop
        L = F * hop
        acc = np.zeros((B, 1, L))
        cnt = np.zeros(L)
        r = rows.numpy().astype(np.float64)
        for k in range(self.tile_count(F)):
            n = min(self.tile, F - k * step) * hop
            s = k * step * hop
            for b in range(B):
                acc[b, :, s:s + n] += r[k * B + b, :, :n]
            cnt[s:s + n] += 1
        return torch.from_numpy((acc / cnt).astype(np.float32))


def _inputs():
    geo = synth.tiny_geometry()
    s = synth.NormalStream(31)
    z = s.normal((SIDES, geo.in_channels, FRAMES))
    params = s.normal((synth.param_count(geo),), 0.0, 0.1)
    return geo, z, params


def _rank(rank, world, port, out):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        geo, z, params = _inputs()
        dec = OracleUnits(geo, params, TILE, OVERLAP)
        y = sharded.decode_sharded(dec, torch.from_numpy(z))
        out[rank] = None if y is None else y.numpy()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_decode_equals_oracle_tiled_decode(oracle, world):
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0
    assert all(out[r] is None for r in range(1, world))
    geo, z, params = _inputs()
    want, count = oracle.decode_tiled(geo, params, z, TILE, OVERLAP)
    n_tiles = oracle.tile_count(FRAMES, TILE, OVERLAP)
    assert n_tiles * SIDES > world  # several units per rank
    assert count.max() == 2  # the overlaps are exercised
    np.testing.assert_allclose(out[0], want, rtol=1e-6, atol=1e-7)
