"""Full-size decoders on the GPU against the oracle's waveform.

The oracle needs minutes per full decode, so its outputs at sampled
positions are stored in tests/golden/<workload>.npz by
tests/golden/make_decoder_goldens.py (which calls only the oracle and the
seeded generator).  Positions: windows at the start, middle and end (and at
the tile overlaps of the tiled workload) plus uniform picks.  The whole
waveform must agree within 1e-4 relative L2.
"""
import os

import numpy as np
import pytest
import torch

from bigvgan_waveform_decoder_alias_b200 import synth

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
WAVE_TOL = 1e-4


def rel_l2(got, want):
    got, want = np.asarray(got, np.float64), np.asarray(want, np.float64)
    return float(np.linalg.norm(got - want) / np.linalg.norm(want))


@pytest.fixture(scope="module")
def nat():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from bigvgan_waveform_decoder_alias_b200 import build_native, native
    build_native.build()
    native.lib()
    return native


@pytest.mark.parametrize("tf32_only", [False, True], ids=["default-split", "3xtf32"])
@pytest.mark.parametrize("name", sorted(synth.DECODER_WORKLOADS))
def test_full_size_decoder_matches_oracle(nat, name, tf32_only):
    """Both conv splits: the default (fp16 parts for the AMP convs that
    qualify) and 3xTF32 throughout."""
    g = np.load(os.path.join(GOLDEN, f"{name}.npz"))
    w = synth.DECODER_WORKLOADS[name]
    z, params = w.make()
    dec = nat.Decoder(w.geometry, params, tile_frames=w.tile_frames,
                      overlap_frames=w.overlap_frames, tf32_only=tf32_only)
    y = dec.decode(torch.from_numpy(z).cuda()).cpu().numpy()
    L = w.frames * w.geometry.hop
    assert y.shape == (w.batch, 1, L)
    idx, want = g["idx"], g["value"]
    got = y[:, 0, idx]
    err = rel_l2(got, want)
    print(f"{name} ({'3xTF32' if tf32_only else 'default split'}): rel-L2 vs oracle {err:.3e} "
          f"over {idx.size} positions x {w.batch} rows, max abs {np.abs(got - want).max():.3e}")
    assert err < WAVE_TOL
    for b in range(w.batch):
        assert rel_l2(got[b], want[b]) < WAVE_TOL
    # the geometry checks the pages run on a decoded waveform
    assert np.isfinite(y).all()
    if w.geometry.final_act in ("tanh", "clamp"):
        assert np.abs(y).max() <= 1.0
    assert np.sqrt(np.mean(y.astype(np.float64) ** 2)) > 1e-4
    assert np.abs(y[0] - y[1]).max() > 0


def test_tiled_long_form_vs_untiled(nat):
    """Tiling changes the result only near tile edges; report how much (the
    tiles are independent decodes by definition, so this is not pinned)."""
    w = synth.H3_60S_TILED
    z, params = w.make()
    zd = torch.from_numpy(z[..., :400]).cuda().contiguous()
    tiled = nat.Decoder(w.geometry, params, tile_frames=w.tile_frames,
                        overlap_frames=w.overlap_frames)
    whole = nat.Decoder(w.geometry, params)
    a = tiled.decode(zd).cpu().numpy()
    b = whole.decode(zd).cpu().numpy()
    d = rel_l2(a, b)
    print(f"tiled (200/16) vs untiled on 400 frames: rel-L2 {d:.3e}")
    assert np.isfinite(d) and d < 1.0
    hop = w.geometry.hop
    # far from every tile edge the two agree closely
    core = slice(60 * hop, 120 * hop)
    assert rel_l2(a[..., core], b[..., core]) < 1e-3
