"""Pins for the oracle's video-aware block organisation and its inverse.

Block organisation (FVAttn pages, paperlayer.ai summary, section 3 "FVAttn
Design", item "Sparse-routing frontend"): spatially adjacent tokens must
share blocks.  Reading: tf x th x tw tiles, tiles numbered in raster order,
tokens inside a tile in raster order, padding zero.
"""
import numpy as np
import pytest

from block_sparse_attention_aware_b200 import synth

GEOMS = [
    dict(B=1, H=2, D=8, F=2, Hs=8, Ws=8, tf=2, th=2, tw=4),      # tiny tiling, no padding
    dict(B=2, H=3, D=8, F=3, Hs=5, Ws=7, tf=2, th=2, tw=4),      # padding on every axis
    dict(B=1, H=1, D=16, F=5, Hs=9, Ws=10, tf=2, th=8, tw=8),    # 128-token blocks, heavy pad
    dict(B=1, H=2, D=8, F=3, Hs=9, Ws=17, tf=1, th=8, tw=8),     # 64-token blocks
    dict(B=1, H=1, D=8, F=1, Hs=1, Ws=1, tf=2, th=8, tw=8),      # a single real token
]


def _w(g):
    return synth.custom_workload(**g)


def _coords(w):
    f, y, x = np.meshgrid(np.arange(w.F), np.arange(w.Hs), np.arange(w.Ws), indexing="ij")
    return f.ravel(), y.ravel(), x.ravel()


@pytest.mark.parametrize("g", GEOMS)
def test_roundtrip_is_identity(orc, g):
    w = _w(g)
    rng = np.random.default_rng(0)
    x = rng.integers(0, 1 << 16, size=(w.B, w.N, w.H, w.D), dtype=np.uint16)
    t = orc.reorder(x, w)
    back = orc.inverse_reorder(t, w)
    assert np.array_equal(back, x)


@pytest.mark.parametrize("g", GEOMS)
def test_permutation_and_padding(orc, g):
    """Every real token appears exactly once; every other row is zero."""
    w = _w(g)
    geo = orc.geometry(w)
    # encode (b, n, h) into the row so each row is unique and non-zero
    x = np.zeros((w.B, w.N, w.H, w.D), dtype=np.uint16)
    b, n, h = np.meshgrid(np.arange(w.B), np.arange(w.N), np.arange(w.H), indexing="ij")
    x[..., 0] = (n + 1).astype(np.uint16)
    x[..., 1] = (h + 1).astype(np.uint16)
    x[..., 2] = (b + 1).astype(np.uint16)
    t = orc.reorder(x, w)
    assert t.shape == (w.B, w.H, geo["Npad"], w.D)
    for bb in range(w.B):
        for hh in range(w.H):
            rows = t[bb, hh]
            real = rows[:, 0] != 0
            assert real.sum() == w.N
            assert np.all(rows[~real] == 0)
            assert np.all(rows[real, 1] == hh + 1) and np.all(rows[real, 2] == bb + 1)
            assert sorted(rows[real, 0].tolist()) == list(range(1, w.N + 1))


@pytest.mark.parametrize("g", GEOMS)
def test_block_membership_and_order(orc, g):
    """Blocks hold exactly one tile each, tiles in raster order, tokens in raster order."""
    w = _w(g)
    geo = orc.geometry(w)
    bs, nb = geo["bs"], geo["nb"]
    x = np.zeros((1, w.N, 1, 8), dtype=np.uint16)
    x[0, :, 0, 0] = np.arange(1, w.N + 1, dtype=np.uint16)
    w1 = synth.custom_workload(**{**g, "B": 1, "H": 1, "D": 8})
    t = orc.reorder(x, w1)[0, 0, :, 0].astype(np.int64)
    f, y, xx = _coords(w)
    tile_keys = []
    for blk in range(nb):
        ids = t[blk * bs:(blk + 1) * bs]
        real = ids[ids != 0] - 1
        assert len(real) > 0, "no block may be pure padding"
        tf_, ty_, tx_ = f[real] // w.tf, y[real] // w.th, xx[real] // w.tw
        assert len(set(zip(tf_, ty_, tx_))) == 1, "a block must hold a single tile"
        tile_keys.append((tf_[0], ty_[0], tx_[0]))
        # tokens inside the tile keep raster order
        assert np.all(np.diff(real) > 0)
        # the tile is complete: every real token of that tile is in this block
        in_tile = (f // w.tf == tf_[0]) & (y // w.th == ty_[0]) & (xx // w.tw == tx_[0])
        assert in_tile.sum() == len(real)
    assert tile_keys == sorted(tile_keys), "tiles must be numbered in raster order"


def test_closed_form_positions(orc):
    """Hand-derived positions for the 2x8x8 tiling of a 21x45x80 latent."""
    w = synth.custom_workload(B=1, H=1, D=8, F=21, Hs=45, Ws=80, tf=2, th=8, tw=8)
    geo = orc.geometry(w)
    assert (geo["Fp"], geo["Hp"], geo["Wp"], geo["nb"], geo["Npad"]) == (22, 48, 80, 660, 84480)
    x = np.zeros((1, w.N, 1, 8), dtype=np.uint16)

    def where(f, y, xx):
        n = (f * w.Hs + y) * w.Ws + xx
        x[:] = 0
        x[0, n, 0, 0] = 7
        t = orc.reorder(x, w)[0, 0, :, 0]
        pos = np.nonzero(t)[0]
        assert len(pos) == 1
        return int(pos[0])

    assert where(0, 0, 0) == 0
    # inside tile 0 the offset is (f*8 + y)*8 + x
    assert where(1, 2, 3) == (1 * 8 + 2) * 8 + 3
    # one tile to the right: block 1
    assert where(0, 0, 8) == 128
    # one tile row down: block 10 (80/8 = 10 tiles per row)
    assert where(0, 8, 0) == 10 * 128
    # next tile frame: block 60 (6 tile rows x 10 tile cols)
    assert where(2, 0, 0) == 60 * 128
    # last real token: frame 20 (tile frame 10, offset frame 0), row 44 (tile 5,
    # offset 4), col 79 (tile 9, offset 7)
    assert where(20, 44, 79) == (10 * 60 + 5 * 10 + 9) * 128 + (0 * 8 + 4) * 8 + 7


def test_geometry_matches_configs(orc):
    """Padded extents and block counts of the named workloads."""
    expect = {"tiny": (2, 8, 8, 16, 8), "480p": (22, 32, 56, 128, 308),
              "720p": (22, 48, 80, 128, 660), "cfg720p": (21, 48, 80, 64, 1260)}
    for name, (Fp, Hp, Wp, bs, nb) in expect.items():
        geo = orc.geometry(synth.WORKLOADS[name])
        assert (geo["Fp"], geo["Hp"], geo["Wp"], geo["bs"], geo["nb"]) == (Fp, Hp, Wp, bs, nb)
