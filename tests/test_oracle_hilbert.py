"""Pins for the oracle's Hilbert block order.

FVAttn pages, paperlayer.ai summary, section 3 "FVAttn Design", item
"Sparse-routing frontend": Hilbert-curve block reordering places spatially
adjacent tokens in nearby blocks.  Reading: the tf x th x tw tile grid sits in
the smallest cube of side 2^b that holds it, and blocks are numbered by
increasing index of their tile along the 3-D Hilbert curve of that cube;
tokens inside a tile keep raster order.

The pins use the defining properties of a Hilbert curve (a walk through
face-adjacent cells that visits every aligned sub-cube in one contiguous
stretch), not a second copy of the index formula.
"""
import numpy as np
import pytest

from block_sparse_attention_aware_b200 import synth


def _cells(order, ny, nx):
    order = np.asarray(order, dtype=np.int64)
    return np.stack([order // (ny * nx), (order // nx) % ny, order % nx], axis=1)


@pytest.mark.parametrize("side", [2, 4, 8, 16])
def test_cube_walk_is_face_adjacent_from_the_origin(orc, side):
    t = orc.block_order(side, side, side)
    assert np.array_equal(np.sort(t), np.arange(side ** 3))
    c = _cells(t, side, side)
    assert np.array_equal(c[0], [0, 0, 0])
    step = np.abs(np.diff(c, axis=0)).sum(axis=1)
    assert np.all(step == 1)


@pytest.mark.parametrize("side,sub", [(4, 2), (8, 2), (8, 4), (16, 4)])
def test_aligned_subcubes_are_contiguous(orc, side, sub):
    t = orc.block_order(side, side, side)
    c = _cells(t, side, side)
    cube_id = (c[:, 0] // sub) * (side // sub) ** 2 + (c[:, 1] // sub) * (side // sub) + c[:, 2] // sub
    # each sub-cube's blocks form one run of sub^3 consecutive indices
    runs = np.nonzero(np.diff(cube_id))[0]
    assert len(runs) == (side // sub) ** 3 - 1
    assert np.all(np.diff(np.concatenate([[-1], runs, [side ** 3 - 1]])) == sub ** 3)


@pytest.mark.parametrize("dims", [(11, 6, 10), (22, 6, 10), (3, 1, 1), (1, 4, 7), (5, 3, 3)])
def test_grid_order_follows_the_enclosing_cube(orc, dims):
    """A non-cube grid keeps the enclosing cube's visiting order of its tiles."""
    nbf, nby, nbx = dims
    t = orc.block_order(nbf, nby, nbx)
    assert np.array_equal(np.sort(t), np.arange(nbf * nby * nbx))
    side = 1 << max(1, int(np.ceil(np.log2(max(dims)))))
    cube = _cells(orc.block_order(side, side, side), side, side)
    inside = (cube[:, 0] < nbf) & (cube[:, 1] < nby) & (cube[:, 2] < nbx)
    want = (cube[inside, 0] * nby + cube[inside, 1]) * nbx + cube[inside, 2]
    assert np.array_equal(t, want)


GEOMS = [
    dict(B=1, H=2, D=8, F=4, Hs=8, Ws=16, tf=2, th=2, tw=4),      # 2 x 4 x 4 tiles
    dict(B=2, H=1, D=8, F=3, Hs=5, Ws=7, tf=2, th=2, tw=4),       # padding on every axis
    dict(B=1, H=1, D=16, F=5, Hs=19, Ws=21, tf=2, th=8, tw=8),    # 3 x 3 x 3 tiles, partial ones
]


@pytest.mark.parametrize("g", GEOMS)
def test_hilbert_reorder_places_tiles_in_curve_order(orc, g):
    w = synth.custom_workload(order="hilbert", **g)
    geo = orc.geometry(w)
    bs, nb = geo["bs"], geo["nb"]
    t_of_b = orc.block_order(geo["nbf"], geo["nby"], geo["nbx"])
    x = np.zeros((1, w.N, 1, 8), dtype=np.uint16)
    x[0, :, 0, 0] = np.arange(1, w.N + 1, dtype=np.uint16)
    w1 = synth.custom_workload(**{**g, "B": 1, "H": 1, "D": 8, "order": "hilbert"})
    t = orc.reorder(x, w1)[0, 0, :, 0].astype(np.int64)
    f, y, xx = np.meshgrid(np.arange(w.F), np.arange(w.Hs), np.arange(w.Ws), indexing="ij")
    f, y, xx = f.ravel(), y.ravel(), xx.ravel()
    raster_tile = ((f // w.tf) * geo["nby"] + y // w.th) * geo["nbx"] + xx // w.tw
    for blk in range(nb):
        ids = t[blk * bs:(blk + 1) * bs]
        real = ids[ids != 0] - 1
        assert np.all(raster_tile[real] == t_of_b[blk])            # the block holds its curve tile
        assert np.all(np.diff(real) > 0)                           # tokens keep raster order
        assert (raster_tile == t_of_b[blk]).sum() == len(real)     # and all of them
    # round trip on random bits, and the block valid counts follow the tiles
    rng = np.random.default_rng(3)
    xr = rng.integers(0, 1 << 16, size=(w.B, w.N, w.H, w.D), dtype=np.uint16)
    assert np.array_equal(orc.inverse_reorder(orc.reorder(xr, w), w), xr)
    raster_counts = orc.block_valid_counts(synth.custom_workload(**g))
    assert np.array_equal(orc.block_valid_counts(w), raster_counts[t_of_b])


@pytest.mark.parametrize("g", GEOMS)
def test_hilbert_pool_is_the_tile_mean(orc, g):
    w = synth.custom_workload(order="hilbert", seed=4, **g)
    geo = orc.geometry(w)
    q, _, _, _ = synth.make_qkv(w)
    bits = synth.bf16_bits(q)
    qp = orc.pool(orc.reorder(bits, w), w)
    vals = bits.astype(np.uint32) << 16
    qf = vals.view(np.float32).astype(np.float64)          # [B, N, H, D]
    f, y, xx = np.meshgrid(np.arange(w.F), np.arange(w.Hs), np.arange(w.Ws), indexing="ij")
    raster_tile = (((f // w.tf) * geo["nby"] + y // w.th) * geo["nbx"] + xx // w.tw).ravel()
    t_of_b = orc.block_order(geo["nbf"], geo["nby"], geo["nbx"])
    for blk in range(geo["nb"]):
        sel = raster_tile == t_of_b[blk]
        want = qf[:, sel].mean(axis=1)                      # [B, H, D]
        assert np.allclose(qp[:, :, blk], want, rtol=0, atol=1e-12)


@pytest.mark.parametrize("g", GEOMS)
def test_hilbert_dense_attention_is_order_free(orc, g):
    """With every block kept the output does not depend on the block order."""
    w_r = synth.custom_workload(seed=5, **g)
    w_h = synth.custom_workload(seed=5, order="hilbert", **g)
    geo = orc.geometry(w_r)
    q, k, v, _ = synth.make_qkv(w_r)
    nb = geo["nb"]
    idx = np.tile(np.arange(nb, dtype=np.int32), (w_r.B * w_r.H * nb, 1))
    cnt = np.full(w_r.B * w_r.H * nb, nb, dtype=np.int32)
    items = list(range(w_r.B * w_r.H * nb))
    outs = []
    for w in (w_r, w_h):
        qt, kt, vt = (orc.reorder(synth.bf16_bits(t), w) for t in (q, k, v))
        o = orc.attention(qt, kt, vt, idx, cnt, items, w, 1.0 / np.sqrt(w.D))
        tiled = o.reshape(w.B, w.H, geo["Npad"], w.D)
        # back to raster through the oracle's own reorder of a token probe
        probe = np.zeros((1, w.N, 1, 8), dtype=np.uint16)
        probe[0, :, 0, 0] = np.arange(1, w.N + 1)
        tp = orc.reorder(probe, synth.custom_workload(**{**w.as_dict(), "B": 1, "H": 1, "D": 8}))[0, 0, :, 0]
        real = np.nonzero(tp)[0]
        ras = np.zeros((w.B, w.N, w.H, w.D))
        ras[:, tp[real].astype(np.int64) - 1] = np.transpose(tiled[:, :, real], (0, 2, 1, 3))
        outs.append(ras)
    assert np.allclose(outs[0], outs[1], rtol=0, atol=1e-12)
