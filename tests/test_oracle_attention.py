"""Pins for the oracle's masked block attention.

FVAttn pages, paperlayer.ai summary, section 2 (dynamic block-sparse
attention) and section 3 "Pipeline" (block-sparse attention on the
materialised mask, then restoration of the original layout).  The oracle
works in the tiled layout; the pins below work in raster layout and never
tile anything, so they also cross-check the block organisation.
"""
import numpy as np
import pytest
import torch

from block_sparse_attention_aware_b200 import synth

GEOMS = [
    dict(B=1, H=2, D=16, F=2, Hs=8, Ws=8, tf=2, th=2, tw=4),
    dict(B=2, H=1, D=8, F=3, Hs=5, Ws=7, tf=2, th=2, tw=4),
    dict(B=1, H=1, D=16, F=3, Hs=9, Ws=9, tf=2, th=8, tw=8),
]


def _setup(g, seed=0):
    w = synth.custom_workload(seed=seed, **g)
    q, k, v, _ = synth.make_qkv(w)
    return w, q, k, v


def _tile_of_tokens(w, geo):
    f, y, x = np.meshgrid(np.arange(w.F), np.arange(w.Hs), np.arange(w.Ws), indexing="ij")
    return (((f // w.tf) * geo["nby"] + y // w.th) * geo["nbx"] + x // w.tw).ravel()


def _raster_masked_attention(q, k, v, allowed):
    """Textbook softmax attention in raster layout, fp64, with a token mask.

    q, k, v: [N, D] float64 for one (b, h); allowed: [N, N] bool."""
    D = q.shape[1]
    s = q @ k.T / np.sqrt(D)
    s = np.where(allowed, s, -np.inf)
    s = s - s.max(axis=1, keepdims=True)
    e = np.exp(s)
    return (e / e.sum(axis=1, keepdims=True)) @ v


def _oracle_raster_output(orc, w, q, k, v, kv_idx, kv_cnt):
    """Run the oracle on every item and scatter back to raster [B, N, H, D]."""
    geo = orc.geometry(w)
    qt, kt, vt = (orc.reorder(synth.bf16_bits(t), w) for t in (q, k, v))
    items = list(range(w.B * w.H * geo["nb"]))
    out = orc.attention(qt, kt, vt, kv_idx, kv_cnt, items, w, 1.0 / np.sqrt(w.D))
    tiled = out.reshape(w.B, w.H, geo["nb"] * geo["bs"], w.D)
    # inverse reorder through bit patterns of a float64 carrier is not
    # possible, so gather by the raster->tiled map of a coordinate tensor
    probe = np.zeros((1, w.N, 1, 8), dtype=np.uint16)
    probe[0, :, 0, 0] = np.arange(w.N) % 65536
    probe[0, :, 0, 1] = np.arange(w.N) // 65536 + 1
    tp = orc.reorder(probe, synth.custom_workload(**{**w.as_dict(), "B": 1, "H": 1, "D": 8}))
    tp = tp[0, 0]
    real = tp[:, 1] != 0
    n_of_pos = tp[:, 0].astype(np.int64) + (tp[:, 1].astype(np.int64) - 1) * 65536
    res = np.zeros((w.B, w.N, w.H, w.D))
    pos = np.nonzero(real)[0]
    res[:, n_of_pos[pos]] = np.transpose(tiled[:, :, pos], (0, 2, 1, 3))
    return res


@pytest.mark.parametrize("g", GEOMS)
def test_full_mask_equals_dense_attention(orc, g):
    """p = 1 keeps every block, so the output is plain dense attention."""
    w, q, k, v = _setup(g)
    geo = orc.geometry(w)
    nb = geo["nb"]
    kv_idx = np.tile(np.arange(nb, dtype=np.int32), (w.B, w.H, nb, 1))
    kv_cnt = np.full((w.B, w.H, nb), nb, dtype=np.int32)
    got = _oracle_raster_output(orc, w, q, k, v, kv_idx, kv_cnt)
    qd, kd, vd = (t.double().numpy() for t in (q, k, v))
    for b in range(w.B):
        for h in range(w.H):
            want = _raster_masked_attention(qd[b, :, h], kd[b, :, h], vd[b, :, h],
                                            np.ones((w.N, w.N), dtype=bool))
            np.testing.assert_allclose(got[b, :, h], want, rtol=0, atol=1e-12)


@pytest.mark.parametrize("order", ["raster", "hilbert"])
@pytest.mark.parametrize("g", GEOMS)
def test_block_mask_equals_token_mask(orc, g, order):
    """A routed block mask, expanded to tokens by tile membership in raster
    layout, gives the same attention as the oracle's block path (under either
    block order: a token's block is its tile's index in that order)."""
    w = synth.custom_workload(seed=7, order=order, **g)
    q, k, v, _ = synth.make_qkv(w)
    geo = orc.geometry(w)
    nb = geo["nb"]
    qt, kt = (orc.reorder(synth.bf16_bits(t), w) for t in (q, k))
    _, _, _, kv_idx, kv_cnt, _, _ = orc.route(qt, kt, w, 0.6, 1, 1.0 / np.sqrt(w.D))
    got = _oracle_raster_output(orc, w, q, k, v, kv_idx, kv_cnt)
    tile = _tile_of_tokens(w, geo)
    if order == "hilbert":
        block_of_tile = np.argsort(orc.block_order(geo["nbf"], geo["nby"], geo["nbx"]))
        tile = block_of_tile[tile]
    qd, kd, vd = (t.double().numpy() for t in (q, k, v))
    for b in range(w.B):
        for h in range(w.H):
            block_mask = np.zeros((nb, nb), dtype=bool)
            for i in range(nb):
                block_mask[i, kv_idx[b, h, i, :kv_cnt[b, h, i]]] = True
            allowed = block_mask[tile[:, None], tile[None, :]]
            want = _raster_masked_attention(qd[b, :, h], kd[b, :, h], vd[b, :, h], allowed)
            np.testing.assert_allclose(got[b, :, h], want, rtol=0, atol=1e-12)


def test_torch_sdpa_second_opinion(orc):
    """torch's scaled_dot_product_attention in fp64 on CPU, boolean mask."""
    g = GEOMS[1]
    w, q, k, v = _setup(g, seed=11)
    geo = orc.geometry(w)
    nb = geo["nb"]
    qt, kt = (orc.reorder(synth.bf16_bits(t), w) for t in (q, k))
    _, _, _, kv_idx, kv_cnt, _, _ = orc.route(qt, kt, w, 0.5, 1, 1.0 / np.sqrt(w.D))
    got = _oracle_raster_output(orc, w, q, k, v, kv_idx, kv_cnt)
    tile = _tile_of_tokens(w, geo)
    for b in range(w.B):
        for h in range(w.H):
            block_mask = np.zeros((nb, nb), dtype=bool)
            for i in range(nb):
                block_mask[i, kv_idx[b, h, i, :kv_cnt[b, h, i]]] = True
            allowed = torch.from_numpy(block_mask[tile[:, None], tile[None, :]])
            want = torch.nn.functional.scaled_dot_product_attention(
                q[b, :, h].double()[None], k[b, :, h].double()[None], v[b, :, h].double()[None],
                attn_mask=allowed[None])[0].numpy()
            np.testing.assert_allclose(got[b, :, h], want, rtol=0, atol=1e-12)


def test_single_kept_block_is_local_softmax(orc):
    """Keeping only block j for row i gives softmax over block j's real tokens."""
    w, q, k, v = _setup(GEOMS[1], seed=3)
    geo = orc.geometry(w)
    nb, bs = geo["nb"], geo["bs"]
    kv_idx = np.zeros((w.B, w.H, nb, nb), dtype=np.int32)
    kv_cnt = np.ones((w.B, w.H, nb), dtype=np.int32)
    j = nb - 1                        # a partial (padded) block
    kv_idx[..., 0] = j
    got = _oracle_raster_output(orc, w, q, k, v, kv_idx, kv_cnt)
    tile = _tile_of_tokens(w, geo)
    keys = np.nonzero(tile == j)[0]
    assert 0 < len(keys) < bs
    qd, kd, vd = (t.double().numpy() for t in (q, k, v))
    s = qd[0, :, 0] @ kd[0, keys, 0].T / np.sqrt(w.D)
    e = np.exp(s - s.max(axis=1, keepdims=True))
    want = (e / e.sum(axis=1, keepdims=True)) @ vd[0, keys, 0]
    np.testing.assert_allclose(got[0, :, 0], want, rtol=0, atol=1e-12)


@pytest.mark.parametrize("g", GEOMS)
def test_equal_scores_average_the_kept_values(orc, g):
    """Closed form: with every key zero all scores are equal, so each output
    row is the plain mean of V over the real tokens of its row's kept blocks
    (padding excluded, each kept block counted once).  No exponential is
    involved, so this pins the masking, the kept-set gather and the
    normalisation independently of any softmax implementation."""
    w, q, k, v = _setup(g, seed=11)
    k = torch.zeros_like(k)
    geo = orc.geometry(w)
    nb = geo["nb"]
    rng = np.random.default_rng(5)
    kv_idx = np.zeros((w.B, w.H, nb, nb), dtype=np.int32)
    kv_cnt = np.zeros((w.B, w.H, nb), dtype=np.int32)
    for b in range(w.B):
        for h in range(w.H):
            for i in range(nb):
                c = int(rng.integers(1, nb + 1))
                kv_idx[b, h, i, :c] = np.sort(rng.choice(nb, size=c, replace=False))
                kv_cnt[b, h, i] = c
    got = _oracle_raster_output(orc, w, q, k, v, kv_idx, kv_cnt)
    tile = _tile_of_tokens(w, geo)
    vd = v.double().numpy()
    for b in range(w.B):
        for h in range(w.H):
            for n in range(w.N):
                i = tile[n]
                kept = kv_idx[b, h, i, :kv_cnt[b, h, i]]
                keys = np.nonzero(np.isin(tile, kept))[0]
                want = vd[b, keys, h].mean(axis=0)
                np.testing.assert_allclose(got[b, n, h], want, rtol=0, atol=1e-12)
