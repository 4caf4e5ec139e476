"""Host-side logic of the binding that needs no GPU."""
import pytest

from block_sparse_attention_aware_b200 import fvattn


@pytest.mark.parametrize("H", [1, 2, 3, 4, 5, 6, 7, 9, 12, 40])
def test_default_head_group_sizes(H):
    sizes = fvattn.default_head_group_sizes(H)
    assert sum(sizes) == H
    assert sizes[0] == 1 and sizes[-1] == 1
    assert all(s in (1, 2) for s in sizes)
    # the middle groups hold two heads each (one leftover head joins the end)
    assert all(s == 2 for s in sizes[1:-2])
    if H == 40:
        assert sizes == [1] + [2] * 19 + [1]


def test_head_group_sizes_rejected():
    with pytest.raises(ValueError):
        fvattn.default_head_group_sizes(0)


@pytest.mark.parametrize("groups", [3, 0, [1, 2], [2, 2, 1], [0, 4], []])
def test_host_pipeline_rejects_bad_groups(fv, groups):
    """HostPipeline checks its head grouping before it allocates anything:
    equal groups must divide H, and a list of sizes must partition it."""
    g = fv.geom(1, 4, 64, 2, 8, 8, 2, 2, 4)
    with pytest.raises(ValueError):
        fv.HostPipeline(g, 0.9, 2, groups=groups, device="cpu")


@pytest.fixture(scope="module")
def fv():
    from block_sparse_attention_aware_b200 import build
    build.build()
    fvattn.load()
    return fvattn


def test_binding_rejects_bad_buffers_before_any_launch(fv):
    """Wrong shape, dtype, layout or device raises ValueError in the binding:
    the kernels read and write dense buffers of exactly the documented shape."""
    import torch
    g = fv.geom(1, 2, 64, 2, 8, 8, 2, 2, 4)
    raster = (g.B, g.N, g.H, g.D)
    tiled = (g.B, g.H, g.Npad, g.D)
    bf = torch.bfloat16
    with pytest.raises(ValueError):            # host tensor
        fv.reorder(g, torch.zeros(raster, dtype=bf))
    with pytest.raises(ValueError):            # wrong shape
        fv.reorder(g, torch.zeros((1, g.N, 3, g.D), dtype=bf))
    with pytest.raises(ValueError):            # a strided view of a wider tensor
        fv.reorder(g, torch.zeros((1, g.N, 4, g.D), dtype=bf)[:, :, :2])
    with pytest.raises(ValueError):
        fv.inverse_reorder(g, torch.zeros(tiled, dtype=torch.float16))
    with pytest.raises(ValueError):
        fv.route(g, torch.zeros(tiled, dtype=bf), torch.zeros(tiled, dtype=bf), 0.9, 1)
    with pytest.raises(ValueError):
        fv.reorder_route(g, torch.zeros(raster, dtype=bf), torch.zeros(raster, dtype=bf), 0.9, 1)
    t = torch.zeros(tiled, dtype=bf)
    idx = torch.zeros((g.B, g.H, g.nb, g.nb), dtype=torch.int64)
    cnt = torch.ones((g.B, g.H, g.nb), dtype=torch.int32)
    for call in (fv.sparse_attn, fv.sparse_attn_raster, fv.sparse_attn_noalloc):
        with pytest.raises(ValueError):
            call(g, t, t, t, idx, cnt)


def test_valid_token_flops_against_brute_force():
    """bench's real-token FLOP count: padding rows and columns of partial
    blocks excluded, entries past kv_cnt ignored (here filled with junk)."""
    import torch
    import bench
    g = fvattn.Geom(B=2, H=3, D=64, F=3, Hs=5, Ws=7, tf=2, th=2, tw=4)
    g.nbf, g.nby, g.nbx = 2, 3, 2
    g.nb, g.bs = 12, 16
    counts = bench.block_real_counts(g)
    # brute force over the token grid
    want = [0] * g.nb
    for f in range(g.F):
        for y in range(g.Hs):
            for x in range(g.Ws):
                want[((f // g.tf) * g.nby + y // g.th) * g.nbx + x // g.tw] += 1
    assert counts == want and sum(counts) == g.F * g.Hs * g.Ws
    gen = torch.Generator().manual_seed(3)
    kv_cnt = torch.randint(1, g.nb + 1, (g.B, g.H, g.nb), generator=gen, dtype=torch.int32)
    kv_idx = torch.randint(-50, 50, (g.B, g.H, g.nb, g.nb), generator=gen, dtype=torch.int32)
    ref = 0
    for b in range(g.B):
        for h in range(g.H):
            for i in range(g.nb):
                c = int(kv_cnt[b, h, i])
                kept = torch.randperm(g.nb, generator=gen)[:c]
                kv_idx[b, h, i, :c] = kept.to(torch.int32)
                ref += counts[i] * sum(counts[j] for j in kept.tolist())
    got = bench.valid_token_flops(g, kv_idx, kv_cnt, counts, rows_per_chunk=4)
    assert got == 4.0 * g.D * ref
    # Hilbert-style table: counts follow each block's tile
    table = list(reversed(range(g.nb)))
    assert bench.block_real_counts(g, table) == list(reversed(counts))
