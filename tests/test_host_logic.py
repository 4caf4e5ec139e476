"""Host-side logic of the binding that needs no GPU."""
import pytest

from block_sparse_attention_aware_b200 import fvattn


@pytest.mark.parametrize("H,want", [(40, 20), (4, 2), (2, 1), (1, 1), (3, 1), (6, 3), (9, 3), (7, 1), (12, 6)])
def test_default_head_groups(H, want):
    groups = fvattn.default_head_groups(H)
    assert groups == want
    assert H % groups == 0
    assert groups == 1 or H // groups >= 2


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
