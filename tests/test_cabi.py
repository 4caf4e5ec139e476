"""The C-ABI library without a GPU: it loads, exports every entry point that
include/fvattn.h declares, and rejects bad arguments on the host before any
launch (none of these calls reaches the CUDA runtime)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def fv():
    from block_sparse_attention_aware_b200 import build, fvattn
    build.build()
    fvattn.load()
    return fvattn


def _declared():
    src = open(os.path.join(ROOT, "include", "fvattn.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(fvattn_[a-z_]+)\s*\(", src)))


def test_exports_every_declared_symbol(fv):
    lib = fv.load()
    names = _declared()
    assert len(names) == 18
    assert sorted(fv.EXPORTED) == names
    for n in names:
        assert hasattr(lib, n), n


def test_geom_init_derives_padding(fv):
    g = fv.geom(1, 40, 128, 21, 45, 80, 2, 8, 8)
    assert (g.Fp, g.Hp, g.Wp, g.nbf, g.nby, g.nbx, g.bs, g.nb, g.N, g.Npad) == \
        (22, 48, 80, 11, 6, 10, 128, 660, 75600, 84480)
    g = fv.geom(2, 40, 128, 21, 45, 80, 1, 8, 8)
    assert (g.bs, g.nb, g.Npad) == (64, 1260, 80640)


@pytest.mark.parametrize("args,code", [
    ((1, 1, 96, 2, 8, 8, 2, 8, 8), 2),      # D not 64/128
    ((1, 1, 128, 2, 8, 8, 3, 8, 8), 2),     # bs = 192
    ((1, 1, 128, 2, 8, 8, 1, 2, 4), 1 + 1),  # bs = 8
    ((0, 1, 128, 2, 8, 8, 2, 8, 8), 1),     # B = 0
    ((1, 1, 128, 200, 256, 256, 1, 8, 8), 2),  # nb > 2560
])
def test_geom_init_rejects(fv, args, code):
    with pytest.raises(fv.FVAttnError) as e:
        fv.geom(*args)
    assert e.value.code == code


def test_null_and_misaligned_pointers_rejected(fv):
    lib = fv.load()
    g = fv.geom(1, 2, 64, 2, 8, 8, 2, 2, 4)
    gp = ctypes.byref(g)
    assert lib.fvattn_reorder(gp, None, None, None) == fv.ERR_INVALID
    assert lib.fvattn_inverse_reorder(gp, None, ctypes.c_void_p(16), None) == fv.ERR_INVALID
    assert lib.fvattn_reorder(gp, ctypes.c_void_p(18), ctypes.c_void_p(32), None) == fv.ERR_INVALID
    assert lib.fvattn_route(gp, ctypes.c_void_p(16), ctypes.c_void_p(32), 0.0, 1, 0.125, ctypes.c_void_p(48),
                            ctypes.c_void_p(64), None, None, None, None, 0, None) == fv.ERR_INVALID
    assert lib.fvattn_route(gp, ctypes.c_void_p(16), ctypes.c_void_p(32), 0.9, 0, 0.125, ctypes.c_void_p(48),
                            ctypes.c_void_p(64), None, None, None, None, 0, None) == fv.ERR_INVALID
    assert lib.fvattn_route(gp, ctypes.c_void_p(16), ctypes.c_void_p(32), 1.5, 1, 0.125, ctypes.c_void_p(48),
                            ctypes.c_void_p(64), None, None, None, None, 0, None) == fv.ERR_INVALID
    # routing variants: p in [0, 1], k_extra >= 0; plain routing needs p > 0
    assert lib.fvattn_route(gp, ctypes.c_void_p(16), ctypes.c_void_p(32), 0.0, 1, 0.125, ctypes.c_void_p(48),
                            ctypes.c_void_p(64), None, None, None, ctypes.c_void_p(256), 1 << 30, None) == fv.ERR_INVALID
    assert lib.fvattn_route_aug(gp, ctypes.c_void_p(16), ctypes.c_void_p(32), 0.5, 1, -1, 0.125, ctypes.c_void_p(48),
                                ctypes.c_void_p(64), None, None, None, ctypes.c_void_p(256), 1 << 30,
                                None) == fv.ERR_INVALID
    assert lib.fvattn_route_aug(gp, ctypes.c_void_p(16), ctypes.c_void_p(32), 1.5, 1, 0, 0.125, ctypes.c_void_p(48),
                                ctypes.c_void_p(64), None, None, None, ctypes.c_void_p(256), 1 << 30,
                                None) == fv.ERR_INVALID
    # fused reorder + routing: raster pointers, two distinct tile buffers, the route_aug parameter checks
    V = ctypes.c_void_p
    assert lib.fvattn_reorder_route(gp, None, V(16), V(32), V(48), 0.9, 1, 0, 0.125, V(64), V(80), None, None,
                                    None, V(256), 1 << 30, None) == fv.ERR_INVALID
    assert lib.fvattn_reorder_route(gp, V(16), V(24), V(32), V(48), 0.9, 1, 0, 0.125, V(64), V(80), None, None,
                                    None, V(256), 1 << 30, None) == fv.ERR_INVALID
    assert lib.fvattn_reorder_route(gp, V(16), V(32), V(48), V(48), 0.9, 1, 0, 0.125, V(64), V(80), None, None,
                                    None, V(256), 1 << 30, None) == fv.ERR_INVALID
    assert lib.fvattn_reorder_route(gp, V(16), V(32), V(48), V(64), 1.5, 1, 0, 0.125, V(80), V(96), None, None,
                                    None, V(256), 1 << 30, None) == fv.ERR_INVALID
    assert lib.fvattn_reorder_route(gp, V(16), V(32), V(48), V(64), 0.9, 1, -2, 0.125, V(80), V(96), None, None,
                                    None, V(256), 1 << 30, None) == fv.ERR_INVALID
    assert lib.fvattn_reorder_route(gp, V(16), V(32), V(48), V(64), 0.9, 1, 0, 0.125, V(80), V(96), None, None,
                                    None, V(256), 16, None) == fv.ERR_INVALID
    # workspace too small
    assert lib.fvattn_route(gp, ctypes.c_void_p(16), ctypes.c_void_p(32), 0.9, 1, 0.125, ctypes.c_void_p(48),
                            ctypes.c_void_p(64), None, None, None, ctypes.c_void_p(256), 16, None) == fv.ERR_INVALID
    assert lib.fvattn_sparse_attn(gp, None, None, None, None, None, 0.125, None, None, None, 0,
                                  None) == fv.ERR_INVALID
    assert lib.fvattn_sparse_attn(gp, *[ctypes.c_void_p(256)] * 5, 0.125, ctypes.c_void_p(256), None,
                                  ctypes.c_void_p(256), 0, None) == fv.ERR_INVALID


def test_copy_heads_rejects_bad_slices(fv):
    """fvattn_copy_heads checks the head slice before any copy is queued."""
    lib = fv.load()
    g = fv.geom(1, 4, 64, 2, 8, 8, 2, 2, 4)
    gp, V = ctypes.byref(g), ctypes.c_void_p
    for h0, nh in ((-1, 2), (0, 0), (3, 2), (0, 5)):
        assert lib.fvattn_copy_heads(gp, h0, nh, V(16), V(32), 1, None) == fv.ERR_INVALID
    assert lib.fvattn_copy_heads(gp, 0, 2, None, V(32), 1, None) == fv.ERR_INVALID
    assert lib.fvattn_copy_heads(gp, 0, 2, V(16), None, 0, None) == fv.ERR_INVALID
    assert lib.fvattn_copy_heads(None, 0, 2, V(16), V(32), 0, None) == fv.ERR_INVALID


def test_block_order_rejects_bad_arguments(fv):
    """fvattn_block_order: null or misaligned table, or a geometry whose tile
    counts do not multiply to nb, is refused before the launch."""
    lib = fv.load()
    g = fv.geom(1, 1, 64, 4, 8, 8, 1, 4, 4)
    V = ctypes.c_void_p
    assert lib.fvattn_block_order(ctypes.byref(g), None, None) == fv.ERR_INVALID
    assert lib.fvattn_block_order(ctypes.byref(g), V(20), None) == fv.ERR_INVALID
    assert lib.fvattn_block_order(None, V(32), None) == fv.ERR_INVALID
    bad = fv.Geom.from_buffer_copy(g)
    bad.nb = g.nb + 1
    assert lib.fvattn_block_order(ctypes.byref(bad), V(32), None) == fv.ERR_INVALID


def test_workspace_sizes(fv):
    lib = fv.load()
    g = fv.geom(1, 40, 128, 21, 45, 80, 2, 8, 8)
    rw = lib.fvattn_route_workspace_size(ctypes.byref(g))
    aw = lib.fvattn_attn_workspace_size(ctypes.byref(g))
    assert rw >= 4 * 40 * 660 * 128 * 4 + 40 * 660 * 660 * 4
    assert aw >= 40 * 660 * 4 + 40 * 8 + 40 * 4 + 4
    assert rw % 256 == 0 and aw % 256 == 0


def test_status_strings(fv):
    for c in range(6):
        assert fv.status_string(c) != "unknown status"
    assert fv.status_string(99) == "unknown status"


def test_product_path_has_no_oracle_import():
    """The CUDA path never imports or loads the oracle."""
    pkg = os.path.join(ROOT, "block_sparse_attention_aware_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"(import\s+oracle|from\s+oracle|liboracle|fvattn_oracle)", txt), f


def test_route_kernel_launches(fv):
    """Routing is three kernels: pooling, scoring, selection."""
    lib = fv.load()
    assert lib.fvattn_route_kernel_launches(None) == 0
    for B, H in ((1, 40), (2, 40), (1, 1)):
        assert fv.route_kernel_launches(fv.geom(B, H, 128, 21, 45, 80, 2, 8, 8)) == 3


def test_test_hook_rejects_unknown_flags(fv):
    """fvattn_test_hook (fault injection for failure-path tests) accepts only
    the documented flag and is reset by (0, 0); no GPU needed."""
    lib = fv.load()
    assert lib.fvattn_test_hook(0, 2) == fv.ERR_INVALID
    assert lib.fvattn_test_hook(0, -1) == fv.ERR_INVALID
    assert lib.fvattn_test_hook(1000, fv.HOOK_SKIP_V_LOADS) == fv.OK
    assert lib.fvattn_test_hook(0, 0) == fv.OK
