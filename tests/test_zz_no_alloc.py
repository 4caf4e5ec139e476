"""fvattn_sparse_attn_noalloc: the attention entry point for callers that
cannot allocate device memory (for example a plugin whose host framework owns
all device memory, or a C caller with no device allocator).  It uses a
scratch array built into the library instead of a caller workspace, so its
results must match fvattn_sparse_attn's on the same inputs, call after call.

This file is named to be collected last, so a run that stops at the first
failure has already run every other test.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

from block_sparse_attention_aware_b200 import synth

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
MEAN_ABS = 2e-3

CASES = [
    synth.custom_workload(B=1, H=2, D=128, F=5, Hs=19, Ws=21, tf=2, th=8, tw=8, seed=6, p=0.9, k=3,
                          qscale="fixed", qscale_values=(1.0, 8.0)),
    synth.custom_workload(B=2, H=3, D=64, F=3, Hs=5, Ws=7, tf=2, th=2, tw=4, seed=5, p=0.8, k=2),
]


@pytest.fixture(scope="module")
def fv():
    from block_sparse_attention_aware_b200 import build, fvattn
    build.build()
    assert torch.cuda.is_available(), "needs a GPU"
    fvattn.load()
    return fvattn


def _real_rows_mask(w, g):
    """[nb, bs] bool: which tiled rows are real tokens."""
    mask = np.zeros((g.nb, g.bs), dtype=bool)
    for blk in range(g.nb):
        bx, by, bf = blk % g.nbx, (blk // g.nbx) % g.nby, blk // (g.nbx * g.nby)
        for o in range(g.bs):
            ox, oy, of = o % w.tw, (o // w.tw) % w.th, o // (w.tw * w.th)
            mask[blk, o] = bf * w.tf + of < w.F and by * w.th + oy < w.Hs and bx * w.tw + ox < w.Ws
    return mask


@pytest.mark.parametrize("w", CASES, ids=["bs128-d128", "bs16-d64"])
def test_noalloc_matches_workspace_entry_point(fv, orc, w):
    """Two calls in a row give the same bits as fvattn_sparse_attn on every
    real row (the output does not depend on the schedule, so equality is the
    right test), and agree with the oracle within the attention bar."""
    g = fv.geom_of(w)
    q, k, v, _ = synth.make_qkv(w, device="cuda")
    qt, kt, vt = fv.reorder(g, q), fv.reorder(g, k), fv.reorder(g, v)
    r = fv.route(g, qt, kt, w.p, w.k)
    scale = 1.0 / math.sqrt(w.D)
    ref = fv.sparse_attn(g, qt, kt, vt, r.kv_idx, r.kv_cnt, scale)
    torch.cuda.synchronize()
    assert fv.get_status() == 0
    real_np = _real_rows_mask(w, g)
    real = torch.from_numpy(real_np).cuda()
    ref_rows = ref.view(w.B * w.H, g.nb, g.bs, w.D)
    for _ in range(2):   # two calls in a row share the scratch array
        out = torch.full_like(ref, float("nan"))
        fv.sparse_attn_noalloc(g, qt, kt, vt, r.kv_idx, r.kv_cnt, scale, out=out)
        torch.cuda.synchronize()
        assert fv.get_status() == 0
        got = out.view(w.B * w.H, g.nb, g.bs, w.D)
        assert torch.equal(got[:, real].view(torch.int16), ref_rows[:, real].view(torch.int16))
    items = list(range(w.B * w.H * g.nb))
    want = orc.attention(synth.bf16_bits(qt), synth.bf16_bits(kt), synth.bf16_bits(vt), r.kv_idx.cpu().numpy(),
                         r.kv_cnt.cpu().numpy(), items, w, scale).reshape(w.B * w.H, g.nb, g.bs, w.D)
    err = np.abs(got.float().cpu().numpy() - want)[:, real_np]
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (err.max(), err.mean())


def test_noalloc_rejects_oversized_work_list(fv):
    """A layer whose work list exceeds the built-in scratch is refused with
    FVATTN_ERR_UNSUPPORTED before anything is launched."""
    lib = fv.load()
    g = fv.geom(2, 200, 128, 40, 64, 128, 2, 8, 8)   # 2*200*2560 items: 4 MB of work list
    assert lib.fvattn_attn_workspace_size(ctypes.byref(g)) > fv.NOALLOC_SCRATCH_BYTES
    p = ctypes.c_void_p(256)
    rc = lib.fvattn_sparse_attn_noalloc(ctypes.byref(g), p, p, p, p, p, 0.0883883, p, None, None)
    assert rc == fv.ERR_UNSUPPORTED
