"""Failure path of the attention kernel, exercised without faulting, trapping
or hanging the GPU.

fvattn_test_hook shortens every wait of the kernel to a couple of
milliseconds and makes its V-loading warp leave at once, so the wait of the
PV issuer for V data can never be satisfied.  That wait must run out: the
kernel records FVATTN_ERR_TIMEOUT, every role leaves, the loads and MMAs in
flight complete, the tensor memory is released and the kernel returns.
fvattn_get_status reports the timeout, and the same process then runs a
normal layer with output bits identical to a run before the fault.
"""
import pytest
import torch

from block_sparse_attention_aware_b200 import synth

pytestmark = pytest.mark.gpu

CASES = [
    ("bs128-d128", synth.custom_workload(B=1, H=2, D=128, F=5, Hs=19, Ws=21, tf=2, th=8, tw=8, seed=6, p=0.9, k=3,
                                         qscale="fixed", qscale_values=(1.0, 8.0))),
    ("bs64-d128", synth.custom_workload(B=2, H=2, D=128, F=3, Hs=16, Ws=24, tf=1, th=8, tw=8, seed=7, p=0.95, k=4,
                                        qscale="fixed", qscale_values=(0.5, 4.0))),
]


@pytest.fixture(scope="module")
def fv():
    from block_sparse_attention_aware_b200 import build, fvattn
    build.build()
    assert torch.cuda.is_available(), "needs a GPU"
    fvattn.load()
    return fvattn


@pytest.mark.parametrize("name,w", CASES, ids=[c[0] for c in CASES])
def test_wait_that_runs_out_reports_timeout_and_recovers(fv, name, w):
    g = fv.geom_of(w)
    q, k, v, _ = synth.make_qkv(w, device="cuda")
    layer = fv.Layer(g, w.p, w.k)
    want = layer(q, k, v).clone()
    torch.cuda.synchronize()
    assert fv.get_status() == fv.OK
    fv.test_hook(2_000_000, fv.HOOK_SKIP_V_LOADS)
    try:
        layer.attend(stats=True)
        status = fv.get_status()
    finally:
        fv.test_hook()
    assert status == fv.ERR_TIMEOUT
    assert fv.get_status() == fv.OK   # reading cleared it
    got = layer(q, k, v)
    torch.cuda.synchronize()
    assert fv.get_status() == fv.OK
    assert torch.equal(got.view(torch.int16), want.view(torch.int16))
