"""ctypes binding of libfvattn.so (the C ABI in include/fvattn.h).

Argument marshalling only: every step of the path runs in the library's
CUDA kernels.  torch provides device memory and the current CUDA stream.
There is no CPU fallback: if the library is missing or no CUDA device is
present, the calls raise.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass
from typing import List, Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfvattn.so")
_lib = None

OK, ERR_INVALID, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_BOUNDS = range(6)
EXPORTED = ("fvattn_geom_init", "fvattn_block_order", "fvattn_copy_heads", "fvattn_reorder", "fvattn_inverse_reorder",
            "fvattn_route_workspace_size", "fvattn_route_kernel_launches", "fvattn_route", "fvattn_route_aug",
            "fvattn_reorder_route",
            "fvattn_attn_workspace_size",
            "fvattn_num_sms", "fvattn_sparse_attn", "fvattn_sparse_attn_raster", "fvattn_sparse_attn_noalloc",
            "fvattn_get_status",
            "fvattn_status_string", "fvattn_test_hook")


class FVAttnError(RuntimeError):
    def __init__(self, what: str, code: int):
        super().__init__(f"{what}: {status_string(code)} (code {code})")
        self.code = code


class Geom(ctypes.Structure):
    """Mirror of fvattn_geom."""
    _fields_ = [(n, ctypes.c_int) for n in
                ("B", "H", "D", "F", "Hs", "Ws", "tf", "th", "tw",
                 "Fp", "Hp", "Wp", "nbf", "nby", "nbx", "bs", "nb")] + \
               [("N", ctypes.c_longlong), ("Npad", ctypes.c_longlong), ("order", ctypes.c_void_p)]


def load(path: str = LIB_PATH):
    """Load libfvattn.so and declare its signatures (raises if missing)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libfvattn.so not built at {path}; run "
                           "`python -m block_sparse_attention_aware_b200.build`")
    L = ctypes.CDLL(path)
    P, I, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    G = ctypes.POINTER(Geom)
    L.fvattn_geom_init.argtypes = [G]
    L.fvattn_geom_init.restype = I
    L.fvattn_block_order.argtypes = [G, P, P]
    L.fvattn_block_order.restype = I
    L.fvattn_copy_heads.argtypes = [G, I, I, P, P, I, P]
    L.fvattn_copy_heads.restype = I
    L.fvattn_reorder.argtypes = [G, P, P, P]
    L.fvattn_reorder.restype = I
    L.fvattn_inverse_reorder.argtypes = [G, P, P, P]
    L.fvattn_inverse_reorder.restype = I
    L.fvattn_route_workspace_size.argtypes = [G]
    L.fvattn_route_workspace_size.restype = S
    L.fvattn_route_kernel_launches.argtypes = [G]
    L.fvattn_route_kernel_launches.restype = I
    L.fvattn_route.argtypes = [G, P, P, ctypes.c_double, I, ctypes.c_float, P, P, P, P, P, P, S, P]
    L.fvattn_route.restype = I
    L.fvattn_route_aug.argtypes = [G, P, P, ctypes.c_double, I, I, ctypes.c_float, P, P, P, P, P, P, S, P]
    L.fvattn_route_aug.restype = I
    L.fvattn_reorder_route.argtypes = [G, P, P, P, P, ctypes.c_double, I, I, ctypes.c_float, P, P, P, P, P, P, S,
                                       P]
    L.fvattn_reorder_route.restype = I
    L.fvattn_attn_workspace_size.argtypes = [G]
    L.fvattn_attn_workspace_size.restype = S
    L.fvattn_num_sms.argtypes = []
    L.fvattn_num_sms.restype = I
    L.fvattn_sparse_attn.argtypes = [G, P, P, P, P, P, ctypes.c_float, P, P, P, S, P]
    L.fvattn_sparse_attn.restype = I
    L.fvattn_sparse_attn_raster.argtypes = [G, P, P, P, P, P, ctypes.c_float, P, P, P, S, P]
    L.fvattn_sparse_attn_raster.restype = I
    L.fvattn_sparse_attn_noalloc.argtypes = [G, P, P, P, P, P, ctypes.c_float, P, P, P]
    L.fvattn_sparse_attn_noalloc.restype = I
    L.fvattn_get_status.argtypes = [P]
    L.fvattn_get_status.restype = I
    L.fvattn_status_string.argtypes = [I]
    L.fvattn_status_string.restype = ctypes.c_char_p
    L.fvattn_test_hook.argtypes = [ctypes.c_ulonglong, I]
    L.fvattn_test_hook.restype = I
    _lib = L
    return L


def status_string(code: int) -> str:
    return load().fvattn_status_string(int(code)).decode()


def _check(what: str, rc: int):
    if rc != OK:
        raise FVAttnError(what, rc)


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t: Optional[torch.Tensor]):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _need_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


def _expect(name: str, t: Optional[torch.Tensor], shape, dtype):
    """The kernels read and write dense buffers of exactly this shape."""
    if t is None:
        return
    if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous() or not t.is_cuda:
        raise ValueError(f"{name}: expected a contiguous CUDA {dtype} tensor of shape {tuple(shape)}, "
                         f"got {t.dtype} {tuple(t.shape)} (contiguous={t.is_contiguous()}, cuda={t.is_cuda})")


def _raster(g: Geom):
    return (g.B, g.N, g.H, g.D)


def _tiled(g: Geom):
    return (g.B, g.H, g.Npad, g.D)


def _expect_attn(g: Geom, qt, kt, vt, kv_idx, kv_cnt, out, out_shape, sm_stats):
    for name, t in (("qt", qt), ("kt", kt), ("vt", vt)):
        if t is None:
            raise ValueError(f"{name} is required")
        _expect(name, t, _tiled(g), torch.bfloat16)
    _expect("kv_idx", kv_idx, (g.B, g.H, g.nb, g.nb), torch.int32)
    _expect("kv_cnt", kv_cnt, (g.B, g.H, g.nb), torch.int32)
    _expect("out", out, out_shape, torch.bfloat16)
    if sm_stats is not None:
        _need_cuda(sm_stats)
        if sm_stats.dtype != torch.int64 or sm_stats.numel() < 2 * num_sms():
            raise ValueError(f"sm_stats: expected int64 with at least {2 * num_sms()} elements")


def _expect_routed(g: Geom, out: "RouteOut"):
    _expect("kv_idx", out.kv_idx, (g.B, g.H, g.nb, g.nb), torch.int32)
    _expect("kv_cnt", out.kv_cnt, (g.B, g.H, g.nb), torch.int32)
    _expect("q_pool", out.q_pool, (g.B, g.H, g.nb, g.D), torch.float32)
    _expect("k_pool", out.k_pool, (g.B, g.H, g.nb, g.D), torch.float32)
    _expect("logits", out.logits, (g.B, g.H, g.nb, g.nb), torch.float32)


def geom(B, H, D, F, Hs, Ws, tf, th, tw) -> Geom:
    g = Geom(B=B, H=H, D=D, F=F, Hs=Hs, Ws=Ws, tf=tf, th=th, tw=tw)
    _check("fvattn_geom_init", load().fvattn_geom_init(ctypes.byref(g)))
    return g


def geom_of(w) -> Geom:
    """Geometry of a synth.Workload."""
    return geom(w.B, w.H, w.D, w.F, w.Hs, w.Ws, w.tf, w.th, w.tw)


def block_order(g: Geom, device="cuda", stream=None) -> torch.Tensor:
    """fvattn_block_order: the Hilbert block-order table (int32 [2*nb]) of a
    geometry.  Put it in a geometry with with_order(g, table)."""
    table = torch.empty(2 * g.nb, dtype=torch.int32, device=device)
    _check("fvattn_block_order", load().fvattn_block_order(ctypes.byref(g), _ptr(table), _stream(stream)))
    return table


def with_order(g: Geom, table: Optional[torch.Tensor]) -> Geom:
    """A copy of g that numbers blocks by `table` (None: raster tile order).
    The table must stay alive while the geometry is used."""
    g2 = Geom.from_buffer_copy(g)
    g2.order = None if table is None else table.data_ptr()
    return g2


def route_kernel_launches(g: Geom) -> int:
    """Kernel launches one fvattn_route call makes for this geometry."""
    return load().fvattn_route_kernel_launches(ctypes.byref(g))


def num_sms() -> int:
    return load().fvattn_num_sms()


def tiled_empty(g: Geom, device="cuda") -> torch.Tensor:
    return torch.empty((g.B, g.H, g.Npad, g.D), dtype=torch.bfloat16, device=device)


def reorder(g: Geom, x: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None):
    """fvattn_reorder: raster [B, N, H, D] bf16 -> tiled [B, H, Npad, D]."""
    _expect("x", x, _raster(g), torch.bfloat16)
    _expect("out", out, _tiled(g), torch.bfloat16)
    if out is None:
        out = tiled_empty(g, x.device)
    _check("fvattn_reorder", load().fvattn_reorder(ctypes.byref(g), _ptr(x), _ptr(out), _stream(stream)))
    return out


def inverse_reorder(g: Geom, ot: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None):
    """fvattn_inverse_reorder: tiled [B, H, Npad, D] -> raster [B, N, H, D]."""
    _expect("ot", ot, _tiled(g), torch.bfloat16)
    _expect("out", out, _raster(g), torch.bfloat16)
    if out is None:
        out = torch.empty((g.B, g.N, g.H, g.D), dtype=torch.bfloat16, device=ot.device)
    _check("fvattn_inverse_reorder",
           load().fvattn_inverse_reorder(ctypes.byref(g), _ptr(ot), _ptr(out), _stream(stream)))
    return out


@dataclass
class RouteOut:
    kv_idx: torch.Tensor
    kv_cnt: torch.Tensor
    q_pool: Optional[torch.Tensor] = None
    k_pool: Optional[torch.Tensor] = None
    logits: Optional[torch.Tensor] = None


def route_workspace(g: Geom, device="cuda") -> torch.Tensor:
    n = load().fvattn_route_workspace_size(ctypes.byref(g))
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device)


def attn_workspace(g: Geom, device="cuda") -> torch.Tensor:
    n = load().fvattn_attn_workspace_size(ctypes.byref(g))
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device)


def _route_out(g: Geom, dev, debug: bool) -> RouteOut:
    out = RouteOut(kv_idx=torch.empty((g.B, g.H, g.nb, g.nb), dtype=torch.int32, device=dev),
                   kv_cnt=torch.empty((g.B, g.H, g.nb), dtype=torch.int32, device=dev))
    if debug:
        out.q_pool = torch.empty((g.B, g.H, g.nb, g.D), dtype=torch.float32, device=dev)
        out.k_pool = torch.empty_like(out.q_pool)
        out.logits = torch.empty((g.B, g.H, g.nb, g.nb), dtype=torch.float32, device=dev)
    return out


def route(g: Geom, qt: torch.Tensor, kt: torch.Tensor, p: float, k: int,
          scale: Optional[float] = None, debug: bool = False, out: Optional[RouteOut] = None,
          workspace: Optional[torch.Tensor] = None, stream=None, k_extra: int = 0) -> RouteOut:
    """fvattn_route: pooled block scores -> Top-p (+ Top-k floor) kv lists.
    p = 0 (fixed Top-k mode) or k_extra > 0 (augmentation) go through
    fvattn_route_aug."""
    _expect("qt", qt, _tiled(g), torch.bfloat16)
    _expect("kt", kt, _tiled(g), torch.bfloat16)
    dev = qt.device
    if scale is None:
        scale = 1.0 / math.sqrt(g.D)
    if out is None:
        out = _route_out(g, dev, debug)
    _expect_routed(g, out)
    if workspace is None:
        workspace = route_workspace(g, dev)
    _need_cuda(workspace)
    if k_extra or p == 0:
        rc = load().fvattn_route_aug(ctypes.byref(g), _ptr(qt), _ptr(kt), float(p), int(k), int(k_extra),
                                     float(scale), _ptr(out.kv_idx), _ptr(out.kv_cnt), _ptr(out.q_pool),
                                     _ptr(out.k_pool), _ptr(out.logits), _ptr(workspace),
                                     0 if workspace is None else workspace.numel(), _stream(stream))
        _check("fvattn_route_aug", rc)
    else:
        rc = load().fvattn_route(ctypes.byref(g), _ptr(qt), _ptr(kt), float(p), int(k), float(scale),
                                 _ptr(out.kv_idx), _ptr(out.kv_cnt), _ptr(out.q_pool), _ptr(out.k_pool),
                                 _ptr(out.logits), _ptr(workspace),
                                 0 if workspace is None else workspace.numel(), _stream(stream))
        _check("fvattn_route", rc)
    return out


def reorder_route(g: Geom, q: torch.Tensor, k: torch.Tensor, p: float, kf: int,
                  scale: Optional[float] = None, debug: bool = False, out: Optional[RouteOut] = None,
                  qt: Optional[torch.Tensor] = None, kt: Optional[torch.Tensor] = None,
                  workspace: Optional[torch.Tensor] = None, stream=None, k_extra: int = 0):
    """fvattn_reorder_route: raster Q, K -> their tiles and the kv lists in
    one pass over Q and K.  Returns (qt, kt, RouteOut)."""
    _expect("q", q, _raster(g), torch.bfloat16)
    _expect("k", k, _raster(g), torch.bfloat16)
    dev = q.device
    if scale is None:
        scale = 1.0 / math.sqrt(g.D)
    if out is None:
        out = _route_out(g, dev, debug)
    _expect_routed(g, out)
    qt = tiled_empty(g, dev) if qt is None else qt
    kt = tiled_empty(g, dev) if kt is None else kt
    _expect("qt", qt, _tiled(g), torch.bfloat16)
    _expect("kt", kt, _tiled(g), torch.bfloat16)
    if qt.data_ptr() == kt.data_ptr():
        raise ValueError("qt and kt must be distinct buffers")
    if workspace is None:
        workspace = route_workspace(g, dev)
    _need_cuda(workspace)
    rc = load().fvattn_reorder_route(ctypes.byref(g), _ptr(q), _ptr(k), _ptr(qt), _ptr(kt), float(p), int(kf),
                                     int(k_extra), float(scale), _ptr(out.kv_idx), _ptr(out.kv_cnt),
                                     _ptr(out.q_pool), _ptr(out.k_pool), _ptr(out.logits), _ptr(workspace),
                                     workspace.numel(), _stream(stream))
    _check("fvattn_reorder_route", rc)
    return qt, kt, out


def sparse_attn(g: Geom, qt, kt, vt, kv_idx, kv_cnt, scale: Optional[float] = None,
                out: Optional[torch.Tensor] = None, sm_stats: Optional[torch.Tensor] = None,
                workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """fvattn_sparse_attn: block-sparse attention on the kept blocks -> tiled O."""
    _expect_attn(g, qt, kt, vt, kv_idx, kv_cnt, out, _tiled(g), sm_stats)
    if scale is None:
        scale = 1.0 / math.sqrt(g.D)
    if out is None:
        out = tiled_empty(g, qt.device)
    if workspace is None:
        workspace = attn_workspace(g, qt.device)
    _need_cuda(workspace)
    rc = load().fvattn_sparse_attn(ctypes.byref(g), _ptr(qt), _ptr(kt), _ptr(vt), _ptr(kv_idx),
                                   _ptr(kv_cnt), float(scale), _ptr(out), _ptr(sm_stats),
                                   _ptr(workspace), workspace.numel(), _stream(stream))
    _check("fvattn_sparse_attn", rc)
    return out


# Scratch bytes available to sparse_attn_noalloc (FVATTN_NOALLOC_SCRATCH_BYTES).
NOALLOC_SCRATCH_BYTES = 2 * 1024 * 1024



def sparse_attn_raster(g: Geom, qt, kt, vt, kv_idx, kv_cnt, scale: Optional[float] = None,
                       out: Optional[torch.Tensor] = None, sm_stats: Optional[torch.Tensor] = None,
                       workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """fvattn_sparse_attn_raster: sparse attention writing O in the raster
    [B, N, H, D] layout (the inverse reorder fused into the epilogue)."""
    _expect_attn(g, qt, kt, vt, kv_idx, kv_cnt, out, _raster(g), sm_stats)
    if scale is None:
        scale = 1.0 / math.sqrt(g.D)
    if out is None:
        out = torch.empty(_raster(g), dtype=torch.bfloat16, device=qt.device)
    if workspace is None:
        workspace = attn_workspace(g, qt.device)
    _need_cuda(workspace)
    rc = load().fvattn_sparse_attn_raster(ctypes.byref(g), _ptr(qt), _ptr(kt), _ptr(vt), _ptr(kv_idx),
                                          _ptr(kv_cnt), float(scale), _ptr(out), _ptr(sm_stats),
                                          _ptr(workspace), workspace.numel(), _stream(stream))
    _check("fvattn_sparse_attn_raster", rc)
    return out

def sparse_attn_noalloc(g: Geom, qt, kt, vt, kv_idx, kv_cnt, scale: Optional[float] = None,
                        out: Optional[torch.Tensor] = None, sm_stats: Optional[torch.Tensor] = None,
                        stream=None) -> torch.Tensor:
    """fvattn_sparse_attn_noalloc: the same attention with the library's own
    scratch array instead of a caller workspace (for callers that cannot
    allocate device memory).  Calls that overlap on the GPU share that
    scratch and must be serialised by the caller."""
    _expect_attn(g, qt, kt, vt, kv_idx, kv_cnt, out, _tiled(g), sm_stats)
    if scale is None:
        scale = 1.0 / math.sqrt(g.D)
    if out is None:
        out = tiled_empty(g, qt.device)
    rc = load().fvattn_sparse_attn_noalloc(ctypes.byref(g), _ptr(qt), _ptr(kt), _ptr(vt), _ptr(kv_idx),
                                           _ptr(kv_cnt), float(scale), _ptr(out), _ptr(sm_stats),
                                           _stream(stream))
    _check("fvattn_sparse_attn_noalloc", rc)
    return out


HOOK_SKIP_V_LOADS = 1   # FVATTN_HOOK_SKIP_V_LOADS


def test_hook(wait_limit_ns: int = 0, flags: int = 0) -> None:
    """fvattn_test_hook: fault injection for failure-path tests (a shorter
    wait limit; FVATTN_HOOK_SKIP_V_LOADS).  test_hook() restores normal
    operation."""
    _check("fvattn_test_hook", load().fvattn_test_hook(int(wait_limit_ns), int(flags)))


def get_status(stream=None) -> int:
    """Synchronise the stream and read/clear the device status word."""
    return load().fvattn_get_status(_stream(stream))


class Layer:
    """One attention layer's buffers, allocated once and reused: the four C
    ABI calls in order (reorder Q, K, V -> route -> sparse attention ->
    inverse reorder).  With fused_route (the default) the reorder of Q and K
    and the routing are one call, fvattn_reorder_route, which reads Q and K
    once; the results are the same bits as the separate calls."""

    def __init__(self, g: Geom, p: float, k: int, scale: Optional[float] = None, device="cuda",
                 debug: bool = False, order: str = "raster", fused_route: bool = True):
        if order not in ("raster", "hilbert"):
            raise ValueError(f"block order {order!r}")
        self.order_table = block_order(g, device) if order == "hilbert" else None
        g = with_order(g, self.order_table)
        self.g, self.p, self.k = g, p, k
        self.fused_route = fused_route
        self.scale = 1.0 / math.sqrt(g.D) if scale is None else scale
        self.qt = tiled_empty(g, device)
        self.kt = tiled_empty(g, device)
        self.vt = tiled_empty(g, device)
        self.ot = tiled_empty(g, device)
        self.o = torch.empty((g.B, g.N, g.H, g.D), dtype=torch.bfloat16, device=device)
        self.routed = RouteOut(kv_idx=torch.empty((g.B, g.H, g.nb, g.nb), dtype=torch.int32, device=device),
                               kv_cnt=torch.empty((g.B, g.H, g.nb), dtype=torch.int32, device=device))
        if debug:
            self.routed.logits = torch.empty((g.B, g.H, g.nb, g.nb), dtype=torch.float32, device=device)
        self.route_ws = route_workspace(g, device)
        self.attn_ws = attn_workspace(g, device)
        self.sm_stats = torch.zeros(2 * num_sms(), dtype=torch.int64, device=device)

    def reorder_qkv(self, q, k, v, stream=None):
        reorder(self.g, q, self.qt, stream)
        reorder(self.g, k, self.kt, stream)
        reorder(self.g, v, self.vt, stream)

    def route(self, stream=None):
        return route(self.g, self.qt, self.kt, self.p, self.k, self.scale, out=self.routed,
                     workspace=self.route_ws, stream=stream)

    def reorder_route(self, q, k, stream=None):
        """Q and K reordered and routed in one pass (fvattn_reorder_route)."""
        reorder_route(self.g, q, k, self.p, self.k, self.scale, out=self.routed, qt=self.qt, kt=self.kt,
                      workspace=self.route_ws, stream=stream)
        return self.routed

    def reorder_v(self, v, stream=None):
        reorder(self.g, v, self.vt, stream)

    def route_qk(self, q, k, stream=None):
        """Q and K to tiles and kv lists: the fused call, or two reorders and
        routing (same bits)."""
        if self.fused_route:
            return self.reorder_route(q, k, stream)
        reorder(self.g, q, self.qt, stream)
        reorder(self.g, k, self.kt, stream)
        return self.route(stream)

    def kernel_launches(self) -> int:
        """Kernels one __call__ (unfused inverse) launches: reorders, routing,
        the work list (plus the query groups' union lists for bs < 128),
        attention, inverse reorder."""
        reorders = 1 if self.fused_route else 3
        worklist = 2 + (1 if self.g.bs < 128 else 0)
        return reorders + route_kernel_launches(self.g) + worklist + 1 + 1

    def attend(self, stats: bool = False, stream=None):
        return sparse_attn(self.g, self.qt, self.kt, self.vt, self.routed.kv_idx, self.routed.kv_cnt,
                           self.scale, out=self.ot, sm_stats=self.sm_stats if stats else None,
                           workspace=self.attn_ws, stream=stream)

    def restore(self, stream=None):
        return inverse_reorder(self.g, self.ot, self.o, stream)

    def attend_raster(self, stats: bool = False, stream=None):
        """Sparse attention with the inverse reorder fused in: O straight to self.o."""
        return sparse_attn_raster(self.g, self.qt, self.kt, self.vt, self.routed.kv_idx, self.routed.kv_cnt,
                                  self.scale, out=self.o, sm_stats=self.sm_stats if stats else None,
                                  workspace=self.attn_ws, stream=stream)

    def __call__(self, q, k, v, stats: bool = False, stream=None, fused_inverse: bool = False):
        self.route_qk(q, k, stream)
        self.reorder_v(v, stream)
        if fused_inverse:
            return self.attend_raster(stats, stream)
        self.attend(stats, stream)
        return self.restore(stream)


def default_head_group_sizes(H: int) -> List[int]:
    """Head-group sizes for HostPipeline: two heads a group, except the first
    and the last group, which hold one head each.  Before the first group's
    routing can start, its Q and K must be uploaded. After the last group's
    compute, its output must be downloaded.  Neither overlaps any compute,
    so both groups are kept small.  For 40 heads: 1, 2 x 19, 1 (21 groups)."""
    if H < 1:
        raise ValueError(f"{H} heads")
    if H <= 2:
        return [1] * H
    m = (H - 2) // 2
    return [1] + [2] * m + [1] * (H - 1 - 2 * m)


class HostPipeline:
    """End to end from page-locked host buffers, pipelined by head groups.

    Heads are independent through every step, so the layer is run as head
    slices: the upload of slice i+1 (one copy stream), the library calls on
    slice i (the compute stream) and the download of slice i-1 (another copy
    stream) overlap.  Within a slice, Q and K are uploaded first and routed
    while V is still on its way.  `groups` is None (default_head_group_sizes),
    a number of equal groups, or a list of group sizes in heads.  Slices of
    one size rotate over two sets of device buffers.  The output equals one
    whole-layer call bit for bit."""

    def __init__(self, g: Geom, p: float, k: int, groups=None, device="cuda",
                 order: str = "raster", fused_route: bool = True):
        if groups is None:
            sizes = default_head_group_sizes(g.H)
        elif isinstance(groups, int):
            if groups < 1 or g.H % groups:
                raise ValueError(f"{g.H} heads do not split into {groups} equal groups")
            sizes = [g.H // groups] * groups
        else:
            sizes = [int(x) for x in groups]
            if not sizes or min(sizes) < 1 or sum(sizes) != g.H:
                raise ValueError(f"group sizes {sizes} do not partition {g.H} heads")
        self.g, self.sizes, self.groups = g, sizes, len(sizes)
        # per group size: one or two (Layer, device Q/K/V slices) buffer sets
        self.sets = {}
        for nh in sorted(set(sizes)):
            gs = geom(g.B, nh, g.D, g.F, g.Hs, g.Ws, g.tf, g.th, g.tw)
            shape = (g.B, g.N, nh, g.D)
            self.sets[nh] = [(Layer(gs, p, k, device=device, order=order, fused_route=fused_route),
                              [torch.empty(shape, dtype=torch.bfloat16, device=device) for _ in range(3)])
                             for _ in range(min(2, sizes.count(nh)))]
        self.up = torch.cuda.Stream(device=device)
        self.down = torch.cuda.Stream(device=device)

    def __call__(self, q_host, k_host, v_host, o_host, stream=None):
        L = load()
        s = stream if stream is not None else torch.cuda.current_stream()
        g = self.g
        start = torch.cuda.Event()
        start.record(s)
        self.up.wait_event(start)
        self.down.wait_event(start)
        freed = {}        # buffer set -> download of the slice that last used it
        seen = {}         # group size -> slices of that size so far
        done = None
        h0 = 0
        for nh in self.sizes:
            sets = self.sets[nh]
            b = (nh, seen.get(nh, 0) % len(sets))
            seen[nh] = seen.get(nh, 0) + 1
            lay, (qd, kd, vd) = sets[b[1]]
            if b in freed:
                self.up.wait_event(freed[b])
            uploaded = []
            for pair in (((q_host, qd), (k_host, kd)), ((v_host, vd),)):
                for src, dst in pair:
                    _check("fvattn_copy_heads", L.fvattn_copy_heads(ctypes.byref(g), h0, nh,
                                                                    ctypes.c_void_p(src.data_ptr()), _ptr(dst), 1,
                                                                    _stream(self.up)))
                uploaded.append(torch.cuda.Event())
                uploaded[-1].record(self.up)
            s.wait_event(uploaded[0])
            lay.route_qk(qd, kd, stream=s)
            s.wait_event(uploaded[1])
            lay.reorder_v(vd, stream=s)
            lay.attend(stream=s)
            out = lay.restore(stream=s)
            computed = torch.cuda.Event()
            computed.record(s)
            self.down.wait_event(computed)
            _check("fvattn_copy_heads", L.fvattn_copy_heads(ctypes.byref(g), h0, nh, _ptr(out),
                                                            ctypes.c_void_p(o_host.data_ptr()), 0,
                                                            _stream(self.down)))
            done = torch.cuda.Event()
            done.record(self.down)
            freed[b] = done
            h0 += nh
        s.wait_event(done)
        return o_host


def attention_from_host(layer: Layer, q_host, k_host, v_host, o_host, stream=None):
    """End to end from pinned host buffers: H2D copies of raster Q, K, V, the
    layer's library calls, and a D2H copy of the raster output, all on one
    stream (HostPipeline overlaps them instead)."""
    s = stream if stream is not None else torch.cuda.current_stream()
    with torch.cuda.stream(s):
        qd = torch.empty_like(q_host, device="cuda")
        kd = torch.empty_like(k_host, device="cuda")
        vd = torch.empty_like(v_host, device="cuda")
        qd.copy_(q_host, non_blocking=True)
        kd.copy_(k_host, non_blocking=True)
        vd.copy_(v_host, non_blocking=True)
        out = layer(qd, kd, vd, stream=s)
        o_host.copy_(out, non_blocking=True)
    return o_host
