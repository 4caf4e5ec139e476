"""Python face of the FVAttn CPU oracle -- TEST INFRASTRUCTURE ONLY.

Loads `liboracle.so` (built from fvattn_oracle.c by `build_oracle`) with
ctypes and exposes numpy-level helpers.  Only the test-suite, the smoke
check and the benchmark's CPU-baseline leg use this module; the product
path never imports it.  It shares no code with the CUDA path.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import time

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fvattn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

# Rows whose cumulative mass lands within this distance of p are "near ties":
# only there may the GPU's kept set differ from the oracle's.
TIE_BAND = 1e-5


def build_oracle(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, strict IEEE: no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared",
                               "-fno-fast-math", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build_oracle()
        L = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I = ctypes.c_int
        Dd = ctypes.c_double
        geo = [I] * 9
        L.oracle_geometry.argtypes = geo + [P]
        L.oracle_block_valid_counts.argtypes = [I] * 7 + [P]
        L.oracle_block_order.argtypes = [I, I, I, P]
        L.oracle_reorder.argtypes = [P, P] + geo + [I]
        L.oracle_inverse_reorder.argtypes = [P, P] + geo + [I]
        L.oracle_pool.argtypes = [P, P] + geo + [I]
        L.oracle_logits.argtypes = [P, P, P, I, I, I, Dd]
        L.oracle_select.argtypes = [P, I, I, Dd, I, Dd, P, P, P, P]
        L.oracle_select_aug.argtypes = [P, I, I, Dd, I, I, Dd, P, P, P, P]
        L.oracle_attention.argtypes = [P, P, P, P, P, P, I, Dd, P] + geo + [I]
        L.oracle_num_threads.restype = I
        L.oracle_set_num_threads.argtypes = [I]
        _lib = L
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _geo(w):
    return (w.B, w.H, w.D, w.F, w.Hs, w.Ws, w.tf, w.th, w.tw)


def _order(w) -> int:
    """Block order of a workload: 0 raster tile order, 1 Hilbert."""
    order = getattr(w, "order", "raster")
    assert order in ("raster", "hilbert"), order
    return 1 if order == "hilbert" else 0


def block_order(nbf: int, nby: int, nbx: int) -> np.ndarray:
    """Hilbert block order of a tile grid: tile_of_block[nb], raster tile
    index (frame-major, then row, then col) of each block."""
    out = np.empty(nbf * nby * nbx, dtype=np.int32)
    lib().oracle_block_order(int(nbf), int(nby), int(nbx), _ptr(out))
    return out


def num_threads() -> int:
    return lib().oracle_num_threads()


def set_num_threads(n: int) -> None:
    lib().oracle_set_num_threads(int(n))


def geometry(w) -> dict:
    out = np.zeros(10, dtype=np.int64)
    lib().oracle_geometry(*_geo(w), _ptr(out))
    keys = ["Fp", "Hp", "Wp", "nbf", "nby", "nbx", "bs", "nb", "N", "Npad"]
    return {k: int(v) for k, v in zip(keys, out)}


def block_valid_counts(w) -> np.ndarray:
    g = geometry(w)
    out = np.zeros(g["nb"], dtype=np.int32)
    lib().oracle_block_valid_counts(w.F, w.Hs, w.Ws, w.tf, w.th, w.tw, _order(w), _ptr(out))
    return out


def reorder(x_bits: np.ndarray, w) -> np.ndarray:
    """Raster [B, N, H, D] 16-bit patterns -> tiled [B, H, Npad, D]."""
    g = geometry(w)
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    assert x.shape == (w.B, g["N"], w.H, w.D)
    out = np.empty((w.B, w.H, g["Npad"], w.D), dtype=np.uint16)
    lib().oracle_reorder(_ptr(x), _ptr(out), *_geo(w), _order(w))
    return out


def inverse_reorder(t_bits: np.ndarray, w) -> np.ndarray:
    """Tiled [B, H, Npad, D] -> raster [B, N, H, D] (padding dropped)."""
    g = geometry(w)
    t = np.ascontiguousarray(t_bits, dtype=np.uint16)
    assert t.shape == (w.B, w.H, g["Npad"], w.D)
    out = np.empty((w.B, g["N"], w.H, w.D), dtype=np.uint16)
    lib().oracle_inverse_reorder(_ptr(t), _ptr(out), *_geo(w), _order(w))
    return out


def pool(t_bits: np.ndarray, w) -> np.ndarray:
    """Mean of each block's real tokens: [B, H, nb, D] float64."""
    g = geometry(w)
    t = np.ascontiguousarray(t_bits, dtype=np.uint16)
    out = np.empty((w.B, w.H, g["nb"], w.D), dtype=np.float64)
    lib().oracle_pool(_ptr(t), _ptr(out), *_geo(w), _order(w))
    return out


def logits(qp: np.ndarray, kp: np.ndarray, scale: float) -> np.ndarray:
    """Block scores scale * Qp Kp^T per (b, h): [..., nb, nb] float64."""
    qp = np.ascontiguousarray(qp, dtype=np.float64)
    kp = np.ascontiguousarray(kp, dtype=np.float64)
    nb, D = qp.shape[-2], qp.shape[-1]
    BH = int(np.prod(qp.shape[:-2])) if qp.ndim > 2 else 1
    out = np.empty(qp.shape[:-1] + (nb,), dtype=np.float64)
    lib().oracle_logits(_ptr(qp), _ptr(kp), _ptr(out), BH, nb, D, float(scale))
    return out


def select(L: np.ndarray, p: float, k: int, tie_band: float = TIE_BAND, k_extra: int = 0):
    """Top-p with Top-k floor on fp32 logits [..., nb]; p = 0 is the fixed
    Top-k mode and k_extra appends that many further blocks of the order.

    Returns (idx, cnt, m_p, near_tie): idx [..., nb] int32 with the kept
    block ids ascending in the first cnt entries and -1 after them.
    """
    L32 = np.ascontiguousarray(L, dtype=np.float32)
    nb = L32.shape[-1]
    rows = int(np.prod(L32.shape[:-1])) if L32.ndim > 1 else 1
    idx = np.empty(L32.shape, dtype=np.int32)
    cnt = np.empty(L32.shape[:-1], dtype=np.int32)
    mp = np.empty(L32.shape[:-1], dtype=np.int32)
    tie = np.empty(L32.shape[:-1], dtype=np.int32)
    if k_extra:
        lib().oracle_select_aug(_ptr(L32), rows, nb, float(p), int(k), int(k_extra), float(tie_band),
                                _ptr(idx), _ptr(cnt), _ptr(mp), _ptr(tie))
    else:
        lib().oracle_select(_ptr(L32), rows, nb, float(p), int(k), float(tie_band),
                            _ptr(idx), _ptr(cnt), _ptr(mp), _ptr(tie))
    return idx, cnt, mp, tie


def attention(qt_bits, kt_bits, vt_bits, kv_idx, kv_cnt, items, w, scale: float):
    """Masked attention for flat items (b*H + h)*nb + i: [n_items, bs, D] float64.

    kv_idx: [B, H, nb, nb] int32 (first cnt entries used); kv_cnt: [B, H, nb].
    """
    g = geometry(w)
    qt = np.ascontiguousarray(qt_bits, dtype=np.uint16)
    kt = np.ascontiguousarray(kt_bits, dtype=np.uint16)
    vt = np.ascontiguousarray(vt_bits, dtype=np.uint16)
    idx = np.ascontiguousarray(kv_idx, dtype=np.int32).reshape(-1, g["nb"])
    cnt = np.ascontiguousarray(kv_cnt, dtype=np.int32).reshape(-1)
    it = np.ascontiguousarray(np.asarray(items, dtype=np.int64))
    out = np.empty((len(it), g["bs"], w.D), dtype=np.float64)
    lib().oracle_attention(_ptr(qt), _ptr(kt), _ptr(vt), _ptr(idx), _ptr(cnt), _ptr(it),
                           len(it), float(scale), _ptr(out), *_geo(w), _order(w))
    return out


def route(qt_bits, kt_bits, w, p: float, k: int, scale: float):
    """Pool, score and select end to end: (qp, kp, L64, idx, cnt, mp, tie)."""
    qp = pool(qt_bits, w)
    kp = pool(kt_bits, w)
    L = logits(qp, kp, scale)
    idx, cnt, mp, tie = select(L.astype(np.float32), p, k)
    return qp, kp, L, idx, cnt, mp, tie


def timed(fn, *a, **kw):
    t0 = time.perf_counter()
    r = fn(*a, **kw)
    return r, time.perf_counter() - t0
