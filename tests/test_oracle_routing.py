"""Pins for the oracle's routing: block mean-pooling, block scores, and
Top-p selection with a Top-k floor.

FVAttn pages, paperlayer.ai summary: section 2 "Background and Related
Work" (Top-p keeps the smallest set of key blocks whose cumulative
importance reaches p; the Top-k safety floor keeps a minimum budget) and
section 3 "FVAttn Design", item "Sparse-routing frontend" (Top-p CDF
thresholding of each query block's similarity distribution).
"""
import itertools
import math
import os

import numpy as np
import pytest

from block_sparse_attention_aware_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16_bits_of(values: np.ndarray) -> np.ndarray:
    """bf16 bit patterns of float32 values that are exactly representable."""
    f = np.ascontiguousarray(values, dtype=np.float32)
    bits = f.view(np.uint32)
    assert np.all(bits & 0xFFFF == 0), "value not exactly representable in bf16"
    return (bits >> 16).astype(np.uint16)


# ---------------------------------------------------------------- pooling

def test_pool_constant(orc):
    w = synth.custom_workload(B=1, H=2, D=8, F=3, Hs=5, Ws=7, tf=2, th=2, tw=4)
    x = np.full((w.B, w.N, w.H, w.D), 1.5, dtype=np.float32)
    t = orc.reorder(_bf16_bits_of(x), w)
    qp = orc.pool(t, w)
    assert np.all(qp == 1.5)


def test_pool_frame_ramp_closed_form(orc):
    """Value = frame index.  A tile over frames {2a, 2a+1} has mean 2a + 0.5;
    the last tile of a 5-frame video holds frame 4 only and has mean 4."""
    w = synth.custom_workload(B=1, H=1, D=4, F=5, Hs=3, Ws=6, tf=2, th=2, tw=4)
    f = np.repeat(np.arange(w.F), w.Hs * w.Ws).astype(np.float32)
    x = np.broadcast_to(f[None, :, None, None], (1, w.N, 1, w.D)).copy()
    qp = orc.pool(orc.reorder(_bf16_bits_of(x), w), w)[0, 0]
    geo = orc.geometry(w)
    per_frame_tile = geo["nby"] * geo["nbx"]
    for blk in range(geo["nb"]):
        a = blk // per_frame_tile
        want = 4.0 if a == 2 else 2 * a + 0.5
        assert np.all(qp[blk] == want)


def test_pool_partial_tiles_use_real_token_count(orc):
    """Value = column index x; the last column tile of a 7-wide video holds
    x in {4, 5, 6} only, so its mean is 5 (padding is not averaged in)."""
    w = synth.custom_workload(B=1, H=1, D=4, F=2, Hs=2, Ws=7, tf=2, th=2, tw=4)
    xs = np.tile(np.arange(w.Ws), w.F * w.Hs).astype(np.float32)
    x = np.broadcast_to(xs[None, :, None, None], (1, w.N, 1, w.D)).copy()
    qp = orc.pool(orc.reorder(_bf16_bits_of(x), w), w)[0, 0]
    assert qp.shape[0] == 2
    assert np.all(qp[0] == 1.5) and np.all(qp[1] == 5.0)
    counts = orc.block_valid_counts(w)
    assert counts.tolist() == [16, 12]


@pytest.mark.parametrize("g", [dict(F=3, Hs=5, Ws=7, tf=2, th=2, tw=4),
                               dict(F=4, Hs=9, Ws=10, tf=2, th=8, tw=8)])
def test_pool_random_vs_numpy_mean(orc, g):
    """Second opinion: numpy's mean over the tokens of each tile, taken
    straight from the raster tensor by tile coordinates."""
    w = synth.custom_workload(B=2, H=2, D=16, **g)
    q, _, _, _ = synth.make_qkv(w)
    bits = synth.bf16_bits(q)
    qf = q.float().numpy().astype(np.float64)
    qp = orc.pool(orc.reorder(bits, w), w)
    geo = orc.geometry(w)
    f, y, x = np.meshgrid(np.arange(w.F), np.arange(w.Hs), np.arange(w.Ws), indexing="ij")
    tile = ((f // w.tf) * geo["nby"] + y // w.th) * geo["nbx"] + x // w.tw
    tile = tile.ravel()
    for blk in range(geo["nb"]):
        sel = tile == blk
        want = qf[:, sel].mean(axis=1)        # [B, H, D]
        np.testing.assert_allclose(qp[:, :, blk], want, rtol=0, atol=1e-13)


# ---------------------------------------------------------------- logits

def test_logits_vs_numpy_matmul(orc):
    rng = np.random.default_rng(3)
    qp = rng.standard_normal((2, 3, 17, 16))
    kp = rng.standard_normal((2, 3, 17, 16))
    L = orc.logits(qp, kp, 0.25)
    want = np.matmul(qp, np.swapaxes(kp, -1, -2)) * 0.25
    np.testing.assert_allclose(L, want, rtol=1e-13, atol=1e-13)


def test_logits_closed_forms(orc):
    """Scores of structured pooled vectors, known without any product:
    unit vectors give scale on the diagonal and 0 elsewhere; constant rows
    give scale * D * a * b; a transposed operand or a dropped scale fails."""
    nb, D, scale = 6, 8, 0.5
    eye = np.zeros((1, 1, nb, D))
    for i in range(nb):
        eye[0, 0, i, i % D] = 1.0
    L = orc.logits(eye, eye, scale)[0, 0]
    np.testing.assert_array_equal(L, scale * np.eye(nb))
    a = np.arange(1, nb + 1, dtype=np.float64)          # row i of Qp is all a_i
    b = np.arange(nb, 0, -1, dtype=np.float64) * 0.25   # row j of Kp is all b_j
    qp = np.repeat(a[:, None], D, axis=1)[None, None]
    kp = np.repeat(b[:, None], D, axis=1)[None, None]
    L = orc.logits(qp, kp, scale)[0, 0]
    for i in range(nb):
        for j in range(nb):
            assert L[i, j] == scale * D * a[i] * b[j]


# ---------------------------------------------------------------- select

def _probs_in_order(L):
    """Probabilities in the order (logit desc, index asc), by numpy."""
    L = np.asarray(L, dtype=np.float32)
    order = np.lexsort((np.arange(len(L)), -L.astype(np.float64)))
    e = np.exp(L.astype(np.float64) - L.max())
    return order, e[order] / e.sum()


def test_select_all_equal_logits(orc):
    """Uniform mass 1/nb: m_p = ceil(p*nb), kept = {0..m-1} by the index tie-break."""
    nb = 10
    for p in (0.05, 0.33, 0.55, 0.91):
        idx, cnt, mp, tie = orc.select(np.zeros((1, nb)), p, 1)
        m = math.ceil(p * nb)
        assert mp[0] == m and cnt[0] == m and tie[0] == 0
        assert idx[0, :m].tolist() == list(range(m))
        assert np.all(idx[0, m:] == -1)


def test_select_dominant_block(orc):
    """One block holds ~all mass: Top-p keeps it alone; the Top-k floor adds
    the next k-1 in order (all tied at 0, so the lowest indices)."""
    nb, j0 = 12, 7
    L = np.zeros((1, nb), dtype=np.float32)
    L[0, j0] = 60.0
    idx, cnt, mp, _ = orc.select(L, 0.9, 1)
    assert mp[0] == 1 and cnt[0] == 1 and idx[0, 0] == j0
    idx, cnt, mp, _ = orc.select(L, 0.9, 4)
    assert mp[0] == 1 and cnt[0] == 4
    assert idx[0, :4].tolist() == [0, 1, 2, 7]


def test_select_floor_at_least_nb(orc):
    rng = np.random.default_rng(5)
    L = rng.standard_normal((3, 9)).astype(np.float32)
    idx, cnt, _, _ = orc.select(L, 0.2, 50)
    assert np.all(cnt == 9)
    assert np.all(idx == np.arange(9))


def test_select_p_one_keeps_everything(orc):
    rng = np.random.default_rng(6)
    L = (rng.standard_normal((4, 11)) * 5).astype(np.float32)
    idx, cnt, mp, tie = orc.select(L, 1.0, 1)
    assert np.all(cnt == 11) and np.all(mp == 11) and np.all(tie == 0)


@pytest.mark.parametrize("seed", range(4))
def test_select_invariants(orc, seed):
    """Minimal prefix (c_{m_p} >= p > c_{m_p-1}), floor, ascending output,
    kept sets nested as p grows."""
    rng = np.random.default_rng(seed)
    nb = 37
    L = (rng.standard_normal((20, nb)) * rng.uniform(0.1, 4, size=(20, 1))).astype(np.float32)
    prev = None
    for p in (0.3, 0.5, 0.7, 0.9, 0.99):
        for k in (1, 5):
            idx, cnt, mp, tie = orc.select(L, p, k)
            for r in range(L.shape[0]):
                order, pr = _probs_in_order(L[r])
                c = np.cumsum(pr)
                m_p = int(mp[r])
                assert c[m_p - 1] >= p - 1e-12
                if m_p > 1:
                    assert c[m_p - 2] < p + 1e-12
                assert cnt[r] == max(m_p, min(k, nb))
                kept = idx[r, :cnt[r]]
                assert np.all(np.diff(kept) > 0)
                assert set(kept.tolist()) == set(order[:cnt[r]].tolist())
        if prev is not None:
            for r in range(L.shape[0]):
                assert set(prev[r]) <= set(idx[r, :cnt[r]].tolist())
        prev = [idx[r, :cnt[r]].tolist() for r in range(L.shape[0])]


@pytest.mark.parametrize("seed", range(6))
def test_select_brute_force_minimal_prefix(orc, seed):
    """Over all subsets of a row with nb <= 10: no smaller subset reaches p,
    and the kept set is the highest-mass subset of its size."""
    rng = np.random.default_rng(100 + seed)
    nb = int(rng.integers(3, 11))
    L = (rng.standard_normal(nb) * rng.uniform(0.5, 3)).astype(np.float32)
    p = float(rng.uniform(0.3, 0.95))
    idx, cnt, mp, tie = orc.select(L[None], p, 1)
    e = np.exp(L.astype(np.float64) - L.max())
    P = e / e.sum()
    m_p = int(mp[0])
    best_by_size = {}
    for size in range(1, nb + 1):
        best_by_size[size] = max(sum(P[list(s)]) for s in itertools.combinations(range(nb), size))
    assert best_by_size[m_p] >= p - 1e-12
    if m_p > 1:
        assert best_by_size[m_p - 1] < p + 1e-12
    kept = idx[0, :cnt[0]].tolist()
    assert abs(sum(P[kept]) - best_by_size[m_p]) < 1e-12


def test_select_near_tie_flag(orc):
    """Masses (0.5, 0.25, 0.25) in exact binary: p = 0.75 is reached exactly
    at m_p = 2, which must be flagged; p = 0.7 is far from any partial sum."""
    L = np.log(np.array([[2.0, 1.0, 1.0]])).astype(np.float32)
    _, cnt, mp, tie = orc.select(L, 0.75, 1)
    assert tie[0] == 1
    _, cnt, mp, tie = orc.select(L, 0.7, 1)
    assert mp[0] == 2 and tie[0] == 0


def _read_golden(name):
    cases = []
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            fields = [s.strip() for s in line.split("|")]
            logit_s, p_s, k_s, kept_s = fields[:4]
            extra = int(fields[4]) if len(fields) > 4 else 0
            logits = [float(v) for v in logit_s.split()]
            kept = [int(v) for v in kept_s.split()]
            cases.append((logits, float(p_s), int(k_s), kept, extra))
    return cases


def test_select_golden_hand_cases(orc):
    """Hand-derived rows (tests/golden/select_hand_cases.txt, each with its
    derivation)."""
    cases = _read_golden("select_hand_cases.txt")
    assert len(cases) >= 6
    assert sum(1 for c in cases if c[1] == 0.0) >= 3 and sum(1 for c in cases if c[4] > 0) >= 3
    for logits, p, k, kept, extra in cases:
        idx, cnt, _, tie = orc.select(np.array([logits], dtype=np.float32), p, k, k_extra=extra)
        assert tie[0] == 0
        assert idx[0, :cnt[0]].tolist() == kept, (logits, p, k, extra)


def _order(row):
    """Block order by (logit descending, index ascending), from numpy's lexsort."""
    return np.lexsort((np.arange(row.size), -row.astype(np.float64)))


def test_fixed_topk_mode_matches_sorted_order(orc):
    """p = 0: exactly min(k, nb) blocks, the first of the (logit desc, index
    asc) order, including rows with repeated logits."""
    rng = np.random.default_rng(11)
    for nb in (1, 5, 37, 200):
        L = rng.normal(size=(30, nb)).astype(np.float32)
        L[::3, : nb // 2] = 0.5   # ties
        for k in (1, 3, nb, nb + 4):
            idx, cnt, mp, _ = orc.select(L, 0.0, k)
            assert np.all(mp == 0)
            assert np.all(cnt == min(k, nb))
            for r in range(L.shape[0]):
                want = np.sort(_order(L[r])[: min(k, nb)])
                assert np.array_equal(idx[r, : cnt[r]], want)


def test_augmentation_appends_the_next_blocks(orc):
    """k_extra = e keeps min(nb, m + e) blocks, m the plain Top-p/Top-k count;
    the added blocks are the next ones of the order, so sets are nested."""
    rng = np.random.default_rng(12)
    nb = 64
    L = (rng.normal(size=(40, nb)) * rng.uniform(0.2, 5.0, size=(40, 1))).astype(np.float32)
    base_idx, base_cnt, base_mp, _ = orc.select(L, 0.8, 3)
    prev = [set(base_idx[r, : base_cnt[r]].tolist()) for r in range(L.shape[0])]
    for e in (1, 2, 7, nb):
        idx, cnt, mp, _ = orc.select(L, 0.8, 3, k_extra=e)
        assert np.array_equal(mp, base_mp)
        assert np.all(cnt == np.minimum(nb, base_cnt + e))
        for r in range(L.shape[0]):
            kept = set(idx[r, : cnt[r]].tolist())
            assert prev[r] <= kept
            assert kept == set(_order(L[r])[: cnt[r]].tolist())
            prev[r] = kept
