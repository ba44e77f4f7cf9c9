"""Pins of the oracle's per-segment Q-boundary option (the last 64 queries of each modality
segment estimate an index that serves that segment's queries; MMInference review page, "core
discovery", read literally) against a hand-drawn mask and hand-derived planted index sets."""
import math

import numpy as np

import oracle
from workload import TEXT, VIDEO, Head, Problem, make_inputs


def _bits(x):
    b = np.ascontiguousarray(np.asarray(x, np.float32)).view(np.uint32)
    assert np.all((b & 0xFFFF) == 0)
    return (b >> 16).astype(np.uint16)


def test_per_segment_mask_hand_drawn():
    """T(3) V(3) T(2); each segment's queries use their own vertical and slash lines."""
    segs = [(0, 3, TEXT), (3, 3, VIDEO), (6, 2, TEXT)]
    p = Problem(L=8, Hq=1, Hkv=1, segments=segs, heads=[Head("qbound", k_v=1, k_s=1, per_segment=True)])
    idx = {"kind": "qbound", "per_segment": True,
           "V": {0: np.array([0]), 1: np.array([2]), 2: np.array([5])},
           "S": {0: np.array([0]), 1: np.array([1]), 2: np.array([0])}}
    expected = ["1.......",
                "11......",
                "1.1.....",
                "..1.....",
                "..11....",
                "..1.1...",
                ".....11.",
                ".....1.1"]
    got = oracle.mask_rows(p, 0, idx, np.arange(p.L))
    exp = np.array([[1 if ch == "1" else 0 for ch in row] for row in expected], np.uint8)
    assert np.array_equal(got, exp), "\n" + "\n".join("".join("1" if x else "." for x in r) for r in got)


def test_per_segment_estimation_planted_columns():
    """Segment k's last rows look along direction e_k, and key c_k (inside their causal range) is
    the only key along it: each segment's vertical line is its own c_k, although the two text
    segments share a modality (one index per modality would give both the same line)."""
    segs = [(0, 128, TEXT), (128, 192, VIDEO), (320, 128, TEXT), (448, 128, VIDEO)]
    L = 576
    cols = {0: 40, 1: 150, 2: 300, 3: 10}
    Q = np.zeros((1, L, 128), np.float32)
    K = np.zeros((1, L, 128), np.float32)
    for k, (st, n, _) in enumerate(segs):
        Q[0, st + n - 64: st + n, k] = 4.0  # logit 4 * 64 * scale = 22.6 against 0 elsewhere
        K[0, cols[k], k] = 64.0
    p = Problem(L=L, Hq=1, Hkv=1, segments=segs, heads=[Head("qbound", k_v=1, k_s=4, per_segment=True)])
    est = oracle.estimate_head(p, 0, _bits(Q), _bits(K))
    assert est["per_segment"]
    for k in range(len(segs)):
        assert est["V"][k].tolist() == [cols[k]], (k, est["V"][k])
        assert len(est["S"][k]) == 4
        # every row of the segment puts nearly all its mass on c_k: v[c_k] close to 64
        assert est["v"][k][cols[k]] > 63.0
    # the per-modality reading estimates one index per modality from its last segment only
    q = Problem(L=L, Hq=1, Hkv=1, segments=segs, heads=[Head("qbound", k_v=1, k_s=4)])
    est_mod = oracle.estimate_head(q, 0, _bits(Q), _bits(K))
    assert est_mod["V"][TEXT].tolist() == [cols[2]] and est_mod["V"][VIDEO].tolist() == [cols[3]]


def test_per_segment_short_segments_use_all_their_rows():
    """A segment shorter than 64 tokens estimates from all of its rows: the vertical sums of
    uniform rows (Q = 0) are the closed form sum_r 1 / (i_r + 1) over the segment's rows."""
    segs = [(0, 100, VIDEO), (100, 20, TEXT), (120, 72, VIDEO)]
    L = 192
    Q = np.zeros((1, L, 128), np.uint16)
    K = np.zeros((1, L, 128), np.uint16)
    p = Problem(L=L, Hq=1, Hkv=1, segments=segs, heads=[Head("qbound", k_v=3, k_s=3, per_segment=True)])
    est = oracle.estimate_head(p, 0, Q, K)
    v1 = est["v"][1]
    rows = np.arange(100, 120)
    for j in (0, 50, 99, 100, 119):
        expect = sum(1.0 / (i + 1) for i in rows if i >= j)
        assert math.isclose(v1[j], expect, rel_tol=1e-12), (j, v1[j], expect)
    assert v1[120:].sum() == 0.0


def test_per_segment_round_trip_through_permutation():
    """permute -> attend -> unpermute equals direct attention for the per-segment option too."""
    segs = [(0, 96, TEXT), (96, 160, VIDEO), (256, 32, TEXT), (288, 96, VIDEO)]
    p = Problem(L=384, Hq=2, Hkv=1, segments=segs,
                heads=[Head("qbound", k_v=12, k_s=20, per_segment=True), Head("qbound", k_v=3, k_s=50, per_segment=True)])
    Q, K, V = make_inputs(p, seed=11)
    idx = oracle.estimate(p, Q, K)
    rng = np.random.default_rng(2)
    for h in range(p.Hq):
        O, lse = oracle.attention_head(p, h, Q, K, V, idx[h])
        qp, kp = rng.permutation(p.L), rng.permutation(p.L)
        Op, lp = oracle.attention_permuted(p, h, Q, K, V, idx[h], qp, kp)
        tol = 2.0 * np.spacing(np.maximum(np.abs(O), np.abs(Op))) + 1e-30
        assert np.all(np.abs(O.astype(np.float64) - Op) <= tol)
        fin = np.isfinite(lse)
        assert np.array_equal(fin, np.isfinite(lp))
