"""Pin of the oracle's masked attention by its permutation invariance.

The MMInference review page ("core discovery") realises the permutation as index-based
loading, so permuting a head's queries and keys, attending in permuted coordinates with the
mask evaluated through the original positions, and scattering the rows back must give the
output of the direct masked attention.  The two oracle routines share the mask predicate and
the logit, but not the order in which rows and keys are visited, so a mistake in how either
of them maps a row or a key to its position (a transposed index, a mask taken in permuted
coordinates, a missing scatter) fails here.  The direct routine is pinned separately (hand
masks, SDPA, closed forms); this file ties the permuted one to it.

Equality is to fp32 rounding of the same fp64 sums taken in another order: at most two units
in the last place of each output element.
"""
import numpy as np
import pytest

import oracle
from workload import TEXT, VIDEO, Head, Problem, make_inputs


def _layouts():
    """L <= 512 layouts of every kind, video frames interrupted by text."""
    segs = [(0, 64, TEXT), (64, 160, VIDEO), (224, 32, TEXT), (256, 192, VIDEO), (448, 64, TEXT)]
    P = {
        "grid": Problem(L=512, Hq=2, Hkv=1, segments=segs, frame_stride=32,
                        heads=[Head("grid", strides=(32,), grid_budget=0.2), Head("grid", strides=(16, 32), n_phases=2)]),
        "qbound": Problem(L=512, Hq=2, Hkv=1, segments=segs,
                          heads=[Head("qbound", k_v=20, k_s=40), Head("qbound", k_v=5, k_s=90)]),
        "bound2d": Problem(L=512, Hq=2, Hkv=1, segments=segs,
                           heads=[Head("bound2d", k_v=30, k_s=40), Head("bound2d", k_v=80, k_s=10)]),
        "vslash": Problem(L=384, Hq=2, Hkv=1, segments=[(0, 384, TEXT)],
                          heads=[Head("vslash", k_v=12, k_s=30), Head("vslash", k_v=40, k_s=5)]),
        "block": Problem(L=448, Hq=2, Hkv=1, segments=[(0, 448, TEXT)],
                         heads=[Head("block", topk_blocks=2), Head("block", block_budget=0.3)]),
        "ashape": Problem(L=320, Hq=1, Hkv=1, segments=[(0, 320, TEXT)], heads=[Head("ashape", sink=16, local=48)]),
        "dense": Problem(L=256, Hq=1, Hkv=1, segments=[(0, 256, TEXT)], heads=[Head("dense")]),
    }
    return P


LAYOUTS = _layouts()


def _assert_same(Oa, la, Ob, lb, what):
    Oa, Ob = np.asarray(Oa, np.float32), np.asarray(Ob, np.float32)
    tol = 2.0 * np.spacing(np.maximum(np.abs(Oa), np.abs(Ob))) + 1e-30
    bad = np.abs(Oa.astype(np.float64) - Ob.astype(np.float64)) > tol
    assert not bad.any(), f"{what}: {int(bad.sum())} output elements differ beyond 2 ulp"
    fin = np.isfinite(la)
    assert np.array_equal(fin, np.isfinite(lb)), f"{what}: empty rows differ"
    assert np.array_equal(la[~fin], lb[~fin])
    ltol = 2.0 * np.spacing(np.maximum(np.abs(la[fin]), np.abs(lb[fin]))) + 1e-30
    assert np.all(np.abs(la[fin].astype(np.float64) - lb[fin].astype(np.float64)) <= ltol), f"{what}: lse differs"


def _is_perm(x, L):
    return np.array_equal(np.sort(np.asarray(x)), np.arange(L))


@pytest.mark.parametrize("name", list(LAYOUTS))
def test_method_permutation_round_trip(name):
    """permute -> attend -> unpermute with the head's own permutation equals direct attention."""
    p = LAYOUTS[name]
    Q, K, V = make_inputs(p, seed=31)
    idx = oracle.estimate(p, Q, K)
    for h in range(p.Hq):
        qperm, kperm = oracle.permutation(p, h, idx[h])
        assert _is_perm(qperm, p.L) and _is_perm(kperm, p.L)
        O, lse = oracle.attention_head(p, h, Q, K, V, idx[h])
        Op, lp = oracle.attention_permuted(p, h, Q, K, V, idx[h], qperm, kperm)
        _assert_same(Op, lp, O, lse, f"{name} head {h}")


def test_method_permutations_make_selected_entries_contiguous():
    """The permutations put what each head selects in front: grid lines (rows and columns),
    queries and keys grouped per modality, vertical lines gathered ahead of the other keys."""
    mod_of = {}
    for name in ("grid", "qbound", "bound2d", "vslash"):
        p = LAYOUTS[name]
        Q, K, _ = make_inputs(p, seed=31)
        idx = oracle.estimate(p, Q, K)[0]
        qperm, kperm = oracle.permutation(p, 0, idx)
        mod = p.modality()
        mod_of[name] = mod
        if name == "grid":
            g = np.nonzero(oracle.grid_marks(p, idx["stride"], idx["phases"]))[0]
            assert 0 < len(g) < p.L
            assert np.array_equal(qperm[:len(g)], g) and np.array_equal(kperm[:len(g)], g)
        elif name in ("qbound", "bound2d"):
            nt = int((mod == TEXT).sum())
            assert np.all(mod[qperm[:nt]] == TEXT) and np.all(mod[qperm[nt:]] == VIDEO)
            assert np.all(np.diff(qperm[:nt]) > 0) and np.all(np.diff(qperm[nt:]) > 0)
            if name == "bound2d":
                assert np.array_equal(kperm, qperm)
            else:
                assert np.array_equal(kperm, np.arange(p.L))
        else:
            nv = len(idx["V"])
            assert np.array_equal(kperm[:nv], np.sort(idx["V"]))
            assert np.array_equal(qperm, np.arange(p.L))
        assert not np.array_equal(qperm, np.arange(p.L)) or not np.array_equal(kperm, np.arange(p.L))


@pytest.mark.parametrize("name", list(LAYOUTS))
@pytest.mark.parametrize("seed", [0, 1])
def test_random_permutation_round_trip(name, seed):
    """Any permutation of the query axis and any (independent) permutation of the key axis."""
    p = LAYOUTS[name]
    Q, K, V = make_inputs(p, seed=40 + seed)
    idx = oracle.estimate(p, Q, K)
    rng = np.random.default_rng(1234 + seed)
    for h in range(p.Hq):
        qperm = rng.permutation(p.L)
        kperm = rng.permutation(p.L)
        O, lse = oracle.attention_head(p, h, Q, K, V, idx[h])
        Op, lp = oracle.attention_permuted(p, h, Q, K, V, idx[h], qperm, kperm)
        _assert_same(Op, lp, O, lse, f"{name} head {h} seed {seed}")


def test_round_trip_detects_a_mask_taken_in_permuted_coordinates():
    """The check has teeth: gathering the rows but evaluating the mask at the permuted row and
    key numbers (positions not carried through) changes the output of a permuted head."""
    p = LAYOUTS["grid"]
    Q, K, V = make_inputs(p, seed=31)
    idx = oracle.estimate(p, Q, K)[0]
    qperm, kperm = oracle.permutation(p, 0, idx)
    O, _ = oracle.attention_head(p, 0, Q, K, V, idx)
    Qp = Q.copy()
    Kp = K.copy()
    Vp = V.copy()
    Qp[0] = Q[0][qperm]
    Kp[0] = K[0][kperm]
    Vp[0] = V[0][kperm]
    wrong, _ = oracle.attention_permuted(p, 0, Qp, Kp, Vp, idx, np.arange(p.L), np.arange(p.L))
    back = np.zeros_like(wrong)
    back[qperm] = wrong
    assert np.abs(back - O).max() > 1e-2


def test_round_trip_detects_a_missing_scatter():
    p = LAYOUTS["bound2d"]
    Q, K, V = make_inputs(p, seed=31)
    idx = oracle.estimate(p, Q, K)[0]
    qperm, kperm = oracle.permutation(p, 0, idx)
    O, _ = oracle.attention_head(p, 0, Q, K, V, idx)
    Op, _ = oracle.attention_permuted(p, 0, Q, K, V, idx, qperm, kperm)
    assert np.abs(Op[qperm] - O).max() > 1e-2  # permuted order read as original order
