"""Pins of the CPU oracle against facts fixed outside the oracle itself.

Each test checks the oracle against something it cannot agree with by
construction: hand-drawn masks, hand-derived planted index sets, closed forms
of uniform softmax, a library attention routine on the special case that
reduces to it, and brute-force enumeration on tiny inputs.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from workload import TEXT, VIDEO, Head, Problem, bf16_to_f32, make_inputs, grid_single_head

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _head(spec):
    spec = dict(spec)
    if "strides" in spec:
        spec["strides"] = tuple(spec["strides"])
    return Head(**spec)


def _problem(case):
    return Problem(L=case["L"], Hq=1, Hkv=1, segments=[tuple(s) for s in case["segments"]],
                   heads=[_head(case["head"])])


def _index(raw):
    idx = {}
    for key, val in raw.items():
        if isinstance(val, dict):
            d = {}
            for k2, v2 in val.items():
                k = tuple(int(x) for x in k2.split(",")) if "," in k2 else int(k2)
                d[k] = np.asarray(v2, np.int64)
            idx[key] = d
        elif isinstance(val, list) and val and isinstance(val[0], list):
            idx[key] = [np.asarray(v, np.int64) for v in val]
        elif isinstance(val, list):
            idx[key] = np.asarray(val, np.int64)
        else:
            idx[key] = val
    return idx


def _bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 values exactly representable in bf16 -> bit patterns."""
    b = np.ascontiguousarray(x, np.float32).view(np.uint32)
    assert np.all((b & 0xFFFF) == 0)
    return (b >> 16).astype(np.uint16)


# ------------------------------------------------------------------------------------------
# masks: hand-drawn fixtures
# ------------------------------------------------------------------------------------------
with open(os.path.join(GOLDEN, "masks.json")) as f:
    MASKS = json.load(f)


@pytest.mark.parametrize("case", MASKS["cases"], ids=[c["name"] for c in MASKS["cases"]])
def test_mask_fixture(case):
    p = _problem(case)
    got = oracle.mask_rows(p, 0, _index(case["index"]), np.arange(p.L))
    exp = np.array([[1 if ch == "1" else 0 for ch in row] for row in case["expected"]], np.uint8)
    assert got.shape == exp.shape
    assert np.array_equal(got, exp), "\n" + "\n".join("".join("1" if x else "." for x in r) for r in got)


def test_block_mask_fixture():
    case = MASKS["block_cases"][0]
    p = Problem(L=case["L"], Hq=1, Hkv=1, segments=[(0, case["L"], TEXT)], heads=[Head("block", topk_blocks=1)])
    idx = {"T": [np.asarray(t, np.int64) for t in case["T"]]}
    got = oracle.mask_rows(p, 0, idx, np.arange(p.L))
    eb = np.array([[1 if ch == "1" else 0 for ch in row] for row in case["expected_blocks"]], np.uint8)
    exp = np.kron(eb, np.ones((64, 64), np.uint8)) & np.tril(np.ones((p.L, p.L), np.uint8))
    assert np.array_equal(got, exp)


# ------------------------------------------------------------------------------------------
# masks: special cases that reduce to another pattern
# ------------------------------------------------------------------------------------------
def test_vslash_reduces_to_ashape():
    L, sink, local = 512, 16, 40
    pa = Problem(L=L, Hq=1, Hkv=1, segments=[(0, L, TEXT)], heads=[Head("ashape", sink=sink, local=local)])
    pv = Problem(L=L, Hq=1, Hkv=1, segments=[(0, L, TEXT)], heads=[Head("vslash")])
    rows = np.arange(L)
    ma = oracle.mask_rows(pa, 0, {}, rows)
    mv = oracle.mask_rows(pv, 0, {"V": np.arange(sink), "S": np.arange(local)}, rows)
    assert np.array_equal(ma, mv)


def test_block_all_blocks_is_dense_causal():
    L = 384
    p = Problem(L=L, Hq=1, Hkv=1, segments=[(0, L, TEXT)], heads=[Head("block", topk_blocks=L // 64)])
    idx = {"T": [np.arange(b + 1) for b in range(L // 64)]}
    assert np.array_equal(oracle.mask_rows(p, 0, idx, np.arange(L)), np.tril(np.ones((L, L), np.uint8)))


def test_grid_all_phases_is_dense_causal():
    p = Problem(L=320, Hq=1, Hkv=1, segments=[(0, 64, TEXT), (64, 256, VIDEO)], heads=[Head("grid", strides=(32,))])
    m = oracle.mask_rows(p, 0, {"stride": 32, "phases": np.arange(32)}, np.arange(p.L))
    assert np.array_equal(m, np.tril(np.ones((p.L, p.L), np.uint8)))


def test_qbound_and_bound2d_reduce_to_vslash_on_one_modality():
    L = 256
    rng = np.random.default_rng(1)
    V = np.sort(rng.choice(L, 9, replace=False))
    S = np.sort(rng.choice(L, 17, replace=False))
    rows = np.arange(L)
    pv = Problem(L=L, Hq=1, Hkv=1, segments=[(0, L, TEXT)], heads=[Head("vslash")])
    pq = Problem(L=L, Hq=1, Hkv=1, segments=[(0, L, TEXT)], heads=[Head("qbound")])
    p2 = Problem(L=L, Hq=1, Hkv=1, segments=[(0, L, TEXT)], heads=[Head("bound2d")])
    mv = oracle.mask_rows(pv, 0, {"V": V, "S": S}, rows)
    mq = oracle.mask_rows(pq, 0, {"V": {TEXT: V}, "S": {TEXT: S}}, rows)
    m2 = oracle.mask_rows(p2, 0, {"V": {(TEXT, TEXT): V}, "S": {TEXT: S}}, rows)
    assert np.array_equal(mv, mq) and np.array_equal(mv, m2)


# ------------------------------------------------------------------------------------------
# last-query sums: closed form of the uniform softmax, and invariants
# ------------------------------------------------------------------------------------------
def test_lastq_sums_uniform_closed_form():
    L, d = 300, 128
    Qh = np.zeros((L, d), np.uint16)  # every logit 0 -> A[r, j] = 1 / (i_r + 1) on j <= i_r
    rng = np.random.default_rng(0)
    Kh = _bf16_bits(np.round(rng.standard_normal((L, d)) * 4) / 4)
    rows = np.array([5, 17, 120, 121, 299])
    v, s = oracle.lastq_sums(Qh, Kh, 0.088, rows)
    ev = np.array([sum(1.0 / (i + 1) for i in rows if i >= j) for j in range(L)])
    es = np.array([sum(1.0 / (i + 1) for i in rows if i >= o) for o in range(L)])
    np.testing.assert_allclose(v, ev, rtol=0, atol=1e-13)
    np.testing.assert_allclose(s, es, rtol=0, atol=1e-13)


def test_lastq_sums_uniform_compacted_coordinates():
    # keys take part in the slash sum only on their own coordinate; offset o sums A[r, j]
    # over keys whose coordinate is rcoord[r] - o
    L, d = 40, 128
    Qh = np.zeros((L, d), np.uint16)
    Kh = np.zeros((L, d), np.uint16)
    rows = np.array([30, 39])
    kco = np.full(L, -1)
    kco[::3] = np.arange(len(kco[::3]))  # keys 0,3,6,... have coordinates 0,1,2,...
    rco = np.array([10, 13])
    _, s = oracle.lastq_sums(Qh, Kh, 0.1, rows, rcoord=rco, kcoord=kco)
    es = np.zeros(L)
    for i, rc in zip(rows, rco):
        for j in range(0, i + 1):
            if kco[j] >= 0 and rc - kco[j] >= 0:
                es[rc - kco[j]] += 1.0 / (i + 1)
    np.testing.assert_allclose(s, es, atol=1e-14)


def test_lastq_sums_mass_invariants():
    p = grid_single_head(L=1024, text=128, stride=128)
    Q, K, _ = make_inputs(p, seed=3)
    rows = np.arange(p.L - 64, p.L)
    v, s = oracle.lastq_sums(Q[0], K[0], p.scale, rows)
    assert abs(v.sum() - 64) < 1e-9 and abs(s.sum() - 64) < 1e-9
    assert np.all(v >= 0) and np.all(s >= 0)


# ------------------------------------------------------------------------------------------
# top-k: brute force on tiny inputs
# ------------------------------------------------------------------------------------------
@pytest.mark.parametrize("seed", range(6))
def test_topk_brute_force(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 60))
    sc = rng.integers(0, 6, n).astype(np.float64) / 7.0  # many exact ties
    cand = rng.random(n) < 0.7
    for k in (0, 1, 3, n, n + 5):
        items = [(-float(np.float32(sc[j])), j) for j in range(n) if cand[j]]
        exp = sorted(j for _, j in sorted(items)[:k])
        got = oracle.topk(sc, k, cand.astype(np.uint8)).tolist()
        assert got == exp


def test_topk_decides_in_fp32():
    # two scores that differ only below fp32 resolution tie, and the lower index wins
    sc = np.array([1.0, 1.0 + 1e-12, 0.5])
    assert oracle.topk(sc, 1).tolist() == [0]


# ------------------------------------------------------------------------------------------
# pooling and grid scores: closed forms and enumeration
# ------------------------------------------------------------------------------------------
def test_pool64_closed_form():
    L, d = 256, 128
    X = np.zeros((L, d), np.float32)
    X[:, 0] = np.arange(L)  # integers < 256 are exact in bf16
    X[:, 5] = -2.0
    P = oracle.pool64(_bf16_bits(X))
    np.testing.assert_array_equal(P[:, 0], 64 * np.arange(4) + 31.5)
    np.testing.assert_array_equal(P[:, 5], -2.0)
    assert np.all(P[:, 1] == 0)


def test_grid_scores_enumeration():
    p = Problem(L=192, Hq=1, Hkv=1, segments=[(0, 37, VIDEO), (37, 27, TEXT), (64, 128, VIDEO)],
                heads=[Head("grid", strides=(5,))])
    rng = np.random.default_rng(7)
    v = rng.random(p.L)
    for st in (3, 5, 16):
        got = oracle.grid_scores(p, v, st)
        for ph in range(st):
            vals = [v[t] for (s0, n, m) in p.segments if m == VIDEO for t in range(s0, s0 + n)
                    if (t - s0) % st == ph]
            assert abs(got[ph] - (np.mean(vals) if vals else 0.0)) < 1e-12


def test_budget_rounding():
    assert oracle.budget_scale(1000, 124740, 131072) == 952   # 951.69 -> 952
    assert oracle.budget_scale(1, 192, 256) == 1
    assert oracle.budget_scale(3, 1, 6) == 1                  # 0.5 rounds half up, at least 1
    assert oracle.budget_scale(7, 0, 10) == 0
    head = Head("grid", strides=(224,), grid_budget=0.10)
    assert oracle.grid_phase_count(head, 224) == 11
    assert oracle.grid_phase_count(Head("grid", strides=(256,), grid_budget=0.05), 256) == 6
    kk = oracle.block_row_k(Head("block", block_budget=0.25), 9)
    assert kk.tolist() == [1, 1, 1, 1, 2, 2, 2, 2, 3]


# ------------------------------------------------------------------------------------------
# planted estimation cases
# ------------------------------------------------------------------------------------------
with open(os.path.join(GOLDEN, "estimation.json")) as f:
    EST = json.load(f)


def _planted(case):
    p = _problem(case)
    L, d = p.L, 128
    Qf = np.zeros((L, d), np.float32)
    Kf = np.zeros((L, d), np.float32)
    for a, b, ax in case["q_rows"]:
        Qf[a:b, ax] = 8.0
    for a, b, ax in case.get("k_rows", []):
        Kf[a:b, ax] = 8.0
    if "k_rows_phase" in case:
        kp = case["k_rows_phase"]
        mask = (p.modality() == VIDEO) & ((np.arange(L) - p.seg_start()) % kp["stride"] == kp["phase"])
        Kf[mask, kp["axis"]] = 8.0
    Q = _bf16_bits(Qf)[None]
    K = _bf16_bits(Kf)[None]
    return p, Q, K


@pytest.mark.parametrize("case", EST["cases"], ids=[c["name"] for c in EST["cases"]])
def test_planted_estimation(case):
    p, Q, K = _planted(case)
    got = oracle.estimate_head(p, 0, Q, K)
    for key, val in _index(case["expect"]).items():
        if key == "T":
            assert [t.tolist() for t in got["T"]] == [list(t) for t in case["expect"]["T"]]
        elif isinstance(val, dict):
            for k2, arr in val.items():
                assert got[key][k2].tolist() == arr.tolist(), (key, k2)
        elif isinstance(val, np.ndarray):
            assert got[key].tolist() == val.tolist(), key
        else:
            assert got[key] == val, key


def test_planted_video_queries_recover_frame_stride():
    # planted Q (last 64 video rows) and K (frame-stride keys) share +2u: phase 0 must win
    p = grid_single_head(L=4096, text=512, stride=224, budget=0.10)
    Q, K, _ = make_inputs(p, seed=0, plant_queries=True)
    est = oracle.estimate_head(p, 0, Q, K)
    assert est["stride"] == 224
    assert 0 in est["phases"].tolist()
    assert int(np.argmax(est["scores"])) == 0


# ------------------------------------------------------------------------------------------
# attention: library routine on the all-ones mask, closed form on uniform logits
# ------------------------------------------------------------------------------------------
def test_dense_attention_matches_sdpa():
    L, d = 320, 128
    p = Problem(L=L, Hq=1, Hkv=1, segments=[(0, L, TEXT)], heads=[Head("dense")])
    Q, K, V = make_inputs(p, seed=11)
    O, lse = oracle.attention_head(p, 0, Q, K, V, {})
    q, k, v = (torch.from_numpy(bf16_to_f32(x[0]).astype(np.float64)) for x in (Q, K, V))
    ref = torch.nn.functional.scaled_dot_product_attention(q[None], k[None], v[None], is_causal=True,
                                                           scale=float(p.scale))[0]
    np.testing.assert_allclose(O, ref.numpy(), atol=2e-6, rtol=1e-5)
    logits = (q @ k.T) * float(p.scale)
    logits = logits.masked_fill(torch.ones(L, L, dtype=torch.bool).triu(1), float("-inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(logits, -1).numpy(), atol=1e-5, rtol=1e-6)


def test_gqa_head_mapping():
    # q-head h reads kv-head h // (Hq / Hkv)
    L = 128
    p = Problem(L=L, Hq=4, Hkv=2, segments=[(0, L, TEXT)], heads=[Head("dense")] * 4)
    Q, K, V = make_inputs(p, seed=2)
    for h in range(4):
        O, _ = oracle.attention_head(p, h, Q, K, V, {})
        kv = h // 2
        q, k, v = (torch.from_numpy(bf16_to_f32(x).astype(np.float64)) for x in (Q[h], K[kv], V[kv]))
        ref = torch.nn.functional.scaled_dot_product_attention(q[None], k[None], v[None], is_causal=True,
                                                               scale=float(p.scale))[0]
        np.testing.assert_allclose(O, ref.numpy(), atol=2e-6, rtol=1e-5)


@pytest.mark.parametrize("case", MASKS["cases"], ids=[c["name"] for c in MASKS["cases"]])
def test_uniform_attention_is_mean_of_allowed_values(case):
    # zero queries: every logit is 0, so O_i = mean of V over the allowed keys and lse_i = log(count)
    p = _problem(case)
    idx = _index(case["index"])
    Q = np.zeros((1, p.L, 128), np.uint16)
    rng = np.random.default_rng(5)
    K = _bf16_bits(np.round(rng.standard_normal((p.L, 128)) * 4) / 4)[None]
    V = _bf16_bits(np.round(rng.standard_normal((p.L, 128)) * 8) / 8)[None]
    O, lse = oracle.attention_head(p, 0, Q, K, V, idx)
    exp = np.array([[1 if ch == "1" else 0 for ch in row] for row in case["expected"]], np.float64)
    Vf = bf16_to_f32(V[0]).astype(np.float64)
    for i in range(p.L):
        n = exp[i].sum()
        if n == 0:
            assert np.all(O[i] == 0) and lse[i] == -np.inf
        else:
            np.testing.assert_allclose(O[i], (exp[i] @ Vf) / n, atol=1e-6)
            assert abs(lse[i] - math.log(n)) < 1e-6
