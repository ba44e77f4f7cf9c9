"""Shared helpers of the test suite: small problems of every head kind, device transfer,
output and index-set comparison rules."""
from __future__ import annotations

import numpy as np

import oracle
from workload import TEXT, VIDEO, Head, Problem, grid_single_head, qwen2_7b_video

# Output tolerance against the fp32 oracle (bf16 P and O on the device).
MAX_ABS = 2e-2
REL_L2 = 1e-2
# Index sets: a difference is accepted only between near-tied candidates.
TIE_REL = 1e-5


def small_problems():
    """Problems a few tiles long, with a ragged tail (L % 128 == 64) where the layout allows,
    two query heads sharing one KV head."""
    P = {}
    L = 1088
    P["dense"] = Problem(L=L, Hq=2, Hkv=1, segments=[(0, L, TEXT)], heads=[Head("dense")] * 2, name="dense")
    P["ashape"] = Problem(L=L, Hq=2, Hkv=1, segments=[(0, L, TEXT)],
                          heads=[Head("ashape", sink=64, local=256), Head("ashape", sink=3, local=100)], name="ashape")
    P["vslash"] = Problem(L=L, Hq=2, Hkv=1, segments=[(0, L, TEXT)],
                          heads=[Head("vslash", k_v=40, k_s=200), Head("vslash", k_v=130, k_s=30)], name="vslash")
    P["block"] = Problem(L=L, Hq=2, Hkv=1, segments=[(0, L, TEXT)],
                         heads=[Head("block", topk_blocks=3), Head("block", block_budget=0.25)], name="block")
    g = grid_single_head(L=1984, text=256, stride=96, budget=0.10)
    P["grid"] = Problem(L=g.L, Hq=2, Hkv=1, segments=g.segments,
                        heads=[Head("grid", strides=(96,), grid_budget=0.10), Head("grid", strides=(48, 96), n_phases=3)],
                        frame_stride=96, name="grid")
    segs = [(0, 576, VIDEO), (576, 256, TEXT), (832, 480, VIDEO), (1312, 160, TEXT)]
    P["qbound"] = Problem(L=1472, Hq=2, Hkv=1, segments=segs,
                          heads=[Head("qbound", k_v=50, k_s=120), Head("qbound", k_v=7, k_s=300)], frame_stride=96,
                          name="qbound")
    P["bound2d"] = Problem(L=1472, Hq=2, Hkv=1, segments=segs,
                           heads=[Head("bound2d", k_v=50, k_s=120), Head("bound2d", k_v=200, k_s=40)], frame_stride=96,
                           name="bound2d")
    return P


def mixed_problem():
    """Every kind in one layer (Hq = 7 over Hkv = 1 ... all heads share one KV head)."""
    segs = [(0, 576, VIDEO), (576, 256, TEXT), (832, 480, VIDEO), (1312, 160, TEXT)]
    heads = [Head("dense"), Head("ashape", sink=64, local=200), Head("vslash", k_v=60, k_s=90),
             Head("block", topk_blocks=4), Head("grid", strides=(96,), grid_budget=0.1),
             Head("qbound", k_v=30, k_s=70), Head("bound2d", k_v=60, k_s=90)]
    return Problem(L=1472, Hq=7, Hkv=1, segments=segs, heads=heads, frame_stride=96, name="mixed")


def to_dev(x: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(x)).view(torch.bfloat16).cuda()


def bf16_host(t) -> np.ndarray:
    import torch
    return t.float().cpu().numpy()


def compare_outputs(got: np.ndarray, ref: np.ndarray, what: str = ""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    mae = float(err.max()) if err.size else 0.0
    den = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(got - ref) / den) if den > 0 else float(np.linalg.norm(got - ref))
    assert mae <= MAX_ABS, f"{what}: max abs error {mae:.3e} > {MAX_ABS}"
    assert rel <= REL_L2, f"{what}: relative L2 error {rel:.3e} > {REL_L2}"
    return mae, rel


def near_tie_ok(got, ref, scores, cand=None, what="", relative_to="tau"):
    """Index sets must be identical except for swaps among near-tied candidates: every index in
    the symmetric difference must have an (fp32) oracle score within TIE_REL of the k-th
    selected score tau.

    relative_to="tau" (probability sums: vertical, slash, grid phase means, all positive):
    the bound is TIE_REL * |tau|, floored at TIE_REL * 1e-3 * max|candidate score| so that a
    k-th score that is itself a rounding-level value does not shrink it below fp32 resolution
    of the sums.  relative_to="max" (pooled block logits, which straddle zero so that tau can
    be arbitrarily close to 0): the bound is TIE_REL * max|candidate score|."""
    got = set(int(x) for x in np.asarray(got).tolist())
    ref = set(int(x) for x in np.asarray(ref).tolist())
    assert len(got) == len(ref), f"{what}: |gpu| = {len(got)} != |oracle| = {len(ref)}"
    diff = got ^ ref
    if not diff:
        return 0
    sc = np.asarray(scores, np.float64).astype(np.float32).astype(np.float64)
    pool = sc if cand is None else sc[np.asarray(cand, bool)]
    top = float(np.max(np.abs(pool))) if pool.size else 0.0
    tau = float(min(sc[list(ref)])) if ref else 0.0
    if relative_to == "tau":
        tol = TIE_REL * max(abs(tau), 1e-3 * top)
    elif relative_to == "max":
        tol = TIE_REL * top
    else:
        raise ValueError(relative_to)
    assert tol > 0.0, f"{what}: degenerate scores (all zero) cannot decide a tie"
    bad = [x for x in diff if abs(sc[x] - tau) > tol]
    assert not bad, f"{what}: {len(bad)} differing indices are not near-ties (tau={tau}, tol={tol}): {sorted(bad)[:8]}"
    return len(diff)


def oracle_full(p, Q, K, V, idx, rows=None):
    return oracle.attention(p, Q, K, V, idx, rows)
