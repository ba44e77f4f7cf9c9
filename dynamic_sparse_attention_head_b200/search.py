"""Attention recall and the per-head pattern search.

MMInference ("Modality-Aware Sparse Attention Search", Algorithm 4) assigns each head its sparse
pattern offline: on a calibration sample, among configurations that fit a FLOPs budget measured
on the kernel, the one whose mask keeps the most attention mass.  The pages' attention-recall
analysis measures that mass as the fraction of the full softmax kept by the mask.

Recall of a mask for query row i is the softmax mass of row i inside the mask,
    recall_i = sum_{j in mask(i)} exp(s_ij) / sum_{j <= i} exp(s_ij) = exp(lse_mask_i - lse_dense_i),
so it comes exactly from the log-sum-exp rows that msa_sparse_prefill writes for the masked
layer and for the same layer with every head dense (an empty row has recall 0).  The cost of a
configuration is what the kernel executes: 4 * 128^3 FLOPs per executed 128 x 128 tile.

Reading (the pages give the search only in outline): a candidate is one head configuration
(kind and parameters); every candidate is run on the calibration layer with all query heads
set to it (the index estimate of each head runs as usual); for each head the search keeps the
candidates whose executed FLOPs are at most `budget` times the head's dense causal FLOPs and
picks the one with the highest recall (the cheaper one on equal recall); a head no candidate fits
gets the cheapest candidate.
"""
import copy
from typing import Dict, List, Sequence

import numpy as np

from . import Plan, executed_flops, weight_share


def _with_heads(problem, heads, name):
    p = copy.copy(problem)
    p.heads = list(heads)
    p.name = name
    return p


def layer_lse(problem, Q, K, V, stream=None):
    """Run one layer (estimate, permute, prefill, unpermute) and return (lse [Hq, L] as a numpy
    array, executed tiles per query head).  Q, K, V: bf16 CUDA tensors [Hq|Hkv, L, 128]."""
    import torch
    plan = Plan(problem)
    ws = plan.alloc_workspace()
    O = torch.empty_like(Q)
    lse = torch.empty((problem.Hq, problem.L), dtype=torch.float32, device=Q.device)
    plan.forward(Q, K, V, ws, O, lse=lse, stream=stream)
    torch.cuda.synchronize()
    if plan.device_status(ws) != 0:
        raise RuntimeError("device status after the calibration layer")
    tiles = [sum(len(it["tiles"]) for it in plan.read_tiles(h, ws)) for h in range(problem.Hq)]
    return lse.cpu().numpy(), np.asarray(tiles, np.int64)


def recall_from_lse(lse_mask: np.ndarray, lse_dense: np.ndarray) -> np.ndarray:
    """Per-row recall exp(lse_mask - lse_dense), 0 for rows the mask leaves empty."""
    r = np.exp(np.where(np.isfinite(lse_mask), lse_mask - lse_dense, -np.inf))
    return np.clip(r, 0.0, 1.0)


def head_recall(problem, Q, K, V, heads, lse_dense=None) -> Dict[str, np.ndarray]:
    """Recall (mean over query rows) and executed FLOPs of every query head of `problem` with the
    head configurations `heads` (one per query head)."""
    if lse_dense is None:
        lse_dense = dense_lse(problem, Q, K, V)
    lse, tiles = layer_lse(_with_heads(problem, heads, problem.name + "-mask"), Q, K, V)
    rec = recall_from_lse(lse, lse_dense)
    return {"recall": rec.mean(axis=1), "flops": np.array([executed_flops(int(t)) for t in tiles], np.int64)}


def dense_lse(problem, Q, K, V) -> np.ndarray:
    dense = copy.copy(problem.heads[0])
    dense.kind = "dense"
    return layer_lse(_with_heads(problem, [dense] * problem.Hq, problem.name + "-dense"), Q, K, V)[0]


def dense_head_flops(problem) -> int:
    """Causal FLOPs of one dense head, counted as the kernel does (4 * 128^3 per 128 x 128 tile;
    a ragged last query tile counts its 64-key units)."""
    L = problem.L
    nq = (L + 127) // 128
    return executed_flops(sum(((min(L, 128 * (i + 1)) - 1) // 64 + 2) // 2 for i in range(nq)))


def choose(recall: np.ndarray, flops: np.ndarray, budget_flops: float) -> List[int]:
    """recall, flops: [candidates, heads].  Per head the candidate of highest recall among those
    within the budget (the cheaper on equal recall); the cheapest when none fits."""
    C, H = recall.shape
    pick = []
    for h in range(H):
        fit = [c for c in range(C) if flops[c, h] <= budget_flops]
        if fit:
            pick.append(max(fit, key=lambda c: (recall[c, h], -flops[c, h], -c)))
        else:
            pick.append(min(range(C), key=lambda c: (flops[c, h], c)))
    return pick


def search(problem, Q, K, V, candidates: Sequence, budget: float):
    """The per-head search on one calibration layer.  candidates: head configurations (objects
    with the attributes of a head configuration, see msa_head_cfg); budget: executed FLOPs per
    head as a fraction of its dense causal FLOPs.  Returns (chosen configuration per head, table
    with the recall and FLOPs of every candidate on every head)."""
    lse_dense = dense_lse(problem, Q, K, V)
    rec, fl = [], []
    for cand in candidates:
        r = head_recall(problem, Q, K, V, [cand] * problem.Hq, lse_dense=lse_dense)
        rec.append(r["recall"])
        fl.append(r["flops"])
    rec, fl = np.stack(rec), np.stack(fl)
    pick = choose(rec, fl, budget * dense_head_flops(problem))
    return [candidates[c] for c in pick], {"recall": rec, "flops": fl, "pick": pick,
                                           "dense_head_flops": dense_head_flops(problem)}


def stratified_rows(L: int, n: int, seed: int = 0) -> np.ndarray:
    """n query rows spread over [0, L): one seeded row in each of n equal strata."""
    rng = np.random.default_rng(seed)
    edges = np.linspace(0, L, n + 1).astype(np.int64)
    return np.array([rng.integers(lo, hi) for lo, hi in zip(edges[:-1], edges[1:]) if hi > lo], np.int64)


def weight_share_stats(problem, Q, K, rows_per_head: int = 16, recall: float = 0.95, seed: int = 0) -> Dict:
    """The pages' second sparsity statistic (MMInference summary page, attention analysis: the
    share of the dense attention weights that `recall` of the mass needs; 1.79 % for video-language
    models against 5.78 % for language models at 95 %), on stratified rows of every query head:
    per head the mean over its rows of count / (row + 1), and the mean over heads of each kind.
    The counts come from msa_weight_share on the device."""
    import torch
    rows = stratified_rows(problem.L, rows_per_head, seed)
    heads = np.repeat(np.arange(problem.Hq), len(rows)).astype(np.int32)
    rr = np.tile(rows, problem.Hq).astype(np.int32)
    counts = weight_share(Q, K, problem.scale, torch.from_numpy(heads).to(Q.device), torch.from_numpy(rr).to(Q.device),
                          recall).cpu().numpy()
    if np.any(counts < 0):
        raise RuntimeError("weight share: sample out of range")
    share = (counts / (rr.astype(np.float64) + 1.0)).reshape(problem.Hq, len(rows))
    per_head = share.mean(axis=1)
    kinds = {}
    for h, hd in enumerate(problem.heads):
        kinds.setdefault(hd.kind, []).append(per_head[h])
    return {"recall": recall, "rows_per_head": int(len(rows)), "mean_share": float(per_head.mean()),
            "per_kind": {k: float(np.mean(v)) for k, v in kinds.items()}, "per_head": per_head}
