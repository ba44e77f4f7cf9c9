"""CPU oracle for modality-aware permutation sparse prefill attention.

TEST INFRASTRUCTURE ONLY: imported by tests/, by ``__graft_entry__.smoke()`` and
by the CPU-baseline leg of ``bench.py``.  The product path never imports it.

The numeric core is plain C (``oracle.c``, fp64 accumulation).  This module
orchestrates the estimation steps per head kind in the order the pages give
them (MInference 1.0 "Approach"; MMInference "key machinery" / "core discovery"):

1. pick the estimation rows: the last 64 queries (of the sequence, or of one
   modality for video-aware heads);
2. reduce their causal softmax to vertical (per key) and slash (per offset) sums;
3. select top-k lines / blocks / grid phases;
4. evaluate the token-level mask and run masked softmax attention.

Where the pages leave a step open the reading used here is stated in the
docstring of the function that takes it.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from typing import Dict, List, Optional

import numpy as np

from workload import TEXT, VIDEO, Problem

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None
LAST_Q = 64
BLOCK = 64
GRID_BAND = 64
KIND_ID = {"dense": 0, "ashape": 1, "vslash": 2, "block": 3, "grid": 4, "qbound": 5, "bound2d": 6}
K_QSEG = 7  # Q-boundary estimated per modality segment

_P = ctypes.c_void_p
_I64 = ctypes.c_int64


def build(force: bool = False) -> str:
    src = os.path.join(_HERE, "oracle.c")
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(src):
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", _LIB_PATH, src, "-lm"])
    return _LIB_PATH


class _Mask(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("_pad", ctypes.c_int32), ("sink", _I64), ("local", _I64),
                ("vcol", _P * 4), ("slash", _P * 2), ("gmark", _P), ("modality", _P), ("rank", _P),
                ("blocksel", _P), ("nb", _I64), ("segid", _P), ("vseg", _P), ("sseg", _P)]


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        lib.orc_lastq_sums.argtypes = [_P, _P, _I64, ctypes.c_int, ctypes.c_float, _P, ctypes.c_int, _P, _P, _P, _P]
        lib.orc_topk.argtypes = [_P, _P, _I64, _I64, _P]
        lib.orc_topk.restype = _I64
        lib.orc_pool64.argtypes = [_P, _I64, ctypes.c_int, _P]
        lib.orc_block_topk.argtypes = [_P, _P, _I64, ctypes.c_int, ctypes.c_float, _P, _I64, _P, _P]
        lib.orc_mask_rows.argtypes = [ctypes.POINTER(_Mask), _I64, _P, _I64, _P]
        lib.orc_mask_count.argtypes = [ctypes.POINTER(_Mask), _P, _I64, _P]
        lib.orc_attention.argtypes = [_P, _P, _P, _I64, ctypes.c_int, ctypes.c_float, ctypes.POINTER(_Mask),
                                      _P, _I64, _P, _P]
        lib.orc_attention_permuted.argtypes = [_P, _P, _P, _P, _I64, _P, _I64, ctypes.c_int, ctypes.c_float,
                                               ctypes.POINTER(_Mask), _P, _P]
        _lib = lib
    return _lib


def _c(a: np.ndarray, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


# --------------------------------------------------------------------------------------
# primitives
# --------------------------------------------------------------------------------------
def lastq_sums(Qh, Kh, scale, rows, rcoord=None, kcoord=None):
    """Vertical sums v[j] and slash sums s[o] of the causal softmax of `rows` (C core)."""
    lib = _load()
    Qh = _c(Qh, np.uint16)
    Kh = _c(Kh, np.uint16)
    L, d = Kh.shape
    rows = _c(rows, np.int64)
    rcoord = _c(rows if rcoord is None else rcoord, np.int64)
    kcoord = _c(np.arange(L) if kcoord is None else kcoord, np.int64)
    v = np.zeros(L, np.float64)
    s = np.zeros(L, np.float64)
    lib.orc_lastq_sums(Qh.ctypes.data, Kh.ctypes.data, L, d, scale, rows.ctypes.data, len(rows),
                       rcoord.ctypes.data, kcoord.ctypes.data, v.ctypes.data, s.ctypes.data)
    return v, s


def topk(score: np.ndarray, k: int, cand: Optional[np.ndarray] = None) -> np.ndarray:
    """Top-k by (fp32 score desc, index asc), returned sorted ascending."""
    lib = _load()
    score = _c(score, np.float64)
    n = len(score)
    out = np.zeros(max(1, min(k, n)), np.int64)
    cp = None
    if cand is not None:
        cand = _c(cand, np.uint8)
        cp = cand.ctypes.data
    c = lib.orc_topk(score.ctypes.data, cp, n, k, out.ctypes.data)
    return out[:c].copy()


def pool64(Xh) -> np.ndarray:
    lib = _load()
    Xh = _c(Xh, np.uint16)
    L, d = Xh.shape
    out = np.zeros((L // BLOCK, d), np.float64)
    lib.orc_pool64(Xh.ctypes.data, L, d, out.ctypes.data)
    return out


def budget_scale(k: int, n: int, L: int) -> int:
    """Budget k rescaled to a modality holding n of the L tokens: max(1, round(k n / L)), halves up."""
    if n <= 0:
        return 0
    return max(1, (2 * k * n + L) // (2 * L))


def grid_phase_count(head, stride: int) -> int:
    """Phases kept for a grid head: explicit count, else max(1, floor(budget * stride / 2))."""
    n = head.n_phases if head.n_phases > 0 else max(1, int(math.floor(head.grid_budget * stride / 2.0)))
    return min(n, stride)


def block_row_k(head, nb: int) -> np.ndarray:
    """Blocks kept per query-block row b: fixed top-k, or ceil(budget (b + 1))."""
    b = np.arange(nb)
    if head.topk_blocks > 0:
        k = np.full(nb, head.topk_blocks, np.int64)
    else:
        k = np.array([int(math.ceil(head.block_budget * (x + 1))) for x in b], np.int64)
    return np.minimum(np.maximum(k, 1), b + 1)


def last_rows(positions: np.ndarray, n: int = LAST_Q) -> np.ndarray:
    return positions[-n:] if len(positions) > n else positions


# --------------------------------------------------------------------------------------
# estimation per head kind
# --------------------------------------------------------------------------------------
def estimate_head(p: Problem, h: int, Q: np.ndarray, K: np.ndarray) -> Dict:
    """Online sparse index of q-head h (uint16 bf16 inputs, head-major)."""
    head = p.heads[h]
    kvh = h // (p.Hq // p.Hkv)
    Qh, Kh = Q[h], K[kvh]
    L = p.L
    mod = p.modality()
    out: Dict = {"kind": head.kind}
    if head.kind in ("dense", "ashape"):
        return out

    if head.kind == "vslash":
        # MInference 1.0 "Approach": the last 64 queries' attention reduced to
        # vertical and slash lines, each taken top-k.
        rows = last_rows(np.arange(L))
        v, s = lastq_sums(Qh, Kh, p.scale, rows)
        hi = rows.max()
        cand = (np.arange(L) <= hi).astype(np.uint8)
        out.update(V=topk(v, head.k_v, cand), S=topk(s, head.k_s, cand), v=v, s=s)
        return out

    if head.kind == "block":
        # MInference 1.0 "Approach": mean-pooled 64-token blocks of Q and K; top-k
        # key blocks per query block from the pooled attention.
        lib = _load()
        Qb, Kb = pool64(Qh), pool64(Kh)
        nb = L // BLOCK
        kk = block_row_k(head, nb)
        kmax = int(kk.max())
        sel = np.zeros((nb, kmax), np.int64)
        cnt = np.zeros(nb, np.int64)
        lib.orc_block_topk(Qb.ctypes.data, Kb.ctypes.data, nb, p.d, p.scale, kk.ctypes.data, kmax,
                           sel.ctypes.data, cnt.ctypes.data)
        out.update(T=[sel[b, :cnt[b]].copy() for b in range(nb)], Qbar=Qb, Kbar=Kb)
        return out

    if head.kind == "grid":
        return _estimate_grid(p, head, Qh, Kh, mod, out)

    if head.kind == "qbound" and head.per_segment:
        # MMInference review page, "core discovery" (the last 64 queries of each modality
        # segment), read literally: every segment k gets its own vertical-slash index from its
        # own last 64 queries (all of them if it is shorter), over all causal keys, and that
        # index serves the queries of segment k only.
        out.update(per_segment=True, V={}, S={}, v={}, s={})
        for k, (st, n, _) in enumerate(p.segments):
            rows = last_rows(np.arange(st, st + n))
            v, s = lastq_sums(Qh, Kh, p.scale, rows)
            cand = (np.arange(L) <= rows.max()).astype(np.uint8)
            out["V"][k] = topk(v, head.k_v, cand)
            out["S"][k] = topk(s, head.k_s, cand)
            out["v"][k], out["s"][k] = v, s
        return out

    if head.kind == "qbound":
        # MMInference Algorithm 2 (Q-boundary): the query axis is split at modality
        # boundaries; each query modality gets its own vertical-slash index from the
        # last 64 queries of that modality, over all causal keys.
        out.update(V={}, S={}, v={}, s={})
        for a in (TEXT, VIDEO):
            pos = np.nonzero(mod == a)[0]
            if len(pos) == 0:
                continue
            rows = last_rows(pos)
            v, s = lastq_sums(Qh, Kh, p.scale, rows)
            cand = (np.arange(L) <= rows.max()).astype(np.uint8)
            out["V"][a] = topk(v, head.k_v, cand)
            out["S"][a] = topk(s, head.k_s, cand)
            out["v"][a], out["s"][a] = v, s
        return out

    if head.kind == "bound2d":
        # MMInference Algorithm 3 (2D-boundary): both axes split by modality; each
        # (query modality a, key modality b) pair is its own region.  Intra-modality
        # slash lines live in within-modality ranks, so one index extrapolates across
        # text-interrupted video; cross-modality pairs keep vertical lines only.
        rank = _ranks(mod)
        out.update(V={}, S={}, v={}, s={})
        n_of = {a: int((mod == a).sum()) for a in (TEXT, VIDEO)}
        for a in (TEXT, VIDEO):
            pos = np.nonzero(mod == a)[0]
            if len(pos) == 0:
                continue
            rows = last_rows(pos)
            kco = np.where(mod == a, rank, -1)
            v, s = lastq_sums(Qh, Kh, p.scale, rows, rcoord=rank[rows], kcoord=kco)
            causal = np.arange(L) <= rows.max()
            for b in (TEXT, VIDEO):
                if n_of[b] == 0:
                    continue
                cand = (causal & (mod == b)).astype(np.uint8)
                out["V"][(a, b)] = topk(v, budget_scale(head.k_v, n_of[b], L), cand)
            scand = (np.arange(L) <= rank[rows.max()]).astype(np.uint8)
            out["S"][a] = topk(s, budget_scale(head.k_s, n_of[a], L), scand)
            out["v"][a], out["s"][a] = v, s
        return out
    raise ValueError(head.kind)


def _ranks(mod: np.ndarray) -> np.ndarray:
    rank = np.zeros(len(mod), np.int64)
    for a in (TEXT, VIDEO):
        idx = np.nonzero(mod == a)[0]
        rank[idx] = np.arange(len(idx))
    return rank


def grid_scores(p: Problem, v: np.ndarray, stride: int) -> np.ndarray:
    """score(stride, phase) = mean of v over video keys whose in-segment offset mod stride == phase."""
    mod = p.modality()
    off = np.arange(p.L) - p.seg_start()
    vid = mod == VIDEO
    ph = off[vid] % stride
    sums = np.bincount(ph, weights=v[vid], minlength=stride)
    cnt = np.bincount(ph, minlength=stride)
    return np.where(cnt > 0, sums / np.maximum(cnt, 1), 0.0)


def _estimate_grid(p, head, Qh, Kh, mod, out):
    """MMInference Algorithm 1 (grid head), "key machinery": the stride and phase of
    the grid are searched online from an approximate attention matrix built from
    the last 64 queries.  Reading: the last 64 *video* queries; the column sums v
    are averaged per (stride, phase) over video keys; the stride whose best phase
    scores highest wins (ties: smaller stride); its top n_p phases are kept
    (ties: smaller phase)."""
    vid = np.nonzero(mod == VIDEO)[0]
    rows = last_rows(vid)
    v, _ = lastq_sums(Qh, Kh, p.scale, rows)
    best_s, best_val, best_sc = None, None, None
    for st in sorted(head.strides):
        sc = grid_scores(p, v, st)
        val = np.float32(sc.astype(np.float32).max())
        if best_val is None or val > best_val:
            best_s, best_val, best_sc = st, val, sc
    n_p = grid_phase_count(head, best_s)
    out.update(stride=int(best_s), phases=topk(best_sc, n_p), v=v, scores=best_sc)
    return out


def estimate(p: Problem, Q: np.ndarray, K: np.ndarray) -> List[Dict]:
    return [estimate_head(p, h, Q, K) for h in range(p.Hq)]


# --------------------------------------------------------------------------------------
# masks and attention
# --------------------------------------------------------------------------------------
def grid_marks(p: Problem, stride: int, phases) -> np.ndarray:
    mod = p.modality()
    off = np.arange(p.L) - p.seg_start()
    return ((mod == VIDEO) & np.isin(off % stride, np.asarray(phases))).astype(np.uint8)


class MaskArrays:
    """Owns the numpy arrays an orc_mask points into."""

    def __init__(self, p: Problem, h: int, idx: Dict):
        head = p.heads[h]
        L = p.L
        self.keep = []
        m = _Mask()
        m.kind = KIND_ID[head.kind]
        m.sink = head.sink
        m.local = head.local
        mod = _c(p.modality(), np.uint8)
        self.keep.append(mod)
        m.modality = mod.ctypes.data
        zero = np.zeros(L, np.uint8)
        self.keep.append(zero)
        for t in range(4):
            m.vcol[t] = zero.ctypes.data
        for t in range(2):
            m.slash[t] = zero.ctypes.data
        m.gmark = zero.ctypes.data
        rank = _ranks(mod)
        self.keep.append(rank)
        m.rank = rank.ctypes.data

        def marks(ix):
            a = np.zeros(L, np.uint8)
            a[np.asarray(ix, np.int64)] = 1
            self.keep.append(a)
            return a.ctypes.data

        k = head.kind
        if k == "vslash":
            m.vcol[0] = marks(idx["V"])
            m.slash[0] = marks(idx["S"])
        elif k == "qbound" and head.per_segment:
            m.kind = K_QSEG
            segid = np.zeros(L, np.int32)
            for kk, (st, n, _) in enumerate(p.segments):
                segid[st:st + n] = kk
            self.keep.append(segid)
            m.segid = segid.ctypes.data
            nseg = len(p.segments)
            vptr = (_P * nseg)(*[marks(idx["V"][kk]) for kk in range(nseg)])
            sptr = (_P * nseg)(*[marks(idx["S"][kk]) for kk in range(nseg)])
            self.keep += [vptr, sptr]
            m.vseg = ctypes.cast(vptr, _P)
            m.sseg = ctypes.cast(sptr, _P)
        elif k == "qbound":
            for a, ix in idx["V"].items():
                m.vcol[a * 2] = marks(ix)
            for a, ix in idx["S"].items():
                m.slash[a] = marks(ix)
        elif k == "bound2d":
            for (a, b), ix in idx["V"].items():
                m.vcol[a * 2 + b] = marks(ix)
            for a, ix in idx["S"].items():
                m.slash[a] = marks(ix)
        elif k == "grid":
            g = grid_marks(p, idx["stride"], idx["phases"])
            self.keep.append(g)
            m.gmark = g.ctypes.data
            m.local = head.local if head.local > 0 else GRID_BAND
        elif k == "block":
            nb = L // BLOCK
            sel = np.zeros((nb, nb), np.uint8)
            for b, ks in enumerate(idx["T"]):
                sel[b, np.asarray(ks, np.int64)] = 1
            self.keep.append(sel)
            m.blocksel = sel.ctypes.data
            m.nb = nb
        self.mask = m


def mask_rows(p: Problem, h: int, idx: Dict, rows) -> np.ndarray:
    lib = _load()
    ma = MaskArrays(p, h, idx)
    rows = _c(rows, np.int64)
    out = np.zeros((len(rows), p.L), np.uint8)
    lib.orc_mask_rows(ctypes.byref(ma.mask), p.L, rows.ctypes.data, len(rows), out.ctypes.data)
    return out


def mask_count(p: Problem, h: int, idx: Dict, rows=None) -> np.ndarray:
    lib = _load()
    ma = MaskArrays(p, h, idx)
    rows = _c(np.arange(p.L) if rows is None else rows, np.int64)
    out = np.zeros(len(rows), np.int64)
    lib.orc_mask_count(ctypes.byref(ma.mask), rows.ctypes.data, len(rows), out.ctypes.data)
    return out


def attention_head(p: Problem, h: int, Q, K, V, idx: Dict, rows=None):
    """Masked attention of q-head h on the given rows: (O [n, d] fp32, lse [n] fp32)."""
    lib = _load()
    kvh = h // (p.Hq // p.Hkv)
    Qh, Kh, Vh = _c(Q[h], np.uint16), _c(K[kvh], np.uint16), _c(V[kvh], np.uint16)
    rows = _c(np.arange(p.L) if rows is None else rows, np.int64)
    O = np.zeros((len(rows), p.d), np.float32)
    lse = np.zeros(len(rows), np.float32)
    ma = MaskArrays(p, h, idx)
    lib.orc_attention(Qh.ctypes.data, Kh.ctypes.data, Vh.ctypes.data, p.L, p.d, p.scale, ctypes.byref(ma.mask),
                      rows.ctypes.data, len(rows), O.ctypes.data, lse.ctypes.data)
    return O, lse


def attention(p: Problem, Q, K, V, idx: List[Dict], rows=None):
    outs = [attention_head(p, h, Q, K, V, idx[h], rows) for h in range(p.Hq)]
    return np.stack([o for o, _ in outs]), np.stack([l for _, l in outs])


# --------------------------------------------------------------------------------------
# permutation (MMInference review page, "key machinery" and "core discovery")
# --------------------------------------------------------------------------------------
def _front(first: np.ndarray) -> np.ndarray:
    """Stable partition of positions 0..L-1: those with first[t] true, then the rest, each
    in ascending order."""
    first = np.asarray(first, bool)
    return np.concatenate([np.nonzero(first)[0], np.nonzero(~first)[0]]).astype(np.int64)


def permutation(p: Problem, h: int, idx: Dict):
    """The row and column permutation of q-head h, as arrays of original positions in permuted
    order (qperm[r] = original query position of permuted row r; likewise kperm for keys).

    Readings (the pages state the goal, contiguous selected entries, not an ordering):
      grid (Algorithm 1): queries and keys on the selected grid lines first, then the others;
      Q-boundary (Algorithm 2): queries grouped by modality (text, then video), keys unchanged;
        estimated per segment, queries grouped by segment (the original order), keys unchanged;
      2D-boundary (Algorithm 3): queries and keys grouped by modality;
      vertical-slash: keys on the vertical lines first (the lines gathered), queries unchanged;
      other kinds: identity.
    Every group keeps ascending original order."""
    kind = p.heads[h].kind
    L = p.L
    ident = np.arange(L, dtype=np.int64)
    mod = p.modality()
    if kind == "grid":
        g = grid_marks(p, idx["stride"], idx["phases"]).astype(bool)
        return _front(g), _front(g)
    if kind == "qbound" and p.heads[h].per_segment:
        return ident, ident
    if kind == "qbound":
        return _front(mod == TEXT), ident
    if kind == "bound2d":
        return _front(mod == TEXT), _front(mod == TEXT)
    if kind == "vslash":
        v = np.zeros(L, bool)
        v[np.asarray(idx["V"], np.int64)] = True
        return ident, _front(v)
    return ident, ident


def attention_permuted(p: Problem, h: int, Q, K, V, idx: Dict, qperm, kperm):
    """Permute -> attend -> unpermute for q-head h: gather Q rows by qperm and K/V rows by
    kperm, run the masked attention in permuted coordinates with the mask evaluated through
    the original positions, and scatter the output rows back to their original positions.
    Returns (O [L, d] fp32, lse [L] fp32) in original order."""
    lib = _load()
    kvh = h // (p.Hq // p.Hkv)
    qperm = _c(qperm, np.int64)
    kperm = _c(kperm, np.int64)
    Qp = _c(np.asarray(Q[h])[qperm], np.uint16)
    Kp = _c(np.asarray(K[kvh])[kperm], np.uint16)
    Vp = _c(np.asarray(V[kvh])[kperm], np.uint16)
    Op = np.zeros((len(qperm), p.d), np.float32)
    lp = np.zeros(len(qperm), np.float32)
    ma = MaskArrays(p, h, idx)
    lib.orc_attention_permuted(Qp.ctypes.data, Kp.ctypes.data, Vp.ctypes.data, qperm.ctypes.data, len(qperm),
                               kperm.ctypes.data, len(kperm), p.d, p.scale, ctypes.byref(ma.mask),
                               Op.ctypes.data, lp.ctypes.data)
    O = np.zeros((p.L, p.d), np.float32)
    lse = np.full(p.L, -np.inf, np.float32)
    O[qperm] = Op
    lse[qperm] = lp
    return O, lse


# --------------------------------------------------------------------------------------
# attention analysis (MMInference summary page, attention-sparsity analysis)
# --------------------------------------------------------------------------------------
def weight_share(Q, K, scale: float, head: int, row: int, group: int, recall: float = 0.95):
    """The fewest dense causal attention weights of query `row` of `head` whose sum reaches
    `recall` of the row's softmax mass (the pages' statistic: the share of the weights that 95 %
    recall needs).  Logits as everywhere in the oracle: fp64 dot products rounded to fp32, times
    the fp32 scale; weights exp(x - max), the descending sort and the running sum in fp64.
    Returns (count, running sum of the sorted weights divided by their total)."""
    from workload import bf16_to_f32
    q = bf16_to_f32(np.asarray(Q[head][row])).astype(np.float64)
    k = bf16_to_f32(np.asarray(K[head // group][: row + 1])).astype(np.float64)
    x = (k @ q).astype(np.float32) * np.float32(scale)
    w = np.exp(x.astype(np.float64) - float(x.max()))
    w = np.sort(w)[::-1]
    cum = np.cumsum(w) / w.sum()
    count = int(np.searchsorted(cum, recall, side="left")) + 1
    return min(count, row + 1), cum
