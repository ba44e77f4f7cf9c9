"""Seeded synthetic workloads for modality-aware permutation sparse prefill.

This module is shared by the CUDA path's tests/bench and by the CPU oracle's
tests.  It holds no part of the attention method: it describes problems
(sequence layout, head patterns, budgets) and draws their bf16 inputs with a
counter-based generator (``gen.c``), so both sides see bit-identical tensors.

Workloads follow the long-context VLM/LLM prefill settings the MMInference
(ICML 2025) and MInference 1.0 (NeurIPS 2024) pages describe: LLaMA-3-8B-shaped
text layers (32 q / 8 kv heads), Qwen2-7B-shaped video layers (28 q / 4 kv
heads), video frames as fixed-stride token runs interleaved with text.  The
real model activations are not available, so Q/K/V are N(0,1) in bf16 with an
optional grid bias (+2u on keys at frame-stride positions, u a shared unit
vector) that plants the grid structure those pages describe.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass, field
from typing import List, Optional, Sequence, Tuple

import numpy as np

TEXT, VIDEO = 0, 1
KINDS = ("dense", "ashape", "vslash", "block", "grid", "qbound", "bound2d")

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libworkload.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile gen.c into libworkload.so (host code only)."""
    src = os.path.join(_HERE, "gen.c")
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(src):
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", _LIB_PATH, src, "-lm"])
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        lib.wl_normals_f64.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int64]
        lib.wl_fill_bf16.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_uint64,
                                     ctypes.c_uint64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_float]
        lib.wl_fill_rope_bf16.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_uint64,
                                          ctypes.c_uint64, ctypes.c_float, ctypes.c_void_p, ctypes.c_float,
                                          ctypes.c_double, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_float]
        _lib = lib
    return _lib


# --------------------------------------------------------------------------------------
# problem description
# --------------------------------------------------------------------------------------
@dataclass
class Head:
    kind: str
    sink: int = 0
    local: int = 0
    k_v: int = 0
    k_s: int = 0
    topk_blocks: int = 0
    block_budget: float = 0.0
    strides: Tuple[int, ...] = ()
    n_phases: int = 0
    grid_budget: float = 0.0
    # Q-boundary heads: estimate from the last 64 queries of each modality segment and apply each
    # index to its own segment (instead of one index per modality)
    per_segment: bool = False

    def __post_init__(self):
        assert self.kind in KINDS, self.kind
        assert not self.per_segment or self.kind == "qbound", "per-segment estimation is a Q-boundary option"


@dataclass
class Problem:
    L: int
    Hq: int
    Hkv: int
    segments: List[Tuple[int, int, int]]  # (start, len, modality)
    heads: List[Head]
    d: int = 128
    name: str = ""
    frame_stride: int = 0  # stride of the planted grid bias (0: none)
    scale: float = field(default=0.0)

    def __post_init__(self):
        if not self.scale:
            self.scale = float(np.float32(1.0 / math.sqrt(self.d)))
        assert len(self.heads) == self.Hq
        pos = 0
        for (s, n, m) in self.segments:
            assert s == pos and n > 0 and m in (TEXT, VIDEO), (s, n, m)
            pos += n
        assert pos == self.L, (pos, self.L)

    def modality(self) -> np.ndarray:
        mod = np.zeros(self.L, np.uint8)
        for (s, n, m) in self.segments:
            mod[s:s + n] = m
        return mod

    def seg_start(self) -> np.ndarray:
        ss = np.zeros(self.L, np.int64)
        for (s, n, m) in self.segments:
            ss[s:s + n] = s
        return ss


def frame_stride_rows(p: Problem, stride: int, phase: int = 0) -> np.ndarray:
    """Video positions t whose in-segment offset (t - segment start) mod stride == phase."""
    mod = p.modality()
    off = np.arange(p.L) - p.seg_start()
    return (mod == VIDEO) & (off % stride == phase)


# --------------------------------------------------------------------------------------
# inputs
# --------------------------------------------------------------------------------------
Q_STREAM, K_STREAM, V_STREAM, U_STREAM = 1000, 2000, 3000, 7


def unit_vector(seed: int, d: int = 128, stream: int = U_STREAM) -> np.ndarray:
    lib = _load()
    u = np.empty(d, np.float64)
    lib.wl_normals_f64(u.ctypes.data, d, seed, stream, 0)
    return (u / np.linalg.norm(u)).astype(np.float32)


def _fill(rows: int, d: int, seed: int, stream: int, bias=None, bias_rows=None, scale=0.0, rope=None) -> np.ndarray:
    lib = _load()
    out = np.empty((rows, d), np.uint16)
    bptr = bias.ctypes.data if bias is not None else None
    rptr = bias_rows.ctypes.data if bias_rows is not None else None
    if rope is None:
        lib.wl_fill_bf16(out.ctypes.data, rows, d, seed, stream, bptr, rptr, scale)
    else:
        shared, shared_scale, base = rope
        lib.wl_fill_rope_bf16(out.ctypes.data, rows, d, seed, stream, 1.0, shared.ctypes.data, shared_scale, base,
                              bptr, rptr, scale)
    return out


# Position structure of the rotary variant: every Q and K row carries ROPE_SHARED x w (w a seeded
# unit vector) before the rotary embedding of its position (base ROPE_BASE, the value of the
# Qwen2 family), so q_i . k_j gains ROPE_SHARED^2 x w^T R(j - i) w, largest at offset 0 and
# falling with distance (mean logits at the 1/sqrt(128) scale: ~20 at offset 0, ~15 at 100, ~9 at
# 1000, ~4 at 4000).  The scale is set so that at 128K tokens a query needs about 2 % of its keys'
# weights for 95 % of its attention mass, near the share the MMInference summary page reports for
# VLM heads (1.79 %).
ROPE_SHARED = 15.0
ROPE_BASE = 1.0e6


def make_inputs(p: Problem, seed: int = 0, bias: float = 2.0, plant_queries: bool = False, inputs: str = "iid",
                q_heads: Optional[Sequence[int]] = None, kv_heads: Optional[Sequence[int]] = None):
    """Q [Hq,L,d], K/V [Hkv,L,d] as bf16 bit patterns (np.uint16), head-major.

    K rows at frame-stride positions get ``bias * u`` when p.frame_stride > 0.
    With plant_queries, the last 64 video queries get the same shift, so the
    planted phase-0 grid dominates the last-64-query estimate.
    inputs="rope": Q and K rows also carry the shared component of ROPE_SHARED and are rotated
    by the rotary embedding of their position (V is unchanged), so that attention depends on the
    offset between query and key as in a rotary model.
    q_heads / kv_heads: draw only these heads of a larger layer (their streams keep the layer's
    head numbers, so a shard's inputs equal the same heads of the whole layer's).
    """
    if inputs not in ("iid", "rope"):
        raise ValueError(f"inputs must be 'iid' or 'rope', not {inputs!r}")
    d = p.d
    u = unit_vector(seed, d)
    rope = (unit_vector(seed, d, U_STREAM + 1), ROPE_SHARED, ROPE_BASE) if inputs == "rope" else None
    krows = None
    if p.frame_stride and bias:
        krows = frame_stride_rows(p, p.frame_stride).astype(np.uint8)
    qrows = None
    if plant_queries:
        vid = np.nonzero(p.modality() == VIDEO)[0]
        qrows = np.zeros(p.L, np.uint8)
        qrows[vid[-64:]] = 1
    qs = list(range(p.Hq)) if q_heads is None else list(q_heads)
    ks = list(range(p.Hkv)) if kv_heads is None else list(kv_heads)
    Q = np.empty((len(qs), p.L, d), np.uint16)
    K = np.empty((len(ks), p.L, d), np.uint16)
    V = np.empty((len(ks), p.L, d), np.uint16)
    for i, h in enumerate(qs):
        Q[i] = _fill(p.L, d, seed, Q_STREAM + h, u if qrows is not None else None, qrows, bias, rope)
    for i, h in enumerate(ks):
        K[i] = _fill(p.L, d, seed, K_STREAM + h, u if krows is not None else None, krows, bias, rope)
        V[i] = _fill(p.L, d, seed, V_STREAM + h, None, None, 0.0)
    return Q, K, V


def shard_kv_heads(p: Problem, rank: int, world: int) -> Tuple[Problem, range, range]:
    """Rank `rank`'s share of one layer split by KV-head group over `world` GPUs: KV heads
    [rank Hkv/world, (rank + 1) Hkv/world) and the query heads that read them (query head h reads
    KV head h // (Hq / Hkv)).  Heads are independent in every step of the path, so the shards
    need no exchange; returns (sub-problem, query heads, KV heads) in the full layer's numbering."""
    if world < 1 or not 0 <= rank < world or p.Hkv % world:
        raise ValueError(f"{p.Hkv} KV heads do not split over {world} ranks")
    nkv = p.Hkv // world
    nq = p.Hq // world
    qh = range(rank * nq, (rank + 1) * nq)
    kvh = range(rank * nkv, (rank + 1) * nkv)
    sub = Problem(L=p.L, Hq=nq, Hkv=nkv, segments=list(p.segments), heads=[p.heads[h] for h in qh], d=p.d,
                  name=f"{p.name}[kv {kvh.start}-{kvh.stop - 1}]", frame_stride=p.frame_stride, scale=p.scale)
    return sub, qh, kvh


def bf16_to_f32(x: np.ndarray) -> np.ndarray:
    return (x.astype(np.uint32) << 16).view(np.float32)


# --------------------------------------------------------------------------------------
# the five workloads (sizes and head splits as the benchmark configurations state them)
# --------------------------------------------------------------------------------------
def _assign(Hq: int, kinds: Sequence[Head]) -> List[Head]:
    """Heads split evenly across the listed patterns: head h takes pattern h mod len(kinds)."""
    return [kinds[h % len(kinds)] for h in range(Hq)]


def grid_single_head(L: int = 4096, text: int = 512, stride: int = 224, budget: float = 0.10) -> Problem:
    """1 layer, 1 head, d=128: text run then video frames of `stride` tokens; grid head."""
    nf = (L - text) // stride
    assert text + nf * stride == L
    segs = [(0, text, TEXT), (text, nf * stride, VIDEO)]
    heads = [Head("grid", strides=(stride,), grid_budget=budget)]
    return Problem(L=L, Hq=1, Hkv=1, segments=segs, heads=heads, frame_stride=stride,
                   name=f"grid-1head-L{L}")


def llama3_8b_text(L: int = 32768, sink: int = 128, local: int = 1024, k_v: int = 1000, k_s: int = 6096,
                   topk: int = 100, Hq: int = 32, Hkv: int = 8) -> Problem:
    """LLaMA-3-8B-shaped layer, text only; heads split across A-shape, vertical-slash, block-sparse."""
    kinds = [Head("ashape", sink=sink, local=local), Head("vslash", k_v=k_v, k_s=k_s),
             Head("block", topk_blocks=topk)]
    return Problem(L=L, Hq=Hq, Hkv=Hkv, segments=[(0, L, TEXT)], heads=_assign(Hq, kinds),
                   name=f"llama3-8b-text-L{L}")


def qwen2_7b_video(frames_per_run: int = 198, stride: int = 210, texts: Sequence[int] = (2048, 2048, 2236),
                   k_v: int = 1000, k_s: int = 6096, grid_budget: float = 0.10, Hq: int = 28, Hkv: int = 4,
                   name: str = "") -> Problem:
    """Qwen2-7B-shaped layer: video runs of frames interleaved with text runs; four head kinds."""
    segs, pos = [], 0
    runs = frames_per_run if isinstance(frames_per_run, (list, tuple)) else [frames_per_run] * len(texts)
    for nf, nt in zip(runs, texts):
        segs.append((pos, nf * stride, VIDEO)); pos += nf * stride
        segs.append((pos, nt, TEXT)); pos += nt
    kinds = [Head("grid", strides=(stride,), grid_budget=grid_budget), Head("qbound", k_v=k_v, k_s=k_s),
             Head("bound2d", k_v=k_v, k_s=k_s), Head("vslash", k_v=k_v, k_s=k_s)]
    return Problem(L=pos, Hq=Hq, Hkv=Hkv, segments=segs, heads=_assign(Hq, kinds), frame_stride=stride,
                   name=name or f"qwen2-7b-video-L{pos}")


def qwen2_7b_video_128k() -> Problem:
    """L = 131072: V(198x210) T(2048) V(198x210) T(2048) V(198x210) T(2236)."""
    return qwen2_7b_video(name="qwen2-7b-video-128k")


def qwen2_7b_video_literal() -> Problem:
    """The literal 64-frame layout (22+21+21 frames of 210 tokens, three 2048-token texts), L = 19584."""
    return qwen2_7b_video(frames_per_run=[22, 21, 21], texts=(2048, 2048, 2048), name="qwen2-7b-video-64f")


def mixed_image_text(L: int = 65536, image: int = 576, width: int = 24, text: Tuple[int, int] = (32, 640),
                     k_v: int = 1000, k_s: int = 6096, grid_budget: float = 0.10, Hq: int = 28, Hkv: int = 4,
                     seed: int = 0, name: str = "") -> Problem:
    """A multi-image document: images of `image` patch tokens (rows of `width` tokens) alternate
    with text runs of seeded random length in [text[0], text[1]], the last run filling up to L;
    many short segments of both modalities stress the Q- and 2D-boundary heads (row-class and
    modality-grouped tiles cut at every segment edge).  Head kinds Q-boundary, 2D-boundary,
    vertical-slash and grid (stride = image row width)."""
    rng = np.random.default_rng(seed)
    segs, pos = [], 0
    while True:
        if pos + image + text[0] > L:
            break
        segs.append((pos, image, VIDEO)); pos += image
        n = int(rng.integers(text[0], text[1] + 1))
        n = min(n, L - pos) if L - pos - n < image + text[0] else n
        segs.append((pos, n, TEXT)); pos += n
    if pos < L:
        if segs and segs[-1][2] == TEXT:
            s0, n0, _ = segs.pop()
            segs.append((s0, n0 + (L - pos), TEXT))
        else:
            segs.append((pos, L - pos, TEXT))
    kinds = [Head("qbound", k_v=k_v, k_s=k_s), Head("bound2d", k_v=k_v, k_s=k_s), Head("vslash", k_v=k_v, k_s=k_s),
             Head("grid", strides=(width,), grid_budget=grid_budget)]
    return Problem(L=L, Hq=Hq, Hkv=Hkv, segments=segs, heads=_assign(Hq, kinds), frame_stride=width,
                   name=name or f"mixed-image-text-L{L}")


def longvila_1m(L: int = 1048576, stride: int = 256, text: int = 512, grid_budget: float = 0.05,
                k_v: int = 1000, k_s: int = 6096, Hq: int = 28, Hkv: int = 4) -> Problem:
    """LongVILA-1M-like layer: video frames of `stride` tokens then one trailing text query."""
    nf = (L - text) // stride
    assert nf * stride + text == L
    segs = [(0, nf * stride, VIDEO), (nf * stride, text, TEXT)]
    kinds = [Head("grid", strides=(stride,), grid_budget=grid_budget), Head("vslash", k_v=k_v, k_s=k_s)]
    return Problem(L=L, Hq=Hq, Hkv=Hkv, segments=segs, heads=_assign(Hq, kinds), frame_stride=stride,
                   name=f"longvila-L{L}")


def sweep_layer(L: int, budget: Optional[float], Hq: int = 32, Hkv: int = 8) -> Problem:
    """The LLaMA-3-8B-shaped layer at length L with one block budget b (None = dense).

    b maps to each pattern as: block-sparse k_row = ceil(b (r+1)); A-shape local =
    b L / 2 - 128 rounded to a multiple of 64 (at least 64, sink 128); vertical-slash
    (k_v, k_s) = round(x (1000, 6096)) with x = b L / 13192.
    """
    if budget is None:
        return Problem(L=L, Hq=Hq, Hkv=Hkv, segments=[(0, L, TEXT)], heads=[Head("dense")] * Hq,
                       name=f"sweep-dense-L{L}")
    local = max(64, int(round((budget * L / 2 - 128) / 64.0)) * 64)
    x = budget * L / 13192.0
    kinds = [Head("ashape", sink=128, local=local),
             Head("vslash", k_v=max(1, int(round(1000 * x))), k_s=max(1, int(round(6096 * x)))),
             Head("block", block_budget=budget)]
    return Problem(L=L, Hq=Hq, Hkv=Hkv, segments=[(0, L, TEXT)], heads=_assign(Hq, kinds),
                   name=f"sweep-b{int(round(budget * 100))}-L{L}")


SWEEP_LENGTHS = (8192, 32768, 131072, 524288, 1048576)
SWEEP_BUDGETS = (0.02, 0.05, 0.10, 0.25)
