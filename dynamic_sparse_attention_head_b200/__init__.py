"""Python binding of libmsa (modality-aware permutation sparse attention, sm_100a).

Argument marshalling only: every step of the path runs in the library's CUDA kernels.
The binding takes torch CUDA tensors (bf16, last dimension 128 contiguous) and passes
their device pointers, strides and the current CUDA stream through the C ABI declared
in include/msa.h.  Importing it without the built library raises ImportError.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, List, Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmsa.so")

KINDS = {"dense": 0, "ashape": 1, "vslash": 2, "block": 3, "grid": 4, "qbound": 5, "bound2d": 6}
KIND_NAMES = {v: k for k, v in KINDS.items()}
MAX_STRIDES = 8
HEAD_PER_SEGMENT = 1  # msa_head_cfg.flags: Q-boundary index per modality segment
STATUS = {0: "ok", 1: "invalid argument", 2: "shape", 3: "alignment", 4: "workspace", 5: "unsupported",
          6: "cuda", 7: "device timeout", 8: "device bounds", 9: "state"}

_I32, _I64, _F32, _F64, _P = ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_double, ctypes.c_void_p


class HeadCfg(ctypes.Structure):
    _fields_ = [("kind", _I32), ("sink", _I32), ("local", _I32), ("k_v", _I32), ("k_s", _I32),
                ("topk_blocks", _I32), ("block_budget", _F64), ("n_strides", _I32), ("strides", _I32 * MAX_STRIDES),
                ("n_phases", _I32), ("flags", _I32), ("grid_budget", _F64)]


class Segment(ctypes.Structure):
    _fields_ = [("start", _I64), ("len", _I64), ("modality", _I32), ("_pad", _I32)]


class ProblemC(ctypes.Structure):
    _fields_ = [("L", _I64), ("Hq", _I32), ("Hkv", _I32), ("d", _I32), ("scale", _F32), ("n_segments", _I32),
                ("segments", _P), ("heads", _P)]


class Strides(ctypes.Structure):
    _fields_ = [("q_head", _I64), ("q_row", _I64), ("k_head", _I64), ("k_row", _I64), ("v_head", _I64),
                ("v_row", _I64), ("o_head", _I64), ("o_row", _I64)]


class HeadIndices(ctypes.Structure):
    _fields_ = [("stride", _I32), ("n_phases", _I32), ("phases", _P), ("n_v", (_I32 * 2) * 2),
                ("v", (_P * 2) * 2), ("n_s", _I32 * 2), ("s", _P * 2), ("blk_ptr", _P), ("blk_idx", _P),
                ("n_seg", _I32), ("seg_nv", _P), ("seg_v", _P), ("seg_ns", _P), ("seg_s", _P)]


class MsaError(RuntimeError):
    def __init__(self, fn: str, code: int, msg: str = ""):
        super().__init__(f"{fn} failed: {STATUS.get(code, code)} ({msg})")
        self.code = code


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libmsa.so is not built ({LIB_PATH}); run dynamic_sparse_attention_head_b200/build.py")
    lib = ctypes.CDLL(LIB_PATH)
    sig = {
        "msa_plan_create": ([ctypes.POINTER(ProblemC), ctypes.POINTER(_P)], _I32),
        "msa_plan_destroy": ([_P], None),
        "msa_workspace_bytes": ([_P], ctypes.c_size_t),
        "msa_workspace_bytes_indexed": ([_P], ctypes.c_size_t),
        "msa_sparse_prefill_indexed": ([_P, _P, _P, _P, _P, ctypes.POINTER(Strides), _P, ctypes.c_size_t, _P, _P],
                                       _I32),
        "msa_estimate": ([_P, _P, _P, ctypes.POINTER(Strides), _P, ctypes.c_size_t, _P], _I32),
        "msa_set_indices": ([_P, _P, _P, ctypes.c_size_t, _P], _I32),
        "msa_permute": ([_P, _P, _P, _P, ctypes.POINTER(Strides), _P, ctypes.c_size_t, _P], _I32),
        "msa_sparse_prefill": ([_P, _P, _P, _P, ctypes.POINTER(Strides), _P, ctypes.c_size_t, _P, _P], _I32),
        "msa_unpermute": ([_P, _P, ctypes.c_size_t, _P, ctypes.POINTER(Strides), _P], _I32),
        "msa_read_indices": ([_P, _P, _I32, _P, ctypes.POINTER(_I64), _P], _I32),
        "msa_read_tiles": ([_P, _P, _I32, _P, ctypes.POINTER(_I64), _P], _I32),
        "msa_tile_stats": ([_P, _P, _P, _P], _I32),
        "msa_tile_stats_heads": ([_P, _P, _P, _P], _I32),
        "msa_attention_units": ([_P, _P], _I32),
        "msa_mask_pairs": ([_P, _P, _P, _P], _I32),
        "msa_selftest_timeout": ([_P, _P, ctypes.c_uint32, _P], _I32),
        "msa_device_status": ([_P, _P, _P], _I32),
        "msa_status_string": ([_I32], ctypes.c_char_p),
        "msa_kernel_launches": ([], ctypes.c_uint64),
        "msa_vslash_estimate_static": ([_P, _P, _I64, _I64, _I64, _F32, _I32, _I32, _P, _P, _P, _P], _I32),
        "msa_weight_share": ([_P, _P, _I64, _I32, _I32, ctypes.POINTER(Strides), _F32, _P, _P, _I32, ctypes.c_double,
                              _P, _P], _I32),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    return lib


_lib = _load()
EXPORTS = ("msa_plan_create", "msa_plan_destroy", "msa_workspace_bytes", "msa_workspace_bytes_indexed",
           "msa_sparse_prefill_indexed", "msa_estimate", "msa_set_indices",
           "msa_permute", "msa_sparse_prefill", "msa_unpermute", "msa_read_indices", "msa_read_tiles",
           "msa_tile_stats", "msa_tile_stats_heads", "msa_attention_units", "msa_mask_pairs", "msa_selftest_timeout", "msa_device_status", "msa_status_string",
           "msa_kernel_launches", "msa_vslash_estimate_static", "msa_weight_share")


def kernel_launches() -> int:
    """Kernels launched by libmsa since it was loaded."""
    return int(_lib.msa_kernel_launches())


def _check(fn: str, code: int):
    if code != 0:
        raise MsaError(fn, code, _lib.msa_status_string(code).decode())


def _stream_ptr(stream=None) -> Optional[int]:
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _head_cfg(h) -> HeadCfg:
    c = HeadCfg()
    c.kind = KINDS[h.kind] if isinstance(h.kind, str) else int(h.kind)
    c.sink, c.local, c.k_v, c.k_s = int(h.sink), int(h.local), int(h.k_v), int(h.k_s)
    c.topk_blocks, c.block_budget = int(h.topk_blocks), float(h.block_budget)
    st = list(getattr(h, "strides", ()) or ())
    c.n_strides = len(st)
    for i, s in enumerate(st[:MAX_STRIDES]):
        c.strides[i] = int(s)
    c.n_phases, c.grid_budget = int(h.n_phases), float(h.grid_budget)
    c.flags = HEAD_PER_SEGMENT if getattr(h, "per_segment", False) else 0
    return c


def _strides(Q=None, K=None, V=None, O=None) -> Strides:
    s = Strides()
    for name, t in (("q", Q), ("k", K), ("v", V), ("o", O)):
        if t is None:
            continue
        assert t.dim() == 3 and t.shape[-1] == 128 and t.stride(-1) == 1, f"{name}: [H, L, 128] with d contiguous"
        setattr(s, f"{name}_head", t.stride(0))
        setattr(s, f"{name}_row", t.stride(1))
    return s


class Plan:
    """A validated problem (layout, head patterns, budgets) and its workspace size.

    `problem` needs attributes L, Hq, Hkv, d, scale, segments [(start, len, modality)]
    and heads (each with kind, sink, local, k_v, k_s, topk_blocks, block_budget, strides,
    n_phases, grid_budget).
    """

    def __init__(self, problem):
        self.problem = problem
        segs = (Segment * len(problem.segments))()
        for i, (s0, n, m) in enumerate(problem.segments):
            segs[i].start, segs[i].len, segs[i].modality = int(s0), int(n), int(m)
        heads = (HeadCfg * problem.Hq)()
        for i, h in enumerate(problem.heads):
            heads[i] = _head_cfg(h)
        pc = ProblemC(L=int(problem.L), Hq=int(problem.Hq), Hkv=int(problem.Hkv), d=int(problem.d),
                      scale=float(problem.scale), n_segments=len(problem.segments),
                      segments=ctypes.cast(segs, _P), heads=ctypes.cast(heads, _P))
        self._keep = (segs, heads)
        h = _P()
        _check("msa_plan_create", _lib.msa_plan_create(ctypes.byref(pc), ctypes.byref(h)))
        self._h = h
        self.workspace_bytes = int(_lib.msa_workspace_bytes(h))
        self.workspace_bytes_indexed = int(_lib.msa_workspace_bytes_indexed(h))

    def __del__(self):
        if getattr(self, "_h", None):
            _lib.msa_plan_destroy(self._h)
            self._h = None

    def alloc_workspace(self, indexed: bool = False):
        """Device workspace for the three-call path, or (indexed) the smaller one of the
        index-based path."""
        import torch
        n = self.workspace_bytes_indexed if indexed else self.workspace_bytes
        return torch.empty(n, dtype=torch.uint8, device="cuda")

    # ---- the four steps --------------------------------------------------------------
    def estimate(self, Q, K, ws, stream=None):
        s = _strides(Q=Q, K=K)
        _check("msa_estimate", _lib.msa_estimate(self._h, Q.data_ptr(), K.data_ptr(), ctypes.byref(s), ws.data_ptr(),
                                                 ws.numel(), _stream_ptr(stream)))

    def set_indices(self, idx: List[Dict], ws, stream=None):
        """idx[h]: dict with 'V'/'S' (vertical-slash), {'V': {a: ...}, 'S': {a: ...}} (Q-boundary),
        {'V': {(a, b): ...}, 'S': {a: ...}} (2D-boundary), 'stride'/'phases' (grid), 'T' (block)."""
        arr = (HeadIndices * self.problem.Hq)()
        keep = []

        def ptr(a):
            a = np.ascontiguousarray(np.asarray(a, np.int32))
            keep.append(a)
            return a.ctypes.data, len(a)

        for h, x in enumerate(idx):
            kind = self.problem.heads[h].kind
            hi = arr[h]
            if kind == "vslash":
                hi.v[0][0], hi.n_v[0][0] = ptr(x["V"])
                hi.s[0], hi.n_s[0] = ptr(x["S"])
            elif kind == "qbound" and getattr(self.problem.heads[h], "per_segment", False):
                nseg = len(self.problem.segments)
                vp, sp = (_P * nseg)(), (_P * nseg)()
                nv, ns = np.zeros(nseg, np.int32), np.zeros(nseg, np.int32)
                for k in range(nseg):
                    vp[k], nv[k] = ptr(x["V"][k])
                    sp[k], ns[k] = ptr(x["S"][k])
                keep += [vp, sp, nv, ns]
                hi.n_seg = nseg
                hi.seg_nv, hi.seg_ns = nv.ctypes.data, ns.ctypes.data
                hi.seg_v, hi.seg_s = ctypes.cast(vp, _P), ctypes.cast(sp, _P)
            elif kind == "qbound":
                for a, v in x["V"].items():
                    hi.v[a][0], hi.n_v[a][0] = ptr(v)
                for a, v in x["S"].items():
                    hi.s[a], hi.n_s[a] = ptr(v)
            elif kind == "bound2d":
                for (a, b), v in x["V"].items():
                    hi.v[a][b], hi.n_v[a][b] = ptr(v)
                for a, v in x["S"].items():
                    hi.s[a], hi.n_s[a] = ptr(v)
            elif kind == "grid":
                hi.stride = int(x["stride"])
                hi.phases, hi.n_phases = ptr(x["phases"])
            elif kind == "block":
                T = x["T"]
                bp = np.zeros(len(T) + 1, np.int32)
                bp[1:] = np.cumsum([len(t) for t in T])
                hi.blk_ptr, _ = ptr(bp)
                hi.blk_idx, _ = ptr(np.concatenate([np.asarray(t, np.int32) for t in T]) if len(T) else [0])
        _check("msa_set_indices", _lib.msa_set_indices(self._h, ctypes.cast(arr, _P), ws.data_ptr(), ws.numel(),
                                                       _stream_ptr(stream)))

    def permute(self, Q, K, V, ws, stream=None):
        s = _strides(Q=Q, K=K, V=V)
        _check("msa_permute", _lib.msa_permute(self._h, Q.data_ptr(), K.data_ptr(), V.data_ptr(), ctypes.byref(s),
                                               ws.data_ptr(), ws.numel(), _stream_ptr(stream)))

    def sparse_prefill(self, Q, K, V, ws, lse=None, stream=None):
        s = _strides(Q=Q, K=K, V=V)
        _check("msa_sparse_prefill",
               _lib.msa_sparse_prefill(self._h, Q.data_ptr(), K.data_ptr(), V.data_ptr(), ctypes.byref(s),
                                       ws.data_ptr(), ws.numel(), lse.data_ptr() if lse is not None else None,
                                       _stream_ptr(stream)))

    def unpermute(self, ws, O, stream=None):
        s = _strides(O=O)
        _check("msa_unpermute", _lib.msa_unpermute(self._h, ws.data_ptr(), ws.numel(), O.data_ptr(), ctypes.byref(s),
                                                   _stream_ptr(stream)))

    def sparse_prefill_indexed(self, Q, K, V, ws, O, lse=None, stream=None):
        """Permute + sparse prefill + unpermute in one call: Q rows gathered by index in the
        kernel, O written at original positions."""
        s = _strides(Q=Q, K=K, V=V, O=O)
        _check("msa_sparse_prefill_indexed",
               _lib.msa_sparse_prefill_indexed(self._h, Q.data_ptr(), K.data_ptr(), V.data_ptr(), O.data_ptr(),
                                               ctypes.byref(s), ws.data_ptr(), ws.numel(),
                                               lse.data_ptr() if lse is not None else None, _stream_ptr(stream)))

    def forward(self, Q, K, V, ws, O, lse=None, stream=None, indexed: bool = False):
        """The whole path: estimate -> permute -> sparse prefill -> unpermute, or (indexed)
        estimate -> index-based sparse prefill."""
        self.estimate(Q, K, ws, stream)
        if indexed:
            self.sparse_prefill_indexed(Q, K, V, ws, O, lse, stream)
            return
        self.permute(Q, K, V, ws, stream)
        self.sparse_prefill(Q, K, V, ws, lse, stream)
        self.unpermute(ws, O, stream)

    # ---- inspection (synchronising) --------------------------------------------------
    def _record(self, fn, head, ws, stream=None) -> np.ndarray:
        n = _I64(0)
        code = fn(self._h, ws.data_ptr(), int(head), None, ctypes.byref(n), _stream_ptr(stream))
        if code not in (0, 1):
            _check(fn.__name__, code)
        buf = np.zeros(max(1, n.value), np.int32)
        _check(fn.__name__, fn(self._h, ws.data_ptr(), int(head), buf.ctypes.data, ctypes.byref(n),
                               _stream_ptr(stream)))
        return buf[:n.value]

    def read_indices(self, head: int, ws, stream=None) -> Dict:
        r = self._record(_lib.msa_read_indices, head, ws, stream).tolist()
        i = 0

        def take(n):
            nonlocal i
            out = np.asarray(r[i:i + n], np.int64)
            i += n
            return out

        kind = KIND_NAMES[r[0]]
        stride, nph = r[1], r[2]
        i = 3
        phases = take(nph)
        v = {}
        for a in (0, 1):
            for b in (0, 1):
                n = r[i]
                i += 1
                v[(a, b)] = take(n)
        s = {}
        for a in (0, 1):
            n = r[i]
            i += 1
            s[a] = take(n)
        nb = r[i]
        i += 1
        T = None
        if kind == "block":
            ptrs = take(nb + 1)
            flat = take(int(ptrs[-1]))
            T = [flat[ptrs[b]:ptrs[b + 1]] for b in range(nb)]
        nseg = r[i]
        i += 1
        segv, segs = {}, {}
        for k in range(nseg):  # per-segment Q-boundary: each segment's vertical and slash lines
            n = r[i]
            i += 1
            segv[k] = take(n)
            n = r[i]
            i += 1
            segs[k] = take(n)
        out = {"kind": kind}
        if kind == "grid":
            out.update(stride=stride, phases=phases)
        elif kind == "vslash":
            out.update(V=v[(0, 0)], S=s[0])
        elif kind == "qbound" and nseg > 0:
            out.update(per_segment=True, V=segv, S=segs)
        elif kind == "qbound":
            out.update(V={a: v[(a, 0)] for a in (0, 1)}, S=s)
        elif kind == "bound2d":
            out.update(V=v, S=s)
        elif kind == "block":
            out["T"] = T
        return out

    def read_tiles(self, head: int, ws, stream=None) -> List[Dict]:
        """Work list of one head: per item its class, rows and tiles (source, the 128 key
        positions, and whether the tile is flagged fully allowed for every row)."""
        r = self._record(_lib.msa_read_tiles, head, ws, stream)
        n_items, i = int(r[0]), 1
        items = []
        for _ in range(n_items):
            cls, nrows = int(r[i]), int(r[i + 1])
            rows = r[i + 2:i + 2 + 128].astype(np.int64)
            i += 2 + 128
            nt = int(r[i])
            i += 1
            tiles = []
            for _ in range(nt):
                src = int(r[i])
                keys = r[i + 1:i + 1 + 128].astype(np.int64)
                i += 129
                tiles.append((src & 7, keys, bool(src & 8)))
            items.append({"cls": cls, "nrows": nrows, "rows": rows, "tiles": tiles})
        return items

    def tile_stats(self, ws, stream=None):
        t = (_I64 * 2)()
        _check("msa_tile_stats", _lib.msa_tile_stats(self._h, ws.data_ptr(), ctypes.cast(t, _P), _stream_ptr(stream)))
        return int(t[0]), int(t[1])

    def tile_stats_heads(self, ws, stream=None):
        """Executed tiles of each query head (int64 [Hq])."""
        import numpy as np
        c = np.zeros(self.problem.Hq, np.int64)
        _check("msa_tile_stats_heads", _lib.msa_tile_stats_heads(self._h, ws.data_ptr(), c.ctypes.data_as(_P),
                                                                 _stream_ptr(stream)))
        return c

    def mask_pairs(self, ws, stream=None):
        """Allowed (query, key) pairs per query head under the current masks (int64 [Hq]);
        useful FLOPs = 4 * d * sum."""
        import numpy as np
        c = np.zeros(self.problem.Hq, np.int64)
        _check("msa_mask_pairs", _lib.msa_mask_pairs(self._h, ws.data_ptr(), c.ctypes.data_as(_P), _stream_ptr(stream)))
        return c

    def attention_units(self):
        """(work units, key chunks) of msa_sparse_prefill for this plan."""
        return self.attention_work()[:2]

    def attention_work(self):
        """(work units, key chunks, unit bands) of msa_sparse_prefill for this plan."""
        t = (_I64 * 3)()
        _check("msa_attention_units", _lib.msa_attention_units(self._h, ctypes.cast(t, _P)))
        return int(t[0]), int(t[1]), int(t[2])

    def selftest_timeout(self, ws, limit_us: int = 10000, stream=None):
        """Launch a bounded wait that runs out after limit_us; device_status then reports
        MSA_ERR_TIMEOUT (7)."""
        _check("msa_selftest_timeout", _lib.msa_selftest_timeout(self._h, ws.data_ptr(), int(limit_us),
                                                                 _stream_ptr(stream)))

    def device_status(self, ws, stream=None) -> int:
        return int(_lib.msa_device_status(self._h, ws.data_ptr(), _stream_ptr(stream)))


def vslash_estimate_static(Qh, Kh, scale: float, k_v: int, k_s: int, v_out, s_out, counts_out, stream=None):
    """msa_vslash_estimate_static: vertical/slash lines of one head without any workspace.
    Qh, Kh: [L, 128] bf16 CUDA tensors; v_out [k_v], s_out [k_s], counts_out [2]: int32 CUDA
    tensors the caller allocated beforehand."""
    assert Qh.dim() == 2 and Kh.dim() == 2 and Qh.stride(1) == 1 and Kh.stride(1) == 1
    _check("msa_vslash_estimate_static",
           _lib.msa_vslash_estimate_static(Qh.data_ptr(), Kh.data_ptr(), Qh.shape[0], Qh.stride(0), Kh.stride(0),
                                           float(scale), int(k_v), int(k_s), v_out.data_ptr(), s_out.data_ptr(),
                                           counts_out.data_ptr(), _stream_ptr(stream)))


def weight_share(Q, K, scale: float, heads, rows, recall: float = 0.95, stream=None):
    """msa_weight_share: for each sample s, the fewest dense causal attention weights of query
    row rows[s] of head heads[s] whose sum reaches `recall` of the row's softmax mass.
    Q [Hq, L, 128], K [Hkv, L, 128]: bf16 CUDA tensors; heads, rows: int32 CUDA tensors [n].
    Returns an int64 CUDA tensor [n] (the share of row i is count / (i + 1))."""
    import torch
    assert Q.dim() == 3 and K.dim() == 3 and Q.stride(2) == 1 and K.stride(2) == 1
    n = int(rows.numel())
    out = torch.empty(n, dtype=torch.int64, device=Q.device)
    _check("msa_weight_share",
           _lib.msa_weight_share(Q.data_ptr(), K.data_ptr(), Q.shape[1], Q.shape[0], K.shape[0],
                                 ctypes.byref(_strides(Q, K)), float(scale), heads.data_ptr(), rows.data_ptr(), n,
                                 float(recall), out.data_ptr(), _stream_ptr(stream)))
    return out


def executed_flops(tiles: int) -> int:
    """FLOPs of the executed 128x128 tiles (QK^T and PV, d = 128)."""
    return 4 * 128 * 128 * 128 * int(tiles)
