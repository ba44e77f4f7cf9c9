"""Estimation row sets whose coordinates are far apart: the last 64 text queries of a document
of short text runs between long video runs span thousands of positions, so the sweep's second
pass adds them to the slash ring in its general (non-consecutive) path with a ring of several
thousand entries; index sets against the oracle's (near-tie rule) and outputs against the oracle
on every row."""
import numpy as np
import pytest

import oracle
from helpers import compare_outputs, to_dev
from test_gpu_estimate import _check_head
from workload import TEXT, VIDEO, Head, Problem, make_inputs

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import dynamic_sparse_attention_head_b200 as msa  # noqa: E402


def _layout(text_len, video_len, n, tail=0):
    segs, t = [], 0
    for i in range(n):
        segs.append((t, text_len, TEXT))
        t += text_len
        segs.append((t, video_len, VIDEO))
        t += video_len
    if tail:
        segs.append((t, tail, TEXT))
        t += tail
    return segs, t


def test_text_rows_spread_over_thousands_of_positions():
    # 8-token text runs between 504-token video runs: the last 64 text rows lie in the last eight
    # runs, spread over ~3.6K positions
    segs, L = _layout(8, 504, 12)
    heads = [Head("qbound", k_v=40, k_s=120), Head("vslash", k_v=40, k_s=120), Head("bound2d", k_v=40, k_s=120),
             Head("qbound", k_v=10, k_s=300)]
    p = Problem(L=L, Hq=4, Hkv=2, segments=segs, heads=heads, frame_stride=50, name="wide-text")
    text_rows = np.nonzero(p.modality() == TEXT)[0][-64:]
    assert text_rows[-1] - text_rows[0] > 3000
    Q, K, V = make_inputs(p, seed=12)
    plan = msa.Plan(p)
    ws = plan.alloc_workspace()
    q, k, v = to_dev(Q), to_dev(K), to_dev(V)
    o = torch.empty_like(q)
    plan.forward(q, k, v, ws, o)
    torch.cuda.synchronize()
    assert plan.device_status(ws) == 0
    idx = [plan.read_indices(h, ws) for h in range(p.Hq)]
    for h in range(p.Hq):
        _check_head(p, h, idx[h], oracle.estimate_head(p, h, Q, K))
    Oref, _ = oracle.attention(p, Q, K, V, idx)
    O = o.float().cpu().numpy()
    for h in range(p.Hq):
        compare_outputs(O[h], Oref[h], f"wide head {h}")
    # the same launch twice gives the same lines (fixed summation order in the general path)
    plan.estimate(q, k, ws)
    torch.cuda.synchronize()
    again = [plan.read_indices(h, ws) for h in range(p.Hq)]
    for h in (0, 3):
        for a in idx[h]["S"]:
            assert idx[h]["S"][a].tolist() == again[h]["S"][a].tolist()

