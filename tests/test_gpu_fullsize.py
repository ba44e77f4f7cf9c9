"""Parity at the benchmark configurations' full sizes, through the same C-ABI calls the bench
times: index sets against the oracle's (near-tie rule) on heads the oracle estimates in
seconds, and outputs on sampled rows (segment edges, estimation rows, seeded random rows)
against the oracle run with the GPU's index sets."""
import numpy as np
import pytest

import oracle
from helpers import compare_outputs, near_tie_ok, to_dev
from test_gpu_estimate import _check_head
import workload
from workload import make_inputs

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import dynamic_sparse_attention_head_b200 as msa  # noqa: E402


def sample_rows(p, n_random, seed=0):
    """Segment edges, some of the last 64 queries of the sequence and of the video, and seeded
    uniformly random rows."""
    rng = np.random.default_rng(seed)
    rows = set()
    for (s, n, _m) in p.segments:
        rows.update([s, s + 1, s + n - 2, s + n - 1])
    rows.update(rng.choice(np.arange(p.L - 64, p.L), size=8, replace=False).tolist())
    vid = np.nonzero(p.modality() == workload.VIDEO)[0]
    if len(vid):
        rows.update(rng.choice(vid[-64:], size=min(8, len(vid[-64:])), replace=False).tolist())
    rows.update(rng.choice(p.L, size=n_random, replace=False).tolist())
    return np.array(sorted(r for r in rows if 0 <= r < p.L))


def run(p, seed=0):
    Q, K, V = make_inputs(p, seed=seed)
    plan = msa.Plan(p)
    ws = plan.alloc_workspace()
    q, k, v = to_dev(Q), to_dev(K), to_dev(V)
    o = torch.empty_like(q)
    plan.forward(q, k, v, ws, o)
    torch.cuda.synchronize()
    assert plan.device_status(ws) == 0
    idx = [plan.read_indices(h, ws) for h in range(p.Hq)]
    return Q, K, V, idx, o, plan, ws


def check_rows(p, Q, K, V, idx, o, heads, rows):
    for h in heads:
        ref, _ = oracle.attention_head(p, h, Q, K, V, idx[h], rows)
        got = o[h, torch.as_tensor(rows, device=o.device)].float().cpu().numpy()
        compare_outputs(got, ref, f"{p.name} head {h}")


def one_head_per_kind(p):
    seen = {}
    for h, hd in enumerate(p.heads):
        seen.setdefault(hd.kind, h)
    return sorted(seen.values())


def test_grid_single_head_4k():
    p = workload.grid_single_head()
    Q, K, V, idx, o, _, _ = run(p)
    ref = oracle.estimate(p, Q, K)
    _check_head(p, 0, idx[0], ref[0])
    Oref, _ = oracle.attention(p, Q, K, V, idx)
    compare_outputs(o.float().cpu().numpy()[0], Oref[0], "grid 4k")


def test_llama3_8b_text_32k():
    p = workload.llama3_8b_text(L=32768)
    Q, K, V, idx, o, _, _ = run(p)
    for h in range(p.Hq):  # every head's index set
        _check_head(p, h, idx[h], oracle.estimate_head(p, h, Q, K))
    check_rows(p, Q, K, V, idx, o, range(p.Hq), sample_rows(p, 48))


def test_qwen2_7b_video_128k():
    p = workload.qwen2_7b_video_128k()
    Q, K, V, idx, o, _, _ = run(p)
    for h in one_head_per_kind(p):
        _check_head(p, h, idx[h], oracle.estimate_head(p, h, Q, K))
    check_rows(p, Q, K, V, idx, o, range(p.Hq), sample_rows(p, 12))


def test_qwen2_7b_video_literal_64_frames():
    p = workload.qwen2_7b_video_literal()
    Q, K, V, idx, o, _, _ = run(p)
    for h in range(p.Hq):
        _check_head(p, h, idx[h], oracle.estimate_head(p, h, Q, K))
    check_rows(p, Q, K, V, idx, o, range(p.Hq), sample_rows(p, 24))


def test_longvila_1m():
    p = workload.longvila_1m()
    Q, K, V, idx, o, plan, ws = run(p)
    for h in one_head_per_kind(p):
        _check_head(p, h, idx[h], oracle.estimate_head(p, h, Q, K))
    rows = sample_rows(p, 2)
    rng = np.random.default_rng(1)
    few = np.sort(rng.choice(rows, size=6, replace=False))
    check_rows(p, Q, K, V, idx, o, range(p.Hq), few)
    tiles, _ = plan.tile_stats(ws)
    assert msa.executed_flops(tiles) < 2 * p.d * p.L * (p.L + 1) * p.Hq


@pytest.mark.parametrize("budget", workload.SWEEP_BUDGETS + (None,))
def test_sweep_8k(budget):
    p = workload.sweep_layer(8192, budget)
    Q, K, V, idx, o, plan, ws = run(p)
    for h in one_head_per_kind(p):
        _check_head(p, h, idx[h], oracle.estimate_head(p, h, Q, K))
    check_rows(p, Q, K, V, idx, o, range(p.Hq), sample_rows(p, 32))
    if budget is None:
        tiles, items = plan.tile_stats(ws)
        nq = p.L // 128
        assert tiles == p.Hq * sum(i + 1 for i in range(nq))  # dense: every causal 128x128 tile
