"""GPU parity of the per-segment Q-boundary option (each modality segment's last 64 queries
estimate the index that serves that segment; MMInference review page, "core discovery", read
literally): index sets against the oracle's (near-tie rule), outputs against the oracle run with
the GPU's index sets on every row, host-provided indices, the index-based path and chunked keys
against the three-call path, on layouts with short segments and a multi-image document."""
import dataclasses

import numpy as np
import pytest

import oracle
from helpers import compare_outputs, to_dev
from test_gpu_estimate import _check_head
from workload import TEXT, VIDEO, Head, Problem, make_inputs, mixed_image_text

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import dynamic_sparse_attention_head_b200 as msa  # noqa: E402


def _layout():
    """Segments of both modalities, two of them shorter than 64 tokens (all their rows estimate),
    a ragged end (L % 128 == 64)."""
    segs = [(0, 200, TEXT), (200, 384, VIDEO), (584, 40, TEXT), (624, 300, VIDEO), (924, 20, TEXT),
            (944, 208, VIDEO), (1152, 64, TEXT)]
    heads = [Head("qbound", k_v=30, k_s=90, per_segment=True), Head("qbound", k_v=5, k_s=200, per_segment=True),
             Head("vslash", k_v=40, k_s=60), Head("qbound", k_v=30, k_s=90)]
    return Problem(L=1216, Hq=4, Hkv=2, segments=segs, heads=heads, frame_stride=96, name="per-segment")


def _run(p, Q, K, V, indexed=False, idx=None):
    plan = msa.Plan(p)
    ws = plan.alloc_workspace(indexed=indexed)
    q, k, v = to_dev(Q), to_dev(K), to_dev(V)
    o = torch.zeros_like(q)
    lse = torch.full((p.Hq, p.L), float("nan"), device="cuda", dtype=torch.float32)
    if idx is None:
        plan.estimate(q, k, ws)
    else:
        plan.set_indices(idx, ws)
    if indexed:
        plan.sparse_prefill_indexed(q, k, v, ws, o, lse=lse)
    else:
        plan.permute(q, k, v, ws)
        plan.sparse_prefill(q, k, v, ws, lse=lse)
        plan.unpermute(ws, o)
    torch.cuda.synchronize()
    assert plan.device_status(ws) == 0
    got = [plan.read_indices(h, ws) for h in range(p.Hq)]
    return got, o.float().cpu().numpy(), lse.cpu().numpy()


def test_per_segment_matches_oracle_on_all_rows():
    p = _layout()
    Q, K, V = make_inputs(p, seed=17)
    idx, O, lse = _run(p, Q, K, V)
    for h in range(p.Hq):
        ref = oracle.estimate_head(p, h, Q, K)
        if p.heads[h].per_segment:
            assert idx[h].get("per_segment") and sorted(idx[h]["V"]) == list(range(len(p.segments)))
        _check_head(p, h, idx[h], ref)
    Oref, lref = oracle.attention(p, Q, K, V, idx)
    for h in range(p.Hq):
        compare_outputs(O[h], Oref[h], f"head {h}")
        fin = np.isfinite(lref[h])
        assert np.array_equal(fin, np.isfinite(lse[h]))
        np.testing.assert_allclose(lse[h][fin], lref[h][fin], atol=2e-3, rtol=1e-3)
    # the allowed pairs the kernels' mask counts equal the oracle's
    plan = msa.Plan(p)
    ws = plan.alloc_workspace()
    plan.set_indices(idx, ws)
    pairs = plan.mask_pairs(ws)
    for h in range(p.Hq):
        assert int(pairs[h]) == int(oracle.mask_count(p, h, idx[h]).sum()), f"head {h}"


def test_per_segment_host_indices_indexed_path_and_chunks(monkeypatch):
    """The oracle's own index sets set from the host; the index-based path and chunked keys give
    the three-call path's output bit for bit (chunks: up to the rounding of the carried state)."""
    p = _layout()
    Q, K, V = make_inputs(p, seed=23)
    ref = oracle.estimate(p, Q, K)
    idx, O, lse = _run(p, Q, K, V, idx=ref)
    for h in range(p.Hq):
        if p.heads[h].per_segment:
            for k in range(len(p.segments)):
                assert idx[h]["V"][k].tolist() == ref[h]["V"][k].tolist()
                assert idx[h]["S"][k].tolist() == ref[h]["S"][k].tolist()
    Oref, _ = oracle.attention(p, Q, K, V, ref)
    for h in range(p.Hq):
        compare_outputs(O[h], Oref[h], f"host indices head {h}")
    _, Oi, li = _run(p, Q, K, V, indexed=True, idx=ref)
    assert np.array_equal(Oi, O) and np.array_equal(li, lse, equal_nan=True)
    monkeypatch.setenv("MSA_ATTN_CHUNK_KEYS", "256")
    assert msa.Plan(p).attention_units()[1] > 1
    _, Oc, lc = _run(p, Q, K, V, idx=ref)
    np.testing.assert_allclose(Oc, O, atol=1e-2, rtol=0)


def test_per_segment_multi_image_document():
    """Many short segments (144-token images between 16-200-token text runs): one class and one
    estimate per segment."""
    base = mixed_image_text(L=3072, image=144, width=12, text=(16, 200), Hq=4, Hkv=2, k_v=60, k_s=200,
                            name="mixed-per-segment")
    heads = [Head("qbound", k_v=60, k_s=200, per_segment=True), Head("bound2d", k_v=60, k_s=200),
             Head("qbound", k_v=20, k_s=400, per_segment=True), Head("grid", strides=(12,), grid_budget=0.1)]
    p = dataclasses.replace(base, heads=heads)
    assert len(p.segments) > 20
    Q, K, V = make_inputs(p, seed=4)
    idx, O, _ = _run(p, Q, K, V)
    for h in range(p.Hq):
        _check_head(p, h, idx[h], oracle.estimate_head(p, h, Q, K))
    Oref, _ = oracle.attention(p, Q, K, V, idx)
    for h in range(p.Hq):
        compare_outputs(O[h], Oref[h], f"{p.name} head {h}")
