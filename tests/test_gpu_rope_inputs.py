"""GPU parity on rotary-structured inputs (attention that depends on the query-key offset, so the
estimated lines cluster near the diagonal and many tiles are skipped): index sets against the
oracle's (near-tie rule) and outputs against the oracle on every row, for every head kind, on a
video/text layout with a ragged end; and the executed tiles against those of the same layout on
unstructured inputs."""
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


def _layout():
    segs = [(0, 300, TEXT), (300, 2048, VIDEO), (2348, 400, TEXT), (2748, 1024, VIDEO), (3772, 324, TEXT)]
    heads = [Head("vslash", k_v=64, k_s=160), Head("qbound", k_v=48, k_s=120), Head("bound2d", k_v=48, k_s=120),
             Head("grid", strides=(64,), grid_budget=0.1), Head("block", topk_blocks=4),
             Head("ashape", sink=64, local=256), Head("vslash", k_v=16, k_s=400), Head("qbound", k_v=100, k_s=60)]
    return Problem(L=4096, Hq=8, Hkv=2, segments=segs, heads=heads, frame_stride=64, name="rope-4k")


def _forward(p, Q, K, V):
    plan = msa.Plan(p)
    ws = plan.alloc_workspace()
    q, k, v = to_dev(Q), to_dev(K), to_dev(V)
    o = torch.empty_like(q)
    lse = torch.empty((p.Hq, p.L), dtype=torch.float32, device="cuda")
    plan.forward(q, k, v, ws, o, lse=lse)
    torch.cuda.synchronize()
    assert plan.device_status(ws) == 0
    idx = [plan.read_indices(h, ws) for h in range(p.Hq)]
    return plan, ws, idx, o.float().cpu().numpy(), lse.cpu().numpy()


def test_rope_inputs_match_oracle_on_all_rows():
    p = _layout()
    Q, K, V = make_inputs(p, seed=9, inputs="rope")
    plan, ws, idx, O, lse = _forward(p, Q, K, V)
    for h in range(p.Hq):
        _check_head(p, h, idx[h], oracle.estimate_head(p, h, Q, K))
    Oref, lref = oracle.attention(p, Q, K, V, idx)
    for h in range(p.Hq):
        compare_outputs(O[h], Oref[h], f"rope head {h}")
        fin = np.isfinite(lref[h])
        assert np.array_equal(fin, np.isfinite(lse[h]))
        np.testing.assert_allclose(lse[h][fin], lref[h][fin], atol=2e-3, rtol=1e-3)
    pairs = plan.mask_pairs(ws)
    for h in range(p.Hq):
        assert int(pairs[h]) == int(oracle.mask_count(p, h, idx[h]).sum()), f"head {h}"


def test_rope_slash_lines_cluster_and_fewer_tiles_run():
    p = _layout()
    Qr, Kr, Vr = make_inputs(p, seed=9, inputs="rope")
    Qi, Ki, Vi = make_inputs(p, seed=9)
    plan_r, ws_r, idx_r, _, _ = _forward(p, Qr, Kr, Vr)
    plan_i, ws_i, idx_i, _, _ = _forward(p, Qi, Ki, Vi)
    # the lines of the vertical-slash head cluster: many more short slash offsets and late
    # vertical keys than on the unstructured draw (oracle on this layout: 62 against 4 offsets
    # below 128, 59 against 9 vertical keys in the last 512)
    S_r, S_i = np.asarray(idx_r[0]["S"]), np.asarray(idx_i[0]["S"])
    V_r, V_i = np.asarray(idx_r[0]["V"]), np.asarray(idx_i[0]["V"])
    assert (S_r < 128).sum() >= 4 * max(1, (S_i < 128).sum())
    assert (V_r >= p.L - 512).sum() >= 3 * max(1, (V_i >= p.L - 512).sum())
    assert plan_r.tile_stats(ws_r)[0] < plan_i.tile_stats(ws_i)[0]
