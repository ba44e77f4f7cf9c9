"""Recall measured from the kernels' log-sum-exp rows (against the dense causal softmax mass
inside the oracle's mask, in fp64), and the per-head pattern search on a calibration layer with
planted structure: keys at frame-stride positions of the video share a strong direction with
every query, so a large part of the attention mass sits on those key columns, which a grid mask
keeps through its phases."""
import numpy as np
import pytest

import oracle
import workload
from workload import Head, make_inputs

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from dynamic_sparse_attention_head_b200 import search  # noqa: E402


def _bf16(x32):
    u = np.ascontiguousarray(x32, np.float32).view(np.uint32)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def calibration_layer(a=8.0):
    p = workload.grid_single_head(L=4096, text=512, stride=224, budget=0.10)
    p = workload.Problem(L=p.L, Hq=4, Hkv=1, segments=p.segments, heads=[p.heads[0]] * 4, frame_stride=0,
                         name="calibration")
    Q, K, V = make_inputs(p, seed=5, bias=0.0)
    u = workload.unit_vector(5, p.d).astype(np.float32)
    q = workload.bf16_to_f32(Q) + a * u
    k = workload.bf16_to_f32(K)
    rows = workload.frame_stride_rows(p, 224).astype(bool)
    k[:, rows] += a * u
    dev = lambda x: torch.from_numpy(x).view(torch.bfloat16).cuda()
    return p, dev(_bf16(q)), dev(_bf16(k)), dev(V)


def test_dense_recall_is_one():
    p, q, k, v = calibration_layer()
    r = search.head_recall(p, q, k, v, [Head("dense")] * p.Hq)
    np.testing.assert_allclose(r["recall"], 1.0, atol=2e-3)
    assert np.all(r["flops"] == search.dense_head_flops(p))


def _oracle_recall(p, q, k, cand):
    """Mean over rows of the dense causal softmax mass inside the oracle's mask (fp64)."""
    qh = q.view(torch.int16).cpu().numpy().view(np.uint16)
    kh = k.view(torch.int16).cpu().numpy().view(np.uint16)
    one = workload.Problem(L=p.L, Hq=1, Hkv=1, segments=p.segments, heads=[cand], frame_stride=0, name="one")
    qf = workload.bf16_to_f32(qh)[0].astype(np.float64)
    kf = workload.bf16_to_f32(kh)[0].astype(np.float64)
    s = np.where(np.tril(np.ones((p.L, p.L), bool)), qf @ kf.T * np.float64(p.scale), -np.inf)
    prob = np.exp(s - s.max(1, keepdims=True))
    prob /= prob.sum(1, keepdims=True)
    idx = oracle.estimate(one, qh[:1], kh)
    mask = oracle.mask_rows(one, 0, idx[0], np.arange(p.L)).astype(bool)
    return float((prob * mask).sum(1).mean())


CANDIDATES = [Head("ashape", sink=64, local=384), Head("grid", strides=(224,), grid_budget=0.10),
              Head("vslash", k_v=64, k_s=128)]


def test_search_recall_matches_oracle_and_picks_grid():
    p, q, k, v = calibration_layer()
    chosen, table = search.search(p, q, k, v, CANDIDATES, budget=0.5)
    rec = table["recall"]
    assert np.all((rec >= 0) & (rec <= 1 + 1e-6))
    for c, cand in enumerate(CANDIDATES):  # every query head shares the one KV head and its bias
        ref = _oracle_recall(p, q[:1], k, cand)
        np.testing.assert_allclose(rec[c, 0], ref, atol=5e-3, err_msg=cand.kind)
    # the planted key columns hold most of the mass a mask can keep: grid keeps them with its
    # phases, and wins on every head
    assert np.all(rec[1] > rec[0] + 0.1) and np.all(rec[1] > rec[2] + 0.1), rec
    assert all(c.kind == "grid" for c in chosen), [c.kind for c in chosen]
    assert np.all(table["flops"][1] <= 0.5 * table["dense_head_flops"])
