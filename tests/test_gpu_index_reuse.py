"""Index reuse across layers of one layout (MMInference: an index estimated once per modality
layout serves the later layers and segments of that layout): the index sets and tile lists
a msa_estimate leaves in the workspace serve a later layer with other Q/K/V of the same layout
(permute -> sparse prefill -> unpermute without estimating again); that layer's output must be
the oracle's masked attention under the first layer's index sets."""
import numpy as np
import pytest

import oracle
from helpers import compare_outputs, mixed_problem, to_dev
from workload import make_inputs

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import dynamic_sparse_attention_head_b200 as msa  # noqa: E402


def _same(a, b):
    """Equal index data: arrays element by element, ragged lists (one array per row) row by row."""
    def seq(x):
        return isinstance(x, (list, tuple)) or (isinstance(x, np.ndarray) and x.dtype == object)
    if isinstance(a, dict) or isinstance(b, dict):
        return isinstance(a, dict) and isinstance(b, dict) and sorted(a) == sorted(b) and \
            all(_same(a[k], b[k]) for k in a)
    if seq(a) or seq(b):
        return len(a) == len(b) and all(_same(x, y) for x, y in zip(a, b))
    return np.array_equal(np.asarray(a), np.asarray(b))


def test_second_layer_reuses_first_layers_indices():
    p = mixed_problem()
    Q1, K1, V1 = make_inputs(p, seed=11)
    Q2, K2, V2 = make_inputs(p, seed=12)
    plan = msa.Plan(p)
    ws = plan.alloc_workspace()
    q, k, v = to_dev(Q1), to_dev(K1), to_dev(V1)
    o = torch.empty_like(q)
    plan.forward(q, k, v, ws, o)  # layer 1: estimate + attend
    torch.cuda.synchronize()
    idx1 = [plan.read_indices(h, ws) for h in range(p.Hq)]
    q2, k2, v2 = to_dev(Q2), to_dev(K2), to_dev(V2)
    o2 = torch.empty_like(q2)
    plan.permute(q2, k2, v2, ws)  # layer 2: no estimate
    plan.sparse_prefill(q2, k2, v2, ws)
    plan.unpermute(ws, o2)
    torch.cuda.synchronize()
    assert plan.device_status(ws) == 0
    for h in range(p.Hq):  # the workspace still holds layer 1's index sets
        again = plan.read_indices(h, ws)
        assert sorted(again) == sorted(idx1[h])
        for key, val in idx1[h].items():
            assert _same(again[key], val), f"head {h} {key}"
    Oref, _ = oracle.attention(p, Q2, K2, V2, idx1)
    got = o2.float().cpu().numpy()
    for h in range(p.Hq):
        compare_outputs(got[h], Oref[h], f"reuse head {h}")
