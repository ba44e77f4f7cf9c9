"""GPU parity of msa_weight_share (the fewest dense attention weights of a query row whose sum
reaches a given recall; MMInference summary page, attention analysis) against the oracle's fp64
computation on the same rows.  The GPU takes its logits in fp32, so a count may differ from the
oracle's where the oracle's running sum passes the target within rounding: a count is accepted
if the oracle's sorted running sum reaches the recall at it and not one weight earlier, both
within 1e-5 relative."""
import math

import numpy as np
import pytest

import oracle
from helpers import to_dev
from workload import TEXT, VIDEO, Head, Problem, make_inputs

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import dynamic_sparse_attention_head_b200 as msa  # noqa: E402

TOL = 1e-5


def _check(count, cum, recall, what):
    assert count >= 1, what
    assert cum[count - 1] >= recall * (1 - TOL), f"{what}: {count} weights reach only {cum[count - 1]}"
    if count > 1:
        assert cum[count - 2] < recall * (1 + TOL), f"{what}: {count - 1} weights already reach {cum[count - 2]}"


@pytest.mark.parametrize("recall", [0.95, 0.5])
def test_weight_share_matches_oracle_on_sampled_rows(recall):
    segs = [(0, 256, TEXT), (256, 1536, VIDEO), (1792, 256, TEXT)]
    p = Problem(L=2048, Hq=4, Hkv=2, segments=segs, heads=[Head("dense")] * 4, frame_stride=96)
    Q, K, _ = make_inputs(p, seed=21)
    rng = np.random.default_rng(5)
    heads, rows = [], []
    for h in range(p.Hq):
        for r in [0, 1, 63, p.L - 1] + sorted(rng.choice(p.L, 12, replace=False).tolist()):
            heads.append(h)
            rows.append(r)
    q, k = to_dev(Q), to_dev(K)
    hd = torch.tensor(heads, dtype=torch.int32, device="cuda")
    rw = torch.tensor(rows, dtype=torch.int32, device="cuda")
    got = msa.weight_share(q, k, p.scale, hd, rw, recall).cpu().numpy()
    for h, r, c in zip(heads, rows, got):
        ref, cum = oracle.weight_share(Q, K, p.scale, h, r, p.Hq // p.Hkv, recall)
        _check(int(c), cum, recall, f"head {h} row {r} (gpu {c}, oracle {ref})")
        assert abs(int(c) - ref) <= 2


def test_weight_share_planted_rows_and_bad_samples():
    L = 512
    Qf = np.zeros((2, L, 128), np.float32)
    Kf = np.zeros((1, L, 128), np.float32)
    Qf[:, :, 0] = 1.0
    Kf[0, 100, 0] = 128.0  # one dominant key for every row from 100 on
    Q = (np.ascontiguousarray(Qf).view(np.uint32) >> 16).astype(np.uint16)
    K = (np.ascontiguousarray(Kf).view(np.uint32) >> 16).astype(np.uint16)
    scale = float(np.float32(1.0 / math.sqrt(128)))
    q, k = to_dev(Q), to_dev(K)
    hd = torch.tensor([0, 1, 0, 0, 2, 0], dtype=torch.int32, device="cuda")
    rw = torch.tensor([99, 99, 100, 511, 5, L], dtype=torch.int32, device="cuda")
    got = msa.weight_share(q, k, scale, hd, rw, 0.95).cpu().tolist()
    assert got[0] == got[1] == math.ceil(0.95 * 100)  # uniform rows before the dominant key
    assert got[2] == 1 and got[3] == 1
    assert got[4] == -1 and got[5] == -1  # head or row out of range
