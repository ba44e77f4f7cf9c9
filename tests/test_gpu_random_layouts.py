"""Seeded random small layers through the whole path against the oracle: segment layouts (one
to six runs of text and video of random lengths), GQA group sizes, head kinds and budgets drawn
at random.  Per layer: the device's index sets against the oracle's (near-tie rule), the output
and lse against the oracle's masked attention under the device's index sets, the device's count
of allowed pairs against the oracle's masks (exact), and the index-based path bit-identical to
the three-call path.  Every third layer runs with its keys cut into small chunks (the
long-sequence path); the Q-boundary heads of odd-numbered layers estimate per segment."""
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

N_CASES = 48


def random_problem(seed: int) -> Problem:
    rng = np.random.default_rng(1000 + seed)
    L = 64 * int(rng.integers(1, 33))  # 64 .. 2048
    nseg = int(rng.integers(1, 7))
    cuts = np.sort(rng.choice(np.arange(1, L), size=nseg - 1, replace=False)) if nseg > 1 else np.array([], int)
    bounds = [0] + [int(c) for c in cuts] + [L]
    segs = [(bounds[i], bounds[i + 1] - bounds[i], int(rng.integers(0, 2))) for i in range(nseg)]
    has_video = any(m == VIDEO for _, _, m in segs)
    fs = int(rng.choice([16, 24, 32, 48, 64]))
    Hkv = int(rng.integers(1, 3))
    Hq = Hkv * int(rng.integers(1, 4))
    kinds = ["dense", "ashape", "vslash", "block", "qbound", "bound2d"] + (["grid"] if has_video else [])
    heads = []
    for _ in range(Hq):
        k = str(rng.choice(kinds))
        if k == "ashape":
            heads.append(Head(k, sink=int(rng.integers(0, 129)), local=int(rng.integers(1, 513))))
        elif k in ("vslash", "qbound", "bound2d"):
            # Q-boundary heads of odd-numbered layers estimate per segment (no extra draw, so the
            # layers' other choices stay as they were)
            heads.append(Head(k, k_v=int(rng.integers(1, L // 4 + 1)), k_s=int(rng.integers(1, L // 2 + 1)),
                              per_segment=(k == "qbound" and seed % 2 == 1)))
        elif k == "block":
            if rng.random() < 0.5:
                heads.append(Head(k, topk_blocks=int(rng.integers(1, 7))))
            else:
                heads.append(Head(k, block_budget=float(rng.uniform(0.05, 0.6))))
        elif k == "grid":
            if rng.random() < 0.5:
                heads.append(Head(k, strides=(fs,), n_phases=int(rng.integers(1, 4))))
            else:
                heads.append(Head(k, strides=(fs,), grid_budget=float(rng.uniform(0.05, 0.3))))
        else:
            heads.append(Head(k))
    return Problem(L=L, Hq=Hq, Hkv=Hkv, segments=segs, heads=heads, frame_stride=fs, name=f"random{seed}")


@pytest.mark.parametrize("seed", range(N_CASES))
def test_random_layer(seed, monkeypatch):
    p = random_problem(seed)
    chunk = 0
    if seed % 3 == 0 and p.L > 128:  # keys cut into small chunks (the long-sequence path)
        chunk = 128 * int(np.random.default_rng(seed).integers(1, (p.L - 1) // 128 + 1))
        monkeypatch.setenv("MSA_ATTN_CHUNK_KEYS", str(chunk))
    what = (f"{p.name} (L={p.L}, Hq={p.Hq}, Hkv={p.Hkv}, segments={p.segments}, "
            f"kinds={[h.kind for h in p.heads]}, key chunk={chunk or 'none'})")
    Q, K, V = make_inputs(p, seed=seed)
    q, k, v = to_dev(Q), to_dev(K), to_dev(V)
    plan = msa.Plan(p)
    if chunk:
        assert plan.attention_units()[1] == (p.L + chunk - 1) // chunk > 1, what
    ws = plan.alloc_workspace()
    o = torch.empty_like(q)
    lse = torch.empty((p.Hq, p.L), dtype=torch.float32, device="cuda")
    plan.forward(q, k, v, ws, o, lse=lse)
    torch.cuda.synchronize()
    assert plan.device_status(ws) == 0, what
    idx = [plan.read_indices(h, ws) for h in range(p.Hq)]
    for h in range(p.Hq):
        _check_head(p, h, idx[h], oracle.estimate_head(p, h, Q, K))
    Oref, lref = oracle.attention(p, Q, K, V, idx)
    got, lse_h = o.float().cpu().numpy(), lse.cpu().numpy()
    for h in range(p.Hq):
        compare_outputs(got[h], Oref[h], f"{what} head {h}")
        fin = np.isfinite(lref[h])
        assert np.array_equal(fin, np.isfinite(lse_h[h])), f"{what} head {h}: empty rows differ"
        np.testing.assert_allclose(lse_h[h][fin], lref[h][fin], atol=2e-3, rtol=1e-3)
    pairs = [int(oracle.mask_count(p, h, idx[h]).sum()) for h in range(p.Hq)]
    assert plan.mask_pairs(ws).tolist() == pairs, what
    ws_i = plan.alloc_workspace(indexed=True)
    o_i = torch.empty_like(q)
    lse_i = torch.empty_like(lse)
    plan.forward(q, k, v, ws_i, o_i, lse=lse_i, indexed=True)
    torch.cuda.synchronize()
    assert plan.device_status(ws_i) == 0, what
    assert torch.equal(o, o_i) and torch.equal(lse, lse_i), f"{what}: index-based path differs"


def random_medium_problem(seed: int) -> Problem:
    """8K-32K tokens, up to 12 text / video runs, frame strides up to 256."""
    rng = np.random.default_rng(5000 + seed)
    L = 1024 * int(rng.integers(8, 33))
    nseg = int(rng.integers(1, 13))
    cuts = np.sort(rng.choice(np.arange(1, L), size=nseg - 1, replace=False)) if nseg > 1 else np.array([], int)
    bounds = [0] + [int(c) for c in cuts] + [L]
    segs = [(bounds[i], bounds[i + 1] - bounds[i], VIDEO if i % 2 == (seed & 1) else TEXT) for i in range(nseg)]
    has_video = any(m == VIDEO for _, _, m in segs)
    fs = int(rng.choice([64, 128, 196, 256]))
    Hkv = int(rng.integers(1, 3))
    Hq = Hkv * int(rng.integers(1, 4))
    kinds = ["ashape", "vslash", "block", "qbound", "bound2d"] + (["grid"] if has_video else [])
    heads = []
    for _ in range(Hq):
        k = str(rng.choice(kinds))
        if k == "ashape":
            heads.append(Head(k, sink=128, local=int(64 * rng.integers(1, 33))))
        elif k in ("vslash", "qbound", "bound2d"):
            heads.append(Head(k, k_v=int(rng.integers(50, 1001)), k_s=int(rng.integers(100, 3001))))
        elif k == "block":
            heads.append(Head(k, block_budget=float(rng.uniform(0.02, 0.2))))
        else:
            heads.append(Head(k, strides=(fs,), grid_budget=float(rng.uniform(0.02, 0.15))))
    return Problem(L=L, Hq=Hq, Hkv=Hkv, segments=segs, heads=heads, frame_stride=fs, name=f"medium{seed}")


@pytest.mark.parametrize("seed", range(6))
def test_random_medium_layer(seed):
    """Medium random layers: index sets against the oracle, outputs on sampled rows (every
    segment's first and last rows, the sequence's last 64, seeded random rows)."""
    p = random_medium_problem(seed)
    what = f"{p.name} (L={p.L}, Hq={p.Hq}, Hkv={p.Hkv}, {len(p.segments)} segments, kinds={[h.kind for h in p.heads]})"
    Q, K, V = make_inputs(p, seed=seed)
    q, k, v = to_dev(Q), to_dev(K), to_dev(V)
    plan = msa.Plan(p)
    ws = plan.alloc_workspace()
    o = torch.empty_like(q)
    plan.forward(q, k, v, ws, o)
    torch.cuda.synchronize()
    assert plan.device_status(ws) == 0, what
    idx = [plan.read_indices(h, ws) for h in range(p.Hq)]
    for h in range(p.Hq):
        _check_head(p, h, idx[h], oracle.estimate_head(p, h, Q, K))
    rng = np.random.default_rng(seed)
    rows = {p.L - 1 - i for i in range(64)}
    for (s0, n, _m) in p.segments:
        rows.update([s0, s0 + n - 1])
    rows.update(rng.choice(p.L, size=96, replace=False).tolist())
    rows = np.array(sorted(rows))
    got = o[:, torch.as_tensor(rows, device=o.device)].float().cpu().numpy()
    for h in range(p.Hq):
        ref, _ = oracle.attention_head(p, h, Q, K, V, idx[h], rows)
        compare_outputs(got[h], ref, f"{what} head {h}")
