"""GPU parity of the permute -> sparse prefill -> unpermute path, driven by index sets the
oracle estimated (msa_set_indices), against the oracle's masked attention; and the
executed-tile coverage of the oracle mask.  Every call goes through the C ABI."""
import numpy as np
import pytest

import oracle
from helpers import compare_outputs, mixed_problem, small_problems, to_dev
from workload import make_inputs

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import dynamic_sparse_attention_head_b200 as msa  # noqa: E402

PROBLEMS = small_problems()


def _run(p, Q, K, V, idx):
    plan = msa.Plan(p)
    ws = plan.alloc_workspace()
    q, k, v = to_dev(Q), to_dev(K), to_dev(V)
    o = torch.zeros_like(q)
    lse = torch.full((p.Hq, p.L), float("nan"), device="cuda", dtype=torch.float32)
    plan.set_indices(idx, ws)
    plan.permute(q, k, v, ws)
    plan.sparse_prefill(q, k, v, ws, lse=lse)
    plan.unpermute(ws, o)
    torch.cuda.synchronize()
    assert plan.device_status(ws) == 0
    return plan, ws, o.float().cpu().numpy(), lse.cpu().numpy()


@pytest.mark.parametrize("name", list(PROBLEMS))
def test_prefill_matches_oracle(name):
    p = PROBLEMS[name]
    Q, K, V = make_inputs(p, seed=1)
    idx = oracle.estimate(p, Q, K)
    plan, ws, O, lse = _run(p, Q, K, V, idx)
    Oref, lref = oracle.attention(p, Q, K, V, idx)
    for h in range(p.Hq):
        compare_outputs(O[h], Oref[h], f"{name} head {h}")
        fin = np.isfinite(lref[h])
        assert np.array_equal(fin, np.isfinite(lse[h])), f"{name} head {h}: empty rows differ"
        np.testing.assert_allclose(lse[h][fin], lref[h][fin], atol=2e-3, rtol=1e-3)


def test_mixed_heads_one_layer():
    p = mixed_problem()
    Q, K, V = make_inputs(p, seed=4)
    idx = oracle.estimate(p, Q, K)
    _, _, O, _ = _run(p, Q, K, V, idx)
    Oref, _ = oracle.attention(p, Q, K, V, idx)
    for h in range(p.Hq):
        compare_outputs(O[h], Oref[h], f"mixed head {h} ({p.heads[h].kind})")


@pytest.mark.parametrize("name", ["ashape", "vslash", "block", "grid", "qbound", "bound2d"])
def test_tiles_cover_mask_exactly_once(name):
    """Every allowed (query, key) pair lies in exactly one executed tile of its query."""
    p = PROBLEMS[name]
    Q, K, V = make_inputs(p, seed=2)
    idx = oracle.estimate(p, Q, K)
    plan, ws, _, _ = _run(p, Q, K, V, idx)
    for h in range(p.Hq):
        mask = oracle.mask_rows(p, h, idx[h], np.arange(p.L)).astype(bool)
        cover = np.zeros((p.L, p.L), np.int32)
        seen_rows = np.zeros(p.L, np.int32)
        n_full = 0
        for it in plan.read_tiles(h, ws):
            rows = it["rows"][it["rows"] >= 0]
            seen_rows[rows] += 1
            for _, keys, full in it["tiles"]:
                kk = keys[keys >= 0]
                cover[np.ix_(rows, kk)] += 1
                if full:  # the kernel skips the element mask: every pair must be allowed
                    assert len(kk) == 128 and mask[np.ix_(rows, kk)].all(), f"{name} head {h}: tile flagged full"
                    n_full += 1
        assert np.all(seen_rows == 1), f"{name} head {h}: every query in exactly one work item"
        assert np.all(cover[mask] == 1), f"{name} head {h}: allowed pairs not covered exactly once"
        assert cover.max() <= 1, f"{name} head {h}: a key appears twice in one row's tiles"
        if name == "ashape" and h == 0:  # local 256: tiles inside the band below the diagonal need no mask
            assert n_full > 0, f"{name} head {h}: no tile flagged full"


@pytest.mark.parametrize("name", list(PROBLEMS) + ["mixed"])
def test_mask_pairs_match_oracle(name):
    """Allowed pairs per head counted on the device with the kernel's mask logic equal the
    oracle's token-level mask counts exactly (the useful FLOPs the bench reports)."""
    p = mixed_problem() if name == "mixed" else PROBLEMS[name]
    Q, K, V = make_inputs(p, seed=5)
    idx = oracle.estimate(p, Q, K)
    plan, ws, _, _ = _run(p, Q, K, V, idx)
    got = plan.mask_pairs(ws)
    ref = np.array([int(oracle.mask_count(p, h, idx[h]).sum()) for h in range(p.Hq)], np.int64)
    assert np.array_equal(got, ref), f"{name}: device {got.tolist()} oracle {ref.tolist()}"
    if name == "dense":
        assert np.all(got == p.L * (p.L + 1) // 2)
    tiles, _ = plan.tile_stats(ws)
    assert got.sum() <= tiles * 128 * 128


def test_dense_executes_causal_tiles_only():
    p = PROBLEMS["dense"]
    Q, K, V = make_inputs(p, seed=3)
    plan, ws, _, _ = _run(p, Q, K, V, [{} for _ in range(p.Hq)])
    tiles, items = plan.tile_stats(ws)
    nq = (p.L + 127) // 128
    # causal 128x128 tiles, the diagonal one split into two 64-key units when the row tile is ragged
    per_head = sum(((min(p.L, 128 * (i + 1)) - 1) // 64 + 2) // 2 for i in range(nq))
    assert tiles == p.Hq * per_head and items == p.Hq * nq
    # every tile strictly below the diagonal of its 128-query item is flagged full
    for h in range(p.Hq):
        n_full = sum(full for it in plan.read_tiles(h, ws) for _, _, full in it["tiles"])
        assert n_full == nq * (nq - 1) // 2
