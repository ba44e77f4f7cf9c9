"""Attention over chunked keys (the long-sequence path: work units of one key chunk each, the
online-softmax state of a work item carried from chunk to chunk through its accumulator)
against the oracle.  The chunk size is forced small (MSA_ATTN_CHUNK_KEYS, read when the plan is
created) so that small problems cross many chunk boundaries, including chunks without keys."""
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


def _run(p, Q, K, V, idx, monkeypatch, chunk_keys):
    monkeypatch.setenv("MSA_ATTN_CHUNK_KEYS", str(chunk_keys))
    plan = msa.Plan(p)
    units, chunks = plan.attention_units()
    assert chunks == (p.L + chunk_keys - 1) // chunk_keys > 1
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
    return o.float().cpu().numpy(), lse.cpu().numpy()


@pytest.mark.parametrize("chunk_keys", [128, 384])
@pytest.mark.parametrize("name", list(PROBLEMS))
def test_chunked_prefill_matches_oracle(name, chunk_keys, monkeypatch):
    p = PROBLEMS[name]
    Q, K, V = make_inputs(p, seed=1)
    idx = oracle.estimate(p, Q, K)
    O, lse = _run(p, Q, K, V, idx, monkeypatch, chunk_keys)
    Oref, lref = oracle.attention(p, Q, K, V, idx)
    for h in range(p.Hq):
        compare_outputs(O[h], Oref[h], f"{name} head {h} chunk {chunk_keys}")
        fin = np.isfinite(lref[h])
        assert np.array_equal(fin, np.isfinite(lse[h])), f"{name} head {h}: empty rows differ"
        np.testing.assert_allclose(lse[h][fin], lref[h][fin], atol=2e-3, rtol=1e-3)


def test_chunked_mixed_layer_equals_unchunked(monkeypatch):
    """Same layer with and without chunking: identical up to the rounding of the carried state."""
    p = mixed_problem()
    Q, K, V = make_inputs(p, seed=4)
    idx = oracle.estimate(p, Q, K)
    O1, l1 = _run(p, Q, K, V, idx, monkeypatch, 256)
    monkeypatch.setenv("MSA_ATTN_CHUNK_KEYS", "0")
    plan = msa.Plan(p)
    assert plan.attention_units()[1] == 1
    ws = plan.alloc_workspace()
    q, k, v = to_dev(Q), to_dev(K), to_dev(V)
    o = torch.zeros_like(q)
    lse = torch.full((p.Hq, p.L), float("nan"), device="cuda", dtype=torch.float32)
    plan.set_indices(idx, ws)
    plan.permute(q, k, v, ws)
    plan.sparse_prefill(q, k, v, ws, lse=lse)
    plan.unpermute(ws, o)
    torch.cuda.synchronize()
    O0, l0 = o.float().cpu().numpy(), lse.cpu().numpy()
    np.testing.assert_allclose(O1, O0, atol=1e-2, rtol=0)
    fin = np.isfinite(l0)
    assert np.array_equal(fin, np.isfinite(l1))
    np.testing.assert_allclose(l1[fin], l0[fin], atol=1e-3, rtol=1e-4)


@pytest.mark.parametrize("band_slots,min_units", [(1, 1), (2, 16), (1, 40)])
def test_tiny_bands_match_oracle_on_all_rows(band_slots, min_units, monkeypatch):
    """Many small unit bands (MSA_ATTN_BAND_SLOTS / MSA_ATTN_MIN_BAND_UNITS) over small key
    chunks, on a layer whose items are long and short (every head kind, one KV head): alternate
    bands share two sets of accumulator slots, so every slot is reused many times while units
    of earlier bands may still be running.  All rows against the oracle, and three launches
    bit-identical (a unit that wrote into a slot still in use would make them differ)."""
    p = mixed_problem()
    Q, K, V = make_inputs(p, seed=12)
    idx = oracle.estimate(p, Q, K)
    monkeypatch.setenv("MSA_ATTN_BAND_SLOTS", str(band_slots))
    monkeypatch.setenv("MSA_ATTN_MIN_BAND_UNITS", str(min_units))
    monkeypatch.setenv("MSA_ATTN_CHUNK_KEYS", "128")
    units, chunks, bands = msa.Plan(p).attention_work()
    assert chunks == (p.L + 127) // 128 and bands >= 8, (units, chunks, bands)
    runs = [_run(p, Q, K, V, idx, monkeypatch, 128) for _ in range(3)]
    O, lse = runs[0]
    for O2, l2 in runs[1:]:
        assert np.array_equal(O2, O) and np.array_equal(l2, lse, equal_nan=True)
    Oref, lref = oracle.attention(p, Q, K, V, idx)
    for h in range(p.Hq):
        compare_outputs(O[h], Oref[h], f"head {h} bands {bands}")
        fin = np.isfinite(lref[h])
        assert np.array_equal(fin, np.isfinite(lse[h])), f"head {h}: empty rows differ"
        np.testing.assert_allclose(lse[h][fin], lref[h][fin], atol=2e-3, rtol=1e-3)
