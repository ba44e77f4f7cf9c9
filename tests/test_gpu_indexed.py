"""The index-based prefill (msa_sparse_prefill_indexed: query rows gathered by index inside the
attention kernel, output rows written at their original positions) against the three-call path
(permute -> sparse prefill -> unpermute) on the same index sets: the same operations in the same
order, so outputs and log-sum-exps must be bit-identical; and against the oracle.  Every call
goes through the C ABI."""
import numpy as np
import pytest

import oracle
from helpers import compare_outputs, mixed_problem, small_problems, to_dev
from workload import TEXT, VIDEO, Head, Problem, make_inputs

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import dynamic_sparse_attention_head_b200 as msa  # noqa: E402

PROBLEMS = small_problems()


def _both(p, Q, K, V, idx, q=None, k=None, v=None, o_shape=None):
    """(O, lse) of the three-call path and of the index-based path on an indexed-size workspace."""
    q = to_dev(Q) if q is None else q
    k = to_dev(K) if k is None else k
    v = to_dev(V) if v is None else v
    out = []
    for indexed in (False, True):
        plan = msa.Plan(p)
        ws = plan.alloc_workspace(indexed=indexed)
        assert ws.numel() == (plan.workspace_bytes_indexed if indexed else plan.workspace_bytes)
        o = torch.full((p.Hq, p.L, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
        if o_shape == "seq-major":
            o = torch.full((p.L, p.Hq, 128), float("nan"), dtype=torch.bfloat16, device="cuda").transpose(0, 1)
        lse = torch.full((p.Hq, p.L), float("nan"), device="cuda", dtype=torch.float32)
        plan.set_indices(idx, ws)
        if indexed:
            plan.sparse_prefill_indexed(q, k, v, ws, o, lse=lse)
        else:
            plan.permute(q, k, v, ws)
            plan.sparse_prefill(q, k, v, ws, lse=lse)
            plan.unpermute(ws, o)
        torch.cuda.synchronize()
        assert plan.device_status(ws) == 0
        out.append((o.float().cpu().numpy(), lse.cpu().numpy()))
    return out


def _same(a, b, what):
    (oa, la), (ob, lb) = a, b
    assert not np.isnan(ob).any(), f"{what}: output rows left unwritten"
    assert np.array_equal(oa, ob), f"{what}: outputs differ (max {np.nanmax(np.abs(oa - ob))})"
    assert np.array_equal(la, lb), f"{what}: lse differ"


@pytest.mark.parametrize("name", list(PROBLEMS) + ["mixed"])
def test_indexed_equals_three_call_path(name):
    p = mixed_problem() if name == "mixed" else PROBLEMS[name]
    Q, K, V = make_inputs(p, seed=11)
    idx = oracle.estimate(p, Q, K)
    mat, ind = _both(p, Q, K, V, idx)
    _same(mat, ind, name)
    if name in ("grid", "bound2d", "mixed"):  # and the oracle, directly
        Oref, _ = oracle.attention(p, Q, K, V, idx)
        for h in range(p.Hq):
            compare_outputs(ind[0][h], Oref[h], f"{name} head {h}")


@pytest.mark.parametrize("chunk_keys", [128, 384])
def test_indexed_over_chunked_keys(chunk_keys, monkeypatch):
    monkeypatch.setenv("MSA_ATTN_CHUNK_KEYS", str(chunk_keys))
    p = mixed_problem()
    Q, K, V = make_inputs(p, seed=12)
    idx = oracle.estimate(p, Q, K)
    mat, ind = _both(p, Q, K, V, idx)
    _same(mat, ind, f"mixed, {chunk_keys}-key chunks")


def test_indexed_sequence_major_tensors():
    """Q, K, V and O as [L, H, 128] views: the row gather and the output scatter follow strides."""
    p = Problem(L=640, Hq=4, Hkv=2, segments=[(0, 384, VIDEO), (384, 256, TEXT)],
                heads=[Head("grid", strides=(64,), grid_budget=0.2), Head("qbound", k_v=16, k_s=32),
                       Head("bound2d", k_v=16, k_s=32), Head("vslash", k_v=16, k_s=32)],
                frame_stride=64, name="seq-major")
    Q, K, V = make_inputs(p, seed=13)
    idx = oracle.estimate(p, Q, K)

    def seq_major(x):
        return to_dev(np.ascontiguousarray(x.transpose(1, 0, 2))).transpose(0, 1)

    mat, ind = _both(p, Q, K, V, idx, q=seq_major(Q), k=seq_major(K), v=seq_major(V), o_shape="seq-major")
    _same(mat, ind, "sequence-major")


def test_indexed_workspace_is_smaller_and_checked():
    p = PROBLEMS["grid"]
    plan = msa.Plan(p)
    assert plan.workspace_bytes_indexed < plan.workspace_bytes
    Q, K, V = make_inputs(p, seed=14)
    q, k, v = to_dev(Q), to_dev(K), to_dev(V)
    ws = plan.alloc_workspace(indexed=True)
    plan.estimate(q, k, ws)
    with pytest.raises(msa.MsaError) as e:  # the three-call path needs the permuted copies
        plan.permute(q, k, v, ws)
    assert e.value.code == 4  # MSA_ERR_WORKSPACE


@pytest.mark.parametrize("wl", ["qwen2-7b-video-128k", "longvila-1m"])
def test_indexed_equals_three_call_path_full_size(wl):
    """At the benchmark sizes, in the launch configuration the bench times (keys chunked at
    1M): both paths leave the same bits in O and lse."""
    import workload
    p = workload.qwen2_7b_video_128k() if wl == "qwen2-7b-video-128k" else workload.longvila_1m()
    Q, K, V = make_inputs(p, seed=0)
    q, k, v = to_dev(Q), to_dev(K), to_dev(V)
    del Q, K, V
    plan = msa.Plan(p)
    outs = []
    for indexed in (False, True):
        ws = plan.alloc_workspace(indexed=indexed)
        o = torch.empty_like(q)
        lse = torch.empty((p.Hq, p.L), device="cuda", dtype=torch.float32)
        plan.forward(q, k, v, ws, o, lse=lse, indexed=indexed)
        torch.cuda.synchronize()
        assert plan.device_status(ws) == 0
        del ws
        torch.cuda.empty_cache()
        outs.append((o, lse))
    assert torch.equal(outs[0][0], outs[1][0]), f"{wl}: outputs differ"
    assert torch.equal(outs[0][1], outs[1][1]), f"{wl}: lse differ"
