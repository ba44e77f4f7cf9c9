"""Degenerate and edge inputs through the C ABI against the oracle: the shortest sequences (one
partial tile), rows the mask leaves empty (O = 0, LSE = -inf), sequence-major [L, H, d] tensors
passed through explicit strides, no GQA and one KV head for many query heads, and layouts with a
single modality under the modality-aware heads."""
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

ALL_KINDS = [Head("dense"), Head("ashape", sink=16, local=40), Head("vslash", k_v=8, k_s=16),
             Head("block", topk_blocks=2), Head("grid", strides=(32,), grid_budget=0.25),
             Head("qbound", k_v=8, k_s=16), Head("bound2d", k_v=8, k_s=16)]


def _forward(p, Q, K, V, q=None, k=None, v=None, o=None):
    plan = msa.Plan(p)
    ws = plan.alloc_workspace()
    q = to_dev(Q) if q is None else q
    k = to_dev(K) if k is None else k
    v = to_dev(V) if v is None else v
    o = torch.empty((p.Hq, p.L, 128), dtype=torch.bfloat16, device="cuda") if o is None else o
    lse = torch.empty((p.Hq, p.L), dtype=torch.float32, device="cuda")
    plan.forward(q, k, v, ws, o, lse=lse)
    torch.cuda.synchronize()
    assert plan.device_status(ws) == 0
    idx = [plan.read_indices(h, ws) for h in range(p.Hq)]
    # allowed pairs per head under the device's index sets: exact against the oracle's masks
    ref = [int(oracle.mask_count(p, h, idx[h]).sum()) for h in range(p.Hq)]
    assert plan.mask_pairs(ws).tolist() == ref, f"{p.name}: mask pair counts"
    return idx, o, lse.cpu().numpy()


def _check(p, Q, K, V, idx, o, lse, what):
    for h in range(p.Hq):
        _check_head(p, h, idx[h], oracle.estimate_head(p, h, Q, K))
    Oref, lref = oracle.attention(p, Q, K, V, idx)
    got = o.float().cpu().numpy()
    for h in range(p.Hq):
        compare_outputs(got[h], Oref[h], f"{what} head {h}")
        fin = np.isfinite(lref[h])
        assert np.array_equal(fin, np.isfinite(lse[h])), f"{what} head {h}: empty rows differ"
        np.testing.assert_allclose(lse[h][fin], lref[h][fin], atol=2e-3, rtol=1e-3)
    return Oref, lref


@pytest.mark.parametrize("L", [64, 128, 192])
def test_shortest_sequences_every_kind(L):
    segs = [(0, L // 2, VIDEO), (L // 2, L - L // 2, TEXT)] if L >= 128 else [(0, L, VIDEO)]
    p = Problem(L=L, Hq=len(ALL_KINDS), Hkv=1, segments=segs, heads=ALL_KINDS, frame_stride=32, name=f"L{L}")
    Q, K, V = make_inputs(p, seed=L)
    idx, o, lse = _forward(p, Q, K, V)
    _check(p, Q, K, V, idx, o, lse, f"L={L}")


def test_rows_left_empty_give_zero_output():
    # one vertical and one slash line: most early rows see neither (no entries are forced)
    p = Problem(L=512, Hq=2, Hkv=1, segments=[(0, 512, TEXT)],
                heads=[Head("vslash", k_v=1, k_s=1), Head("block", topk_blocks=1)], name="empty-rows")
    Q, K, V = make_inputs(p, seed=3)
    idx, o, lse = _forward(p, Q, K, V)
    Oref, lref = _check(p, Q, K, V, idx, o, lse, "empty rows")
    empty = ~np.isfinite(lref[0])
    assert empty.any(), "the layout leaves some rows without keys"
    assert np.all(o[0].float().cpu().numpy()[empty] == 0.0)


def test_sequence_major_tensors_through_strides():
    p = Problem(L=1088, Hq=4, Hkv=2, segments=[(0, 512, VIDEO), (512, 576, TEXT)],
                heads=[Head("qbound", k_v=20, k_s=50), Head("grid", strides=(64,), grid_budget=0.2),
                       Head("vslash", k_v=30, k_s=60), Head("ashape", sink=32, local=100)],
                frame_stride=64, name="seq-major")
    Q, K, V = make_inputs(p, seed=6)
    lhd = lambda x: to_dev(x).permute(1, 0, 2).contiguous()  # noqa: E731  [L, H, d] buffers
    q, k, v = lhd(Q), lhd(K), lhd(V)
    o = torch.empty((p.L, p.Hq, 128), dtype=torch.bfloat16, device="cuda")
    idx, _, lse = _forward(p, Q, K, V, q.permute(1, 0, 2), k.permute(1, 0, 2), v.permute(1, 0, 2),
                           o.permute(1, 0, 2))
    _check(p, Q, K, V, idx, o.permute(1, 0, 2), lse, "seq-major")


@pytest.mark.parametrize("hq,hkv", [(4, 4), (8, 1)])
def test_group_sizes(hq, hkv):
    kinds = [Head("vslash", k_v=16, k_s=40), Head("block", block_budget=0.3), Head("ashape", sink=8, local=64),
             Head("dense")]
    p = Problem(L=704, Hq=hq, Hkv=hkv, segments=[(0, 704, TEXT)], heads=[kinds[h % 4] for h in range(hq)],
                name=f"g{hq}x{hkv}")
    Q, K, V = make_inputs(p, seed=hq + hkv)
    idx, o, lse = _forward(p, Q, K, V)
    _check(p, Q, K, V, idx, o, lse, p.name)


@pytest.mark.parametrize("modality", [VIDEO, TEXT])
def test_single_modality_layout(modality):
    p = Problem(L=1024, Hq=3, Hkv=1, segments=[(0, 1024, modality)],
                heads=[Head("qbound", k_v=16, k_s=40), Head("bound2d", k_v=16, k_s=40),
                       Head("grid", strides=(64,), grid_budget=0.2) if modality == VIDEO else Head("vslash", k_v=16, k_s=40)],
                frame_stride=64 if modality == VIDEO else 0, name=f"only-{modality}")
    Q, K, V = make_inputs(p, seed=9)
    idx, o, lse = _forward(p, Q, K, V)
    _check(p, Q, K, V, idx, o, lse, p.name)


def test_calls_out_of_order_are_refused():
    """Permute, prefill and the mask count need this plan's indices in the workspace first."""
    p = Problem(L=256, Hq=1, Hkv=1, segments=[(0, 256, TEXT)], heads=[Head("vslash", k_v=4, k_s=8)],
                name="order")
    Q, K, V = make_inputs(p, seed=9)
    plan = msa.Plan(p)
    ws = plan.alloc_workspace()
    q, k, v = to_dev(Q), to_dev(K), to_dev(V)
    for call in (lambda: plan.mask_pairs(ws), lambda: plan.permute(q, k, v, ws),
                 lambda: plan.sparse_prefill(q, k, v, ws)):
        with pytest.raises(msa.MsaError) as e:
            call()
        assert e.value.code == 9  # MSA_ERR_STATE
    plan.estimate(q, k, ws)
    assert plan.mask_pairs(ws).shape == (1,)


def test_expired_wait_is_reported_and_the_context_stays_usable():
    """A bounded wait that nothing completes (msa_selftest_timeout: the kernels' own wait helper
    on a barrier no thread arrives at) gives up after its limit, is reported as MSA_ERR_TIMEOUT
    by msa_device_status, is cleared by that call, and leaves the context usable: the rest of the
    path on the same workspace afterwards still matches the oracle."""
    import time
    p = Problem(L=512, Hq=2, Hkv=1, segments=[(0, 512, TEXT)],
                heads=[Head("vslash", k_v=8, k_s=16), Head("ashape", sink=16, local=64)], name="timeout")
    Q, K, V = make_inputs(p, seed=21)
    q, k, v = to_dev(Q), to_dev(K), to_dev(V)
    plan = msa.Plan(p)
    ws = plan.alloc_workspace()
    plan.estimate(q, k, ws)  # uploads the plan tables: the status word starts clear
    assert plan.device_status(ws) == 0
    t0 = time.perf_counter()
    plan.selftest_timeout(ws, limit_us=20000)
    assert plan.device_status(ws) == 7  # MSA_ERR_TIMEOUT, once the wait ran out
    elapsed = time.perf_counter() - t0
    assert 0.015 < elapsed < 5.0, f"wait took {elapsed:.3f} s"
    assert plan.device_status(ws) == 0  # cleared by the read
    o = torch.empty_like(q)
    lse = torch.empty((p.Hq, p.L), dtype=torch.float32, device="cuda")
    plan.permute(q, k, v, ws)
    plan.sparse_prefill(q, k, v, ws, lse=lse)
    plan.unpermute(ws, o)
    torch.cuda.synchronize()
    assert plan.device_status(ws) == 0
    idx = [plan.read_indices(h, ws) for h in range(p.Hq)]
    _check(p, Q, K, V, idx, o, lse.cpu().numpy(), "after a timeout")


def test_concurrent_prefills_on_two_streams():
    """All device state lives in the caller's workspace (work counters, index sets, tile lists,
    status word), so two layers on two streams, each with its own workspace, may run at the same
    time: each output equals its sequential run bit for bit."""
    P = [Problem(L=1472, Hq=7, Hkv=1, segments=[(0, 576, VIDEO), (576, 256, TEXT), (832, 480, VIDEO), (1312, 160, TEXT)],
                 heads=ALL_KINDS, frame_stride=32, name="streams-a"),
         Problem(L=2048, Hq=4, Hkv=2, segments=[(0, 2048, TEXT)],
                 heads=[Head("vslash", k_v=40, k_s=200), Head("ashape", sink=64, local=256),
                        Head("block", topk_blocks=4), Head("dense")], name="streams-b")]
    runs = []
    for p in P:
        Q, K, V = make_inputs(p, seed=31)
        plan = msa.Plan(p)
        runs.append((p, plan, plan.alloc_workspace(), to_dev(Q), to_dev(K), to_dev(V)))
    seq = []
    for p, plan, ws, q, k, v in runs:
        o = torch.empty_like(q)
        plan.forward(q, k, v, ws, o)
        torch.cuda.synchronize()
        assert plan.device_status(ws) == 0
        seq.append(o)
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs = [torch.empty_like(r[3]) for r in runs]
    for _ in range(3):
        for (p, plan, ws, q, k, v), o, st in zip(runs, outs, streams):
            with torch.cuda.stream(st):
                plan.forward(q, k, v, ws, o, stream=st)
        torch.cuda.synchronize()
        for (p, plan, ws, *_), o, ref in zip(runs, outs, seq):
            assert plan.device_status(ws) == 0
            assert torch.equal(o, ref), f"{p.name}: concurrent run differs"


def test_path_replays_from_a_cuda_graph():
    """The whole per-layer path (estimate -> permute -> sparse prefill -> unpermute, and the
    index-based pair) is stream-ordered with no synchronisation, so it can be captured in a CUDA
    graph; replays with new inputs copied into the captured buffers match eager runs bit for bit."""
    p = Problem(L=1472, Hq=7, Hkv=1, segments=[(0, 576, VIDEO), (576, 256, TEXT), (832, 480, VIDEO), (1312, 160, TEXT)],
                heads=ALL_KINDS, frame_stride=32, name="graph")
    plan = msa.Plan(p)
    for indexed in (False, True):
        ws = plan.alloc_workspace(indexed=indexed)
        inputs = [make_inputs(p, seed=s) for s in (41, 42)]
        q, k, v = (to_dev(x) for x in inputs[0])
        o = torch.empty_like(q)
        eager = []
        for Q, K, V in inputs:
            qq, kk, vv = to_dev(Q), to_dev(K), to_dev(V)
            oo = torch.empty_like(qq)
            plan.forward(qq, kk, vv, ws, oo, indexed=indexed)
            torch.cuda.synchronize()
            eager.append(oo)
        st = torch.cuda.Stream()
        st.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(st):  # warm-up on the capture stream
            plan.forward(q, k, v, ws, o, stream=st, indexed=indexed)
        torch.cuda.current_stream().wait_stream(st)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=st):
            plan.forward(q, k, v, ws, o, stream=st, indexed=indexed)
        for (Q, K, V), ref in zip(inputs, eager):
            q.copy_(to_dev(Q))
            k.copy_(to_dev(K))
            v.copy_(to_dev(V))
            g.replay()
            torch.cuda.synchronize()
            assert plan.device_status(ws) == 0
            assert torch.equal(o, ref), f"graph replay differs (indexed={indexed})"
        del g
