"""The allocation-free vertical-slash estimation (msa_vslash_estimate_static) serves callers
that cannot allocate device memory or hand over a workspace (code running inside another
framework's memory manager, serving loops where cudaMalloc and its device synchronisation are
not allowed).  Its index sets must match the oracle's under the near-tie rule and equal those of
the regular entry point (msa_estimate on a one-head vertical-slash plan: the same kernels and key
chunking), call after call: its scratch is one static array that every call reuses.  Collected
last so a failure here comes after every other test has run."""
import numpy as np
import pytest

import oracle
from helpers import near_tie_ok, to_dev
from workload import TEXT, Head, Problem, make_inputs

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import dynamic_sparse_attention_head_b200 as msa  # noqa: E402


def _regular(p, q, k):
    plan = msa.Plan(p)
    ws = plan.alloc_workspace()
    plan.estimate(q, k, ws)
    torch.cuda.synchronize()
    return plan.read_indices(0, ws)


@pytest.mark.parametrize("L,k_v,k_s,seed", [(8192, 100, 300, 0), (4096, 7, 2000, 1)])
def test_static_scratch_matches_regular_entry_point_twice(L, k_v, k_s, seed):
    p = Problem(L=L, Hq=1, Hkv=1, segments=[(0, L, TEXT)], heads=[Head("vslash", k_v=k_v, k_s=k_s)])
    Q, K, _ = make_inputs(p, seed=seed)
    q, k = to_dev(Q), to_dev(K)
    ref = _regular(p, q, k)
    orc = oracle.estimate_head(p, 0, Q, K)
    # the regular entry point against the oracle first, so that a failure below is the
    # allocation-free call's own
    near_tie_ok(ref["V"], orc["V"], orc["v"], what="regular vertical")
    near_tie_ok(ref["S"], orc["S"], orc["s"], what="regular slash")
    v_out = torch.full((k_v,), -1, dtype=torch.int32, device="cuda")
    s_out = torch.full((k_s,), -1, dtype=torch.int32, device="cuda")
    counts = torch.zeros(2, dtype=torch.int32, device="cuda")
    first = None
    for _ in range(2):  # the second call runs on the scratch the first one left behind
        v_out.fill_(-1)
        s_out.fill_(-1)
        msa.vslash_estimate_static(q[0], k[0], p.scale, k_v, k_s, v_out, s_out, counts)
        torch.cuda.synchronize()
        nv, ns = counts.tolist()
        assert nv == k_v and ns == k_s
        V = v_out[:nv].cpu().numpy()
        S = s_out[:ns].cpu().numpy()
        assert np.all(np.diff(V) > 0) and np.all(np.diff(S) > 0)
        near_tie_ok(V, orc["V"], orc["v"], what="vertical vs oracle")
        near_tie_ok(S, orc["S"], orc["s"], what="slash vs oracle")
        # the same sweep (one-head tile, same key chunks) as msa_estimate: the same lines
        assert V.tolist() == ref["V"].tolist() and S.tolist() == ref["S"].tolist()
        if first is None:
            first = (V.tolist(), S.tolist())
        else:  # deterministic: the second call gives what the first gave
            assert (V.tolist(), S.tolist()) == first


def test_static_scratch_rejects_oversized_problem():
    L = 65536 + 64
    q = torch.zeros((L, 128), dtype=torch.bfloat16, device="cuda")
    v_out = torch.zeros(4, dtype=torch.int32, device="cuda")
    counts = torch.zeros(2, dtype=torch.int32, device="cuda")
    with pytest.raises(msa.MsaError) as e:
        msa.vslash_estimate_static(q, q, 0.088, 4, 4, v_out, v_out, counts)
    assert e.value.code == 5  # MSA_ERR_UNSUPPORTED
