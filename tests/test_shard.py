"""Split of one layer by KV-head group over ranks (each rank: its KV heads and the query heads
that read them, no exchange): the shards cover every head once with the GQA mapping intact, a
shard's inputs are the same heads of the whole layer's, and the oracle on a shard gives the
whole layer's results for those heads."""
import numpy as np
import pytest

import oracle
from workload import TEXT, VIDEO, Head, Problem, make_inputs, shard_kv_heads


def _same(a, b):
    """Exact equality of nested index-set records (dicts, lists, arrays, scalars)."""
    if isinstance(a, dict):
        return isinstance(b, dict) and a.keys() == b.keys() and all(_same(a[k], b[k]) for k in a)
    if isinstance(a, (list, tuple)):
        return len(a) == len(b) and all(_same(x, y) for x, y in zip(a, b))
    if isinstance(a, np.ndarray) or isinstance(b, np.ndarray):
        return np.array_equal(np.asarray(a), np.asarray(b))
    return a == b


def _layer():
    heads = [Head("vslash", k_v=8, k_s=16), Head("qbound", k_v=6, k_s=12), Head("grid", strides=(32,), grid_budget=0.2),
             Head("bound2d", k_v=6, k_s=12), Head("ashape", sink=16, local=64), Head("block", topk_blocks=2),
             Head("vslash", k_v=20, k_s=8), Head("dense")]
    return Problem(L=512, Hq=8, Hkv=4, segments=[(0, 160, TEXT), (160, 288, VIDEO), (448, 64, TEXT)],
                   heads=heads, frame_stride=32, name="shard-test")


@pytest.mark.parametrize("world", [1, 2, 4])
def test_shards_cover_every_head_once_with_their_kv_heads(world):
    p = _layer()
    G = p.Hq // p.Hkv
    seen_q, seen_kv = [], []
    for r in range(world):
        sub, qh, kvh = shard_kv_heads(p, r, world)
        assert sub.Hq == len(qh) and sub.Hkv == len(kvh) and sub.Hq // sub.Hkv == G
        assert all(h // G in kvh for h in qh)
        assert [sub.heads[i].kind for i in range(sub.Hq)] == [p.heads[h].kind for h in qh]
        seen_q += list(qh)
        seen_kv += list(kvh)
    assert seen_q == list(range(p.Hq)) and seen_kv == list(range(p.Hkv))


def test_bad_splits_are_refused():
    p = _layer()
    with pytest.raises(ValueError):
        shard_kv_heads(p, 0, 3)
    with pytest.raises(ValueError):
        shard_kv_heads(p, 2, 2)


def test_shard_inputs_and_oracle_equal_the_whole_layers():
    p = _layer()
    Q, K, V = make_inputs(p, seed=4, inputs="rope")
    full = oracle.estimate(p, Q, K)
    for r in range(2):
        sub, qh, kvh = shard_kv_heads(p, r, 2)
        Qs, Ks, Vs = make_inputs(sub, seed=4, inputs="rope", q_heads=qh, kv_heads=kvh)
        assert np.array_equal(Qs, Q[qh.start:qh.stop]) and np.array_equal(Ks, K[kvh.start:kvh.stop])
        assert np.array_equal(Vs, V[kvh.start:kvh.stop])
        part = oracle.estimate(sub, Qs, Ks)
        for i, h in enumerate(qh):
            a, b = part[i], full[h]
            assert _same(a, b), h
        O, _ = oracle.attention(sub, Qs, Ks, Vs, part)
        Of, _ = oracle.attention(p, Q, K, V, full)
        assert np.array_equal(O, Of[qh.start:qh.stop])
