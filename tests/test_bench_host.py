"""Host logic of bench.py (no GPU): the oracle's stratified row sample and the per-kind density
accounting of the bench line."""
import numpy as np

import bench
import workload


def test_sample_rows_one_per_stratum():
    L, n = 131072, 4096
    rows = bench.sample_rows(L, n, seed=3)
    assert len(rows) == n
    edges = np.linspace(0, L, n + 1).astype(np.int64)
    assert np.all(rows >= edges[:-1]) and np.all(rows < edges[1:])
    assert np.array_equal(rows, bench.sample_rows(L, n, seed=3))  # seeded
    assert len(bench.sample_rows(100, 4096, seed=0)) == 100  # never more rows than L


def test_per_kind_stats_closed_form():
    p = workload.llama3_8b_text(L=2048)
    dense_head = 2 * p.d * p.L * (p.L + 1)
    tiles = np.zeros(p.Hq, np.int64)
    pairs = np.zeros(p.Hq, np.int64)
    kinds = {}
    for h, hd in enumerate(p.heads):
        kinds.setdefault(hd.kind, []).append(h)
    # every head of the first kind executes exactly its dense causal tiles' worth and uses a quarter
    k0 = next(iter(kinds))
    per_tile = 4 * 128 ** 3
    for h in kinds[k0]:
        tiles[h] = dense_head // per_tile
        pairs[h] = (dense_head // (4 * p.d)) // 4
    st = bench.per_kind_stats(p, tiles, pairs)
    assert set(st) == set(kinds)
    assert st[k0]["heads"] == len(kinds[k0])
    assert abs(st[k0]["executed_density"] - (dense_head // per_tile) * per_tile / dense_head) < 1e-12
    assert abs(st[k0]["mask_density"] - 0.25) < 1e-3
    for k in kinds:
        if k != k0:
            assert st[k]["executed_density"] == 0.0 and st[k]["useful_over_executed"] is None
