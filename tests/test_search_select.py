"""Pattern search selection rule and recall arithmetic (host only)."""
import numpy as np

from dynamic_sparse_attention_head_b200 import search


def test_choose_highest_recall_within_budget():
    recall = np.array([[0.90, 0.50], [0.95, 0.60], [0.99, 0.70]])
    flops = np.array([[10, 10], [20, 20], [40, 15]])
    # budget 25: head 0 may take candidates 0 or 1 (picks 1), head 1 any of them (picks 2)
    assert search.choose(recall, flops, 25) == [1, 2]


def test_choose_cheapest_when_nothing_fits_and_cheaper_on_ties():
    recall = np.array([[0.9], [0.9], [0.5]])
    flops = np.array([[30], [20], [50]])
    assert search.choose(recall, flops, 25) == [1]       # tie in recall: the cheaper
    assert search.choose(recall, flops, 10) == [1]       # nothing fits: the cheapest


def test_recall_from_lse():
    dense = np.log(np.array([[1.0, 2.0, 4.0]]))
    mask = np.array([[0.0, 0.0, -np.inf]])
    r = search.recall_from_lse(mask, dense)
    np.testing.assert_allclose(r, [[1.0, 0.5, 0.0]])


def test_dense_head_flops_counts_causal_tiles():
    class P:
        L = 256
    # two 128-query tiles: 1 + 2 executed tiles
    assert search.dense_head_flops(P) == 3 * 4 * 128 ** 3
