"""Pins of the oracle's weight-share statistic (the fewest dense attention weights of a query row
whose sum reaches a given recall; MMInference summary page, attention analysis) against counts
derived by hand: uniform rows, one dominant key, and a two-level row whose count follows from
the two weights in closed form."""
import math

import numpy as np

import oracle

SCALE = float(np.float32(1.0 / math.sqrt(128)))


def _bits(x):
    b = np.ascontiguousarray(np.asarray(x, np.float32)).view(np.uint32)
    assert np.all((b & 0xFFFF) == 0), "values must be exact in bf16"
    return (b >> 16).astype(np.uint16)


def _inputs(L, key_values, q0=1.0):
    """One head; q = q0 * e_0, key j = key_values[j] * e_0: logit_j = q0 * key_values[j] * scale."""
    Q = np.zeros((1, L, 128), np.float32)
    K = np.zeros((1, L, 128), np.float32)
    Q[0, :, 0] = q0
    K[0, :, 0] = key_values
    return _bits(Q), _bits(K)


def test_uniform_row_needs_the_recall_fraction_of_its_keys():
    L = 200
    Q, K = _inputs(L, np.zeros(L), q0=0.0)
    for row in (0, 1, 19, 99, 199):
        for recall in (0.5, 0.95, 1.0):
            count, _ = oracle.weight_share(Q, K, SCALE, 0, row, 1, recall)
            assert count == math.ceil(recall * (row + 1) - 1e-9), (row, recall, count)


def test_one_dominant_key_is_enough():
    L = 128
    vals = np.zeros(L)
    vals[37] = 128.0  # logit 128 * scale = 11.3: weight e^11.3 against at most 127 ones
    Q, K = _inputs(L, vals)
    count, cum = oracle.weight_share(Q, K, SCALE, 0, 127, 1, 0.95)
    assert count == 1 and cum[0] > 0.95
    # before the dominant key appears, the row is uniform
    count, _ = oracle.weight_share(Q, K, SCALE, 0, 36, 1, 0.95)
    assert count == math.ceil(0.95 * 37)


def test_two_level_row_closed_form():
    """m keys of logit a, the rest of logit 0: the count follows from e^a and the total."""
    L = 256
    rng = np.random.default_rng(3)
    for m, val in ((5, 16.0), (20, 8.0), (3, 32.0), (60, 4.0)):
        vals = np.zeros(L)
        vals[rng.choice(L, m, replace=False)] = val
        Q, K = _inputs(L, vals)
        row = L - 1
        a = float(np.float32(val) * np.float32(SCALE))
        wa, wb = math.exp(a), 1.0
        total = m * wa + (row + 1 - m) * wb
        target = 0.95 * total
        if m * wa >= target:
            expect = math.ceil(target / wa - 1e-12)
        else:
            expect = m + math.ceil((target - m * wa) / wb - 1e-12)
        count, _ = oracle.weight_share(Q, K, SCALE, 0, row, 1, 0.95)
        assert count == expect, (m, val, count, expect)


def test_gqa_head_reads_its_kv_head():
    """Query head h reads KV head h // group: a dominant key planted in KV head 1 only."""
    L = 128
    Q = np.zeros((4, L, 128), np.float32)
    K = np.zeros((2, L, 128), np.float32)
    Q[:, :, 0] = 1.0
    K[1, 10, 0] = 128.0
    Qb, Kb = _bits(Q), _bits(K)
    assert oracle.weight_share(Qb, Kb, SCALE, 3, 127, 2, 0.95)[0] == 1
    assert oracle.weight_share(Qb, Kb, SCALE, 1, 127, 2, 0.95)[0] == math.ceil(0.95 * 128)
