"""The rotary-structured input variant: noise-free rows under the rotary embedding have dot
products that depend on the two positions only through their offset; with noise, the logits of
the last query fall with the distance to the key; the default draw is unchanged."""
import ctypes

import numpy as np
import pytest

import workload
from workload import TEXT, Head, Problem, bf16_to_f32, make_inputs


def _rows(n, d=128, shared_scale=4.0, base=1.0e4, noise=0.0, seed=3):
    lib = workload._load()
    w = workload.unit_vector(seed, d, workload.U_STREAM + 1)
    out = np.empty((n, d), np.uint16)
    lib.wl_fill_rope_bf16(out.ctypes.data, n, d, seed, 5, noise, w.ctypes.data, shared_scale, base, None, None, 0.0)
    return bf16_to_f32(out).astype(np.float64), w.astype(np.float64)


def test_noise_free_dots_depend_on_offset_only():
    x, w = _rows(512)
    g = x @ x.T
    # offset t between rows: the same dot for every pair at that offset (up to bf16 rounding of
    # the rotated rows: relative 2^-8 per element)
    for t in (0, 1, 7, 100, 300):
        diag = np.array([g[i, i + t] for i in range(0, 512 - t)])
        assert np.all(np.abs(diag - diag[0]) <= 0.05 * 16.0), (t, diag.min(), diag.max())
    # offset 0: |row|^2 = shared_scale^2 (rotation keeps norms)
    assert abs(g[0, 0] - 16.0) < 0.1 and abs(g[200, 200] - 16.0) < 0.1
    # row 0 is not rotated: it is shared_scale * w rounded to bf16
    assert np.allclose(x[0], 4.0 * w, atol=4.0 * np.abs(w).max() * 2 ** -8)


def test_rotation_follows_the_pair_layout():
    # one shared unit vector along dimension 0: row r is (cos(r), 0, .., sin(r), 0, ..) at base^0
    lib = workload._load()
    e = np.zeros(128, np.float32)
    e[0] = 1.0
    out = np.empty((8, 128), np.uint16)
    lib.wl_fill_rope_bf16(out.ctypes.data, 8, 128, 1, 5, 0.0, e.ctypes.data, 1.0, 1.0e4, None, None, 0.0)
    x = bf16_to_f32(out)
    r = np.arange(8)
    np.testing.assert_allclose(x[:, 0], np.cos(r), atol=2 ** -8)
    np.testing.assert_allclose(x[:, 64], np.sin(r), atol=2 ** -8)
    assert np.all(x[:, 1:64] == 0) and np.all(x[:, 65:] == 0)


def test_logits_fall_with_distance_and_default_is_unchanged():
    p = Problem(L=2048, Hq=1, Hkv=1, segments=[(0, 2048, TEXT)], heads=[Head("vslash", k_v=8, k_s=8)])
    Q, K, V = make_inputs(p, seed=2, inputs="rope")
    q = bf16_to_f32(Q[0]).astype(np.float64)
    k = bf16_to_f32(K[0]).astype(np.float64)
    s = q[-64:] @ k.T / np.sqrt(128.0)
    by_off = np.array([np.mean([s[r, 1984 + r - o] for r in range(64)]) for o in (0, 8, 64, 512, 1900)])
    assert by_off[0] > by_off[1] > by_off[3] > by_off[4], by_off
    Q0, K0, V0 = make_inputs(p, seed=2)
    Qi, Ki, Vi = make_inputs(p, seed=2, inputs="iid")
    assert np.array_equal(Q0, Qi) and np.array_equal(K0, Ki) and np.array_equal(V0, Vi)
    assert np.array_equal(V0, V)  # V carries no position structure
    with pytest.raises(ValueError):
        make_inputs(p, seed=2, inputs="other")
