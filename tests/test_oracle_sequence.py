"""Pins of the sequence-parallel oracle (oracle/tp_sequence.py), on the CPU.

Nothing here trusts the oracle's own formula: RMSNorm is checked against
torch's rms_norm in float64 and against math.fsum brute force; the
reduce-scatter / all-gather pair against the all-reduce it replaces; and
closed-form properties (unit root-mean-square output, invariance to positive
scaling, independence from t).  Planted mistakes must fail the pins.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import tp_sequence


def _rng(seed):
    return np.random.default_rng(seed)


def _partials(T, H, K, t, seed):
    r = _rng(seed)
    h = r.standard_normal((T, K))
    w = r.standard_normal((H, K)) * 0.1
    return oracle.rowpar_partials(h, w, t)


def test_rms_norm_matches_torch_fp64():
    r = _rng(1)
    x = r.standard_normal((7, 96)) * 3.0
    g = r.standard_normal(96)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x), (96,), torch.from_numpy(g),
                                       eps=1e-5).numpy()
    np.testing.assert_allclose(oracle.rms_norm(x, g, 1e-5), ref, rtol=1e-13, atol=1e-13)


def test_rms_norm_brute_force_fsum():
    x = [[0.5, -1.25, 2.0, 0.125], [3.0, 0.0, -0.75, 1.5]]
    g = [1.0, 2.0, -0.5, 0.25]
    eps = 1e-5
    out = oracle.rms_norm(np.array(x), np.array(g), eps)
    for i, row in enumerate(x):
        ms = math.fsum(v * v for v in row) / len(row)
        for j, v in enumerate(row):
            assert out[i, j] == pytest.approx(v / math.sqrt(ms + eps) * g[j], rel=1e-14)


def test_rms_norm_closed_forms():
    r = _rng(2)
    x = r.standard_normal((5, 64)) + 0.3
    ones = np.ones(64)
    n = oracle.rms_norm(x, ones, 0.0)
    np.testing.assert_allclose(np.sqrt((n * n).mean(axis=1)), 1.0, rtol=1e-14)
    # invariant to scaling a row by c > 0 when eps = 0
    np.testing.assert_allclose(oracle.rms_norm(x * 7.5, ones, 0.0), n, rtol=1e-13)


@pytest.mark.parametrize("t", [1, 2, 4, 8])
def test_reduce_scatter_then_all_gather_is_the_all_reduce(t):
    T, H, K = 16, 24, 64
    parts = _partials(T, H, K, 8, 3)   # 8 row-parallel shards of K
    b = _rng(4).standard_normal(H)
    pieces = oracle.reduce_scatter(parts, b, t)
    assert len(pieces) == t and all(p.shape == (T // t, H) for p in pieces)
    np.testing.assert_array_equal(oracle.all_gather(pieces), oracle.shard_sum(parts, b))


def test_sp_region_equals_plain_residual_and_norm_for_every_t():
    T, H, K = 24, 32, 128
    parts = _partials(T, H, K, 4, 5)
    r = _rng(6)
    b = r.standard_normal(H) * 0.1
    res = r.standard_normal((T, H))
    g = r.standard_normal(H)
    y = oracle.shard_sum(parts, b)
    for t in (1, 2, 3, 4, 6, 8):
        rr, nn = oracle.sp_residual_norm(parts, b, res, g, t)
        np.testing.assert_array_equal(rr, res + y)
        np.testing.assert_allclose(nn, oracle.rms_norm(res + y, g), rtol=1e-14, atol=1e-15)


def test_token_shards_reject_uneven_split():
    assert oracle.token_shards(12, 4) == [(0, 3), (3, 6), (6, 9), (9, 12)]
    with pytest.raises(ValueError):
        oracle.token_shards(10, 4)


def _torch_region(parts, b, res, g):
    """The region's (r, n) from torch's rms_norm and the plain all-reduce."""
    r = res + oracle.shard_sum(parts, b)
    n = torch.nn.functional.rms_norm(torch.from_numpy(r), (r.shape[1],), torch.from_numpy(g),
                                     eps=1e-5).numpy()
    return r, n


def test_region_matches_torch_reference():
    rng = _rng(9)
    parts = _partials(8, 32, 64, 2, 10)
    res, g = rng.standard_normal((8, 32)), rng.standard_normal(32)
    rr, nn = oracle.sp_residual_norm(parts, None, res, g, 4)
    r_ref, n_ref = _torch_region(parts, None, res, g)
    np.testing.assert_array_equal(rr, r_ref)
    np.testing.assert_allclose(nn, n_ref, rtol=1e-13, atol=1e-13)


def test_planted_mistakes_are_caught(monkeypatch):
    # each mistake is planted in the oracle's own norm; the region it feeds must
    # then disagree with the torch reference
    rng = _rng(7)
    parts = _partials(8, 32, 64, 2, 11)
    res, g = rng.standard_normal((8, 32)), rng.standard_normal(32)
    r_ref, n_ref = _torch_region(parts, None, res, g)

    def sum_not_mean(rr, gg, eps=1e-5):
        rf = np.asarray(rr, float)
        return rf / np.sqrt((rf * rf).sum(axis=1, keepdims=True) + eps) * np.asarray(gg)[None]

    def no_gamma(rr, gg, eps=1e-5):
        rf = np.asarray(rr, float)
        return rf / np.sqrt((rf * rf).mean(axis=1, keepdims=True) + eps)

    def eps_outside(rr, gg, eps=1e-5):
        rf = np.asarray(rr, float)
        return rf / (np.sqrt((rf * rf).mean(axis=1, keepdims=True)) + 0.1) * np.asarray(gg)[None]

    for bad in (sum_not_mean, no_gamma, eps_outside):
        monkeypatch.setattr(tp_sequence, "rms_norm", bad)
        _, nn = oracle.sp_residual_norm(parts, None, res, g, 2)
        assert not np.allclose(nn, n_ref, rtol=1e-6, atol=1e-8), bad.__name__
    monkeypatch.undo()

    # a forgotten residual, and a shard's rows summed from the wrong partials
    real_rs = tp_sequence.reduce_scatter
    monkeypatch.setattr(tp_sequence, "reduce_scatter", lambda p, b, t: real_rs(p[:-1], b, t))
    rr, _ = oracle.sp_residual_norm(parts, None, res, g, 2)
    assert not np.allclose(rr, r_ref)
    monkeypatch.undo()
    rr, _ = oracle.sp_residual_norm(parts, None, np.zeros_like(res), g, 2)
    assert not np.allclose(rr, r_ref)
