"""Pins of the attention-core oracle against things other than itself (CPU only).

* pure-Python brute force (math.exp, math.fsum) on tiny inputs;
* torch's scaled_dot_product_attention in float64 (a library routine), causal
  prefill and decode over a cache;
* special cases: a single visible key returns its value; equal scores return
  the mean of the visible values;
* the cache: prefill in chunks, carrying each shard's cache, equals one-shot
  prefill; the grown cache holds exactly the new keys and values;
* independence from t (each query head's key-value head is on its shard);
* planted mistakes (in the oracle, on the CPU) that these pins must catch.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import tp_attention

pytestmark = pytest.mark.filterwarnings("ignore::DeprecationWarning")

NQ, NKV, D = 8, 4, 4


def _qkv(T, seed, nq=NQ, nkv=NKV, d=D, scale=1.0):
    return np.random.default_rng(seed).normal(0.0, scale, (T, (nq + 2 * nkv) * d))


def _heads(qkv, nq, nkv, d):
    T = qkv.shape[0]
    q = qkv[:, : nq * d].reshape(T, nq, d)
    k = qkv[:, nq * d:(nq + nkv) * d].reshape(T, nkv, d)
    v = qkv[:, (nq + nkv) * d:].reshape(T, nkv, d)
    return q, k, v


def _bruteforce(qkv, nq, nkv, d):
    """Causal GQA attention with Python floats only, no cache."""
    q, k, v = _heads(qkv, nq, nkv, d)
    T = qkv.shape[0]
    out = np.empty((T, nq * d))
    for h in range(nq):
        g = h // (nq // nkv)
        for i in range(T):
            scores = [math.fsum(float(q[i, h, e]) * float(k[j, g, e]) for e in range(d))
                      / math.sqrt(d) for j in range(i + 1)]
            m = max(scores)
            w = [math.exp(s - m) for s in scores]
            z = math.fsum(w)
            for e in range(d):
                out[i, h * d + e] = math.fsum(w[j] * float(v[j, g, e]) for j in range(i + 1)) / z
    return out


def _torch_sdpa(qkv_all, nq, nkv, d, past):
    """torch SDPA in float64 for the last T - past tokens over all keys."""
    q, k, v = (torch.tensor(a).permute(1, 0, 2) for a in _heads(qkv_all, nq, nkv, d))
    rep = nq // nkv
    k, v = k.repeat_interleave(rep, 0), v.repeat_interleave(rep, 0)
    n = qkv_all.shape[0]
    qn = q[:, past:]
    mask = torch.ones(n - past, n, dtype=torch.bool).tril(diagonal=past)
    o = torch.nn.functional.scaled_dot_product_attention(qn, k, v, attn_mask=mask)
    return o.permute(1, 0, 2).reshape(n - past, nq * d).numpy()


@pytest.mark.parametrize("t", [1, 2, 4])
def test_attn_core_matches_bruteforce(t):
    qkv = _qkv(5, 10 + t)
    ctx, _ = oracle.attn_core(qkv, NQ, NKV, D, t)
    np.testing.assert_allclose(ctx, _bruteforce(qkv, NQ, NKV, D), rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("nq,nkv,d,t", [(8, 4, 4, 2), (8, 8, 8, 4), (16, 2, 8, 2), (4, 1, 16, 1)])
def test_attn_core_prefill_matches_torch_sdpa(nq, nkv, d, t):
    qkv = _qkv(9, 20 + nq + nkv, nq, nkv, d)
    ctx, _ = oracle.attn_core(qkv, nq, nkv, d, t)
    np.testing.assert_allclose(ctx, _torch_sdpa(qkv, nq, nkv, d, 0), rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("past,T", [(6, 1), (5, 3), (1, 4)])
def test_attn_core_decode_over_cache_matches_torch_sdpa(past, T):
    t = 2
    qkv_all = _qkv(past + T, 30 + past)
    _, cache = oracle.attn_core(qkv_all[:past], NQ, NKV, D, t)
    ctx, _ = oracle.attn_core(qkv_all[past:], NQ, NKV, D, t, cache)
    np.testing.assert_allclose(ctx, _torch_sdpa(qkv_all, NQ, NKV, D, past), rtol=1e-12,
                               atol=1e-13)


def test_chunked_prefill_through_the_cache_equals_one_shot():
    t = 4
    qkv = _qkv(11, 40)
    whole, whole_cache = oracle.attn_core(qkv, NQ, NKV, D, t)
    parts, cache = [], None
    for a, b in ((0, 3), (3, 4), (4, 11)):
        c, cache = oracle.attn_core(qkv[a:b], NQ, NKV, D, t, cache)
        parts.append(c)
    np.testing.assert_allclose(np.concatenate(parts), whole, rtol=1e-13, atol=1e-14)
    for (k1, v1), (k2, v2) in zip(cache, whole_cache):
        np.testing.assert_array_equal(k1, k2)
        np.testing.assert_array_equal(v1, v2)


def test_grown_cache_holds_each_shards_own_heads():
    t = 2
    qkv = _qkv(3, 50)
    _, cache = oracle.attn_core(qkv, NQ, NKV, D, t)
    _, k, v = _heads(qkv, NQ, NKV, D)
    kh = NKV // t
    for s, (ck, cv) in enumerate(cache):
        assert ck.shape == (kh, 3, D) and cv.shape == (kh, 3, D)
        np.testing.assert_array_equal(ck, k[:, s * kh:(s + 1) * kh].transpose(1, 0, 2))
        np.testing.assert_array_equal(cv, v[:, s * kh:(s + 1) * kh].transpose(1, 0, 2))


def test_first_token_sees_only_itself():
    qkv = _qkv(4, 60)
    ctx, _ = oracle.attn_core(qkv, NQ, NKV, D, 2)
    _, _, v = _heads(qkv, NQ, NKV, D)
    for h in range(NQ):
        np.testing.assert_allclose(ctx[0, h * D:(h + 1) * D], v[0, h // (NQ // NKV)],
                                   rtol=0, atol=1e-15)


def test_equal_scores_average_the_visible_values():
    # zero queries: every score is 0, so token i returns the mean of values 0..i
    qkv = _qkv(5, 70)
    qkv[:, : NQ * D] = 0.0
    ctx, _ = oracle.attn_core(qkv, NQ, NKV, D, 1)
    _, _, v = _heads(qkv, NQ, NKV, D)
    for i in range(5):
        for h in range(NQ):
            np.testing.assert_allclose(ctx[i, h * D:(h + 1) * D],
                                       v[: i + 1, h // (NQ // NKV)].mean(axis=0), atol=1e-15)


def test_attn_core_independent_of_tp_degree():
    qkv = _qkv(6, 80, 16, 8, 8)
    ref, _ = oracle.attn_core(qkv, 16, 8, 8, 1)
    for t in (2, 4, 8):
        ctx, _ = oracle.attn_core(qkv, 16, 8, 8, t)
        np.testing.assert_array_equal(ctx, ref)


def test_attn_core_large_scores_stay_finite():
    qkv = _qkv(7, 90, scale=30.0)
    ctx, _ = oracle.attn_core(qkv, NQ, NKV, D, 2)
    assert np.isfinite(ctx).all()
    np.testing.assert_allclose(ctx, _torch_sdpa(qkv, NQ, NKV, D, 0), rtol=1e-9, atol=1e-9)


def test_attn_core_rejects_bad_splits_and_caches():
    qkv = _qkv(2, 100)
    with pytest.raises(ValueError):
        oracle.attn_core(qkv, NQ, NKV, D, 3)
    with pytest.raises(ValueError):
        oracle.attn_core(qkv, NQ, NKV, D, 8)   # t > nkv would need replicated cache
    with pytest.raises(ValueError):
        oracle.attn_core(qkv, NQ, NKV, D, 2, oracle.empty_cache(4, NKV, D))
    with pytest.raises(ValueError):
        oracle.attn_core(qkv[:, :-1], NQ, NKV, D, 2)


# ---------------------------------------------------------------- planted mistakes

def _pins_fail(monkeypatch, name, bad):
    """Plant ``bad`` in the attention oracle and count the pins that catch it."""
    monkeypatch.setattr(tp_attention, name, bad)
    checks = [lambda: test_attn_core_matches_bruteforce(2),
              lambda: test_attn_core_prefill_matches_torch_sdpa(16, 2, 8, 2),
              lambda: test_attn_core_decode_over_cache_matches_torch_sdpa(5, 3),
              test_first_token_sees_only_itself,
              test_equal_scores_average_the_visible_values]
    caught = 0
    for c in checks:
        try:
            c()
        except (AssertionError, ValueError, IndexError):
            caught += 1
    return caught


def test_planted_missing_scale_is_caught(monkeypatch):
    def bad(q, k_all, v_all, past):
        T, d = q.shape
        out = np.empty((T, d))
        for i in range(T):
            s = k_all[: past + i + 1] @ q[i]
            p = np.exp(s - s.max())
            out[i] = (p / p.sum()) @ v_all[: past + i + 1]
        return out
    assert _pins_fail(monkeypatch, "attend_head", bad) >= 3


def test_planted_off_by_one_mask_is_caught(monkeypatch):
    def bad(q, k_all, v_all, past):
        T, d = q.shape
        out = np.empty((T, d))
        for i in range(T):
            n = max(1, past + i)          # a token does not see itself
            s = (k_all[:n] @ q[i]) / math.sqrt(d)
            p = np.exp(s - s.max())
            out[i] = (p / p.sum()) @ v_all[:n]
        return out
    assert _pins_fail(monkeypatch, "attend_head", bad) >= 3


def test_planted_wrong_kv_group_is_caught(monkeypatch):
    real_split = tp_attention._split_qkv

    def bad(qkv, nq, nkv, d):
        # a head-index slip: query heads paired with the wrong key-value heads
        # (query head h lands where head (h % nkv) * group + h // nkv belongs)
        q, k, v = real_split(qkv, nq, nkv, d)
        group = nq // nkv
        perm = [(h % nkv) * group + h // nkv for h in range(nq)]
        inv = np.argsort(perm)
        return q[inv], k, v
    assert _pins_fail(monkeypatch, "_split_qkv", bad) >= 2


def test_planted_dropped_cache_is_caught(monkeypatch):
    real = tp_attention.attn_core

    def bad(qkv, nq, nkv, d, t, cache=None):
        return real(qkv, nq, nkv, d, t, None)     # the earlier tokens are forgotten
    monkeypatch.setattr(oracle, "attn_core", bad)
    assert _pins_fail(monkeypatch, "attn_core", bad) >= 1
