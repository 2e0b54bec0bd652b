"""Pins of the fp64 oracle against things other than itself (CPU only).

* brute force: pure-Python ``math.fsum`` dot products on tiny inputs;
* GeLU: torch's own tanh-GeLU in float64 (an independent library routine), the
  erf GeLU x*Phi(x) it approximates (``math.erf``), and the odd-part identity
  gelu(z) - gelu(-z) = z that holds for any tanh form;
* invariants the method fixes: column shards side by side equal the unsplit
  layer, row-shard partials sum to the unsplit layer, for every t;
* special cases: identity weights, one-hot inputs, t = 1;
* the pages' printed shapes and head-divisibility rules (tests/golden);
* planted mistakes (in the oracle, on the CPU) that these pins must catch.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import tp_oracle
from workloads import random_bf16_small

pytestmark = pytest.mark.filterwarnings("ignore::DeprecationWarning")


def _bf16_np(shape, std, seed):
    return oracle.to_f64(random_bf16_small(shape, std, seed))


def _fsum_linear(x, w, b):
    """Reference-by-brute-force: y[r][j] = fsum_k x[r][k] w[j][k] (+ b[j])."""
    T, K = x.shape
    N = w.shape[0]
    y = np.empty((T, N))
    for r in range(T):
        for j in range(N):
            terms = [float(x[r, k]) * float(w[j, k]) for k in range(K)]
            if b is not None:
                terms.append(float(b[j]))
            y[r, j] = math.fsum(terms)
    return y


def _gelu_scalar(z):
    return 0.5 * z * (1.0 + math.tanh(math.sqrt(2.0 / math.pi) * (z + 0.044715 * z ** 3)))


def _divisors(n):
    return [d for d in range(1, n + 1) if n % d == 0]


def _close(a, b, scale, rel=1e-12):
    return np.all(np.abs(a - b) <= rel * scale)


# ---------------------------------------------------------------- brute force

def test_linear_matches_fsum_bruteforce():
    x = _bf16_np((3, 24), 1.0, 1)
    w = _bf16_np((10, 24), 0.02, 2)
    b = _bf16_np((10,), 0.01, 3)
    ref = _fsum_linear(x, w, b)
    got = oracle.linear(x, w, b)
    scale = np.abs(x) @ np.abs(w).T + np.abs(b)
    assert _close(got, ref, scale, 1e-14)


def test_linear_accepts_bf16_torch_tensors_exactly():
    xt = random_bf16_small((2, 16), 1.0, 4)
    wt = random_bf16_small((5, 16), 0.02, 5)
    got = oracle.linear(xt, wt)
    ref = _fsum_linear(xt.double().numpy(), wt.double().numpy(), None)
    assert np.allclose(got, ref, rtol=1e-14, atol=1e-16)


def test_mlp_block_matches_fsum_bruteforce():
    T, H, F, t = 3, 8, 16, 2
    x = _bf16_np((T, H), 1.0, 10)
    w1 = _bf16_np((F, H), 0.3, 11)
    b1 = _bf16_np((F,), 0.1, 12)
    w2 = _bf16_np((H, F), 0.3, 13)
    b2 = _bf16_np((H,), 0.1, 14)
    z = _fsum_linear(x, w1, b1)
    h = np.vectorize(_gelu_scalar)(z)
    y_ref = _fsum_linear(h, w2, b2)
    y = oracle.mlp_block(x, w1, b1, w2, b2, t, "gelu_tanh")
    assert np.allclose(y, y_ref, rtol=1e-13, atol=1e-15)


# ---------------------------------------------------------------- GeLU pins

def test_gelu_matches_torch_tanh_gelu_fp64():
    z = torch.linspace(-12.0, 12.0, 4801, dtype=torch.float64)
    ref = torch.nn.functional.gelu(z, approximate="tanh").numpy()
    got = oracle.gelu_tanh(z.numpy())
    # 1 + tanh(u) cancels for z << 0, so both sides are ~0 there within ~1e-15
    assert np.allclose(got, ref, rtol=1e-12, atol=2e-15)


def test_gelu_close_to_erf_gelu():
    # the tanh form approximates x * Phi(x); its worst-case gap is a few 1e-4
    zs = np.linspace(-8.0, 8.0, 3201)
    erf_gelu = np.array([0.5 * z * (1.0 + math.erf(z / math.sqrt(2.0))) for z in zs])
    gap = np.max(np.abs(oracle.gelu_tanh(zs) - erf_gelu))
    assert gap < 1e-3
    assert gap > 1e-5  # it is the tanh approximation, not the erf form itself


def test_gelu_identities():
    zs = np.linspace(-30.0, 30.0, 6001)
    g = oracle.gelu_tanh(zs)
    gm = oracle.gelu_tanh(-zs)
    assert np.allclose(g - gm, zs, rtol=1e-14, atol=1e-14)
    assert oracle.gelu_tanh(np.array([0.0]))[0] == 0.0
    assert abs(oracle.gelu_tanh(np.array([20.0]))[0] - 20.0) < 1e-12
    assert abs(oracle.gelu_tanh(np.array([-20.0]))[0]) < 1e-12
    # slope 1/2 at the origin
    e = 1e-6
    d = (oracle.gelu_tanh(np.array([e]))[0] - oracle.gelu_tanh(np.array([-e]))[0]) / (2 * e)
    assert abs(d - 0.5) < 1e-9


# ---------------------------------------------------------------- invariants

@pytest.mark.parametrize("act", ["none", "gelu_tanh"])
def test_column_shards_side_by_side_equal_unsplit(act):
    x = _bf16_np((5, 32), 1.0, 20)
    w = _bf16_np((48, 32), 0.1, 21)
    b = _bf16_np((48,), 0.05, 22)
    full = oracle.apply_act(oracle.linear(x, w, b), act)
    for t in _divisors(48):
        got = oracle.colpar_linear(x, w, b, t, act)
        assert got.shape == full.shape
        assert np.allclose(got, full, rtol=1e-13, atol=1e-15), t


def test_row_shard_partials_sum_to_unsplit():
    h = _bf16_np((4, 96), 1.0, 30)
    w = _bf16_np((20, 96), 0.1, 31)
    b = _bf16_np((20,), 0.05, 32)
    full = oracle.linear(h, w, b)
    scale = np.abs(h) @ np.abs(w).T + np.abs(b)
    for t in _divisors(96):
        parts = oracle.rowpar_partials(h, w, t)
        assert len(parts) == t and all(p.shape == full.shape for p in parts)
        got = oracle.rowpar_linear(h, w, b, t)
        assert _close(got, full, scale, 1e-13), t


def test_mlp_block_independent_of_tp_degree():
    T, H, F = 3, 16, 64
    x = _bf16_np((T, H), 1.0, 40)
    w1 = _bf16_np((F, H), 0.2, 41)
    b1 = _bf16_np((F,), 0.05, 42)
    w2 = _bf16_np((H, F), 0.2, 43)
    b2 = _bf16_np((H,), 0.05, 44)
    ref = oracle.mlp_block(x, w1, b1, w2, b2, 1)
    for t in _divisors(F):
        assert np.allclose(oracle.mlp_block(x, w1, b1, w2, b2, t), ref, rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------- special cases

def test_identity_first_layer_reduces_to_second_linear():
    T, H = 4, 16
    x = _bf16_np((T, H), 1.0, 50)
    w2 = _bf16_np((H, H), 0.2, 51)
    b2 = _bf16_np((H,), 0.05, 52)
    eye = np.eye(H)
    for t in (1, 2, 4, 8, 16):
        y = oracle.mlp_block(x, eye, None, w2, b2, t, "none")
        assert np.allclose(y, _fsum_linear(x, w2, b2), rtol=1e-14, atol=1e-15)


def test_one_hot_input_selects_weight_column():
    H, F = 12, 20
    w1 = _bf16_np((F, H), 0.3, 60)
    b1 = _bf16_np((F,), 0.1, 61)
    for k in range(H):
        x = np.zeros((1, H))
        x[0, k] = 1.0
        z = oracle.colpar_linear(x, w1, b1, 4, "none")
        assert np.array_equal(z[0], w1[:, k] + b1)


def test_tp1_is_plain_linear():
    x = _bf16_np((3, 40), 1.0, 70)
    w = _bf16_np((24, 40), 0.1, 71)
    assert np.array_equal(oracle.colpar_linear(x, w, None, 1), oracle.linear(x, w))
    assert np.array_equal(oracle.rowpar_linear(x, w, None, 1), oracle.linear(x, w))


def test_shard_ranges_reject_uneven_split():
    with pytest.raises(ValueError):
        oracle.shard_ranges(10, 3)
    with pytest.raises(ValueError):
        oracle.shard_ranges(10, 0)


# ---------------------------------------------------------------- attention

def test_qkv_head_shards_partition_columns():
    nq, nkv, d = 8, 4, 4
    n = (nq + 2 * nkv) * d
    for t in (1, 2, 4):
        seen = np.concatenate([oracle.qkv_shard_columns(nq, nkv, d, t, s) for s in range(t)])
        assert sorted(seen.tolist()) == list(range(n))
        for s in range(t):
            cols = oracle.qkv_shard_columns(nq, nkv, d, t, s)
            assert len(cols) == (nq // t + 2 * nkv // t) * d
            # shard s holds its own query heads and its own key/value heads
            assert cols[0] == s * (nq // t) * d


def test_attn_projections_match_bruteforce():
    nq, nkv, d, H, T = 8, 2, 4, 16, 3
    x = _bf16_np((T, H), 1.0, 80)
    w_qkv = _bf16_np(((nq + 2 * nkv) * d, H), 0.2, 81)
    b_qkv = _bf16_np(((nq + 2 * nkv) * d,), 0.05, 82)
    ctx = _bf16_np((T, nq * d), 1.0, 83)
    w_o = _bf16_np((H, nq * d), 0.2, 84)
    b_o = _bf16_np((H,), 0.05, 85)
    q_ref = _fsum_linear(x, w_qkv, b_qkv)
    o_ref = _fsum_linear(ctx, w_o, b_o)
    for t in (1, 2):
        assert np.allclose(oracle.attn_qkv(x, w_qkv, b_qkv, nq, nkv, d, t), q_ref, rtol=1e-13, atol=1e-15)
        assert np.allclose(oracle.attn_out(ctx, w_o, b_o, nq, d, t), o_ref, rtol=1e-13, atol=1e-15)


# ---------------------------------------------------------------- the pages' printed values

def test_pages_tp2_split_shapes(golden):
    g = golden["tp2_column_split"]
    n_in, n_out = g["weight_math_shape_in_out"]
    ranges = oracle.shard_ranges(n_out, g["tp_degree"])
    assert len(ranges) == g["tp_degree"]
    for (j0, j1) in ranges:
        assert [n_in, j1 - j0] == g["shard_math_shape_in_out"]
        assert [j1 - j0, n_in] == g["shard_stored_shape_out_in"]


def test_pages_head_divisibility(golden):
    g = golden["head_divisibility"]
    for t in g["tp_degrees_that_work"]:
        assert oracle.heads_divisible(g["n_q_heads"], g["n_kv_heads"], t)
    for t in g["tp_degrees_that_fail"]:
        assert not oracle.heads_divisible(g["n_q_heads"], g["n_kv_heads"], t)


def test_pages_exchange_sizes_match_block_shapes(golden):
    # the row-parallel partial of one token is one hidden-size vector: that is
    # what the all-reduce carries per token
    g = golden["llama70b_exchange"]
    H = g["hidden"]
    h = np.ones((1, 64))
    w2 = np.ones((H, 64))
    parts = oracle.rowpar_partials(h, w2, 8)
    assert parts[0].shape == (1, H)
    assert parts[0].shape[1] * g["bytes_per_element"] == g["decode_message_bytes_per_token"]
    assert g["layers"] * g["all_reduces_per_layer_forward"] == g["all_reduces_per_forward"]
    g405 = golden["llama405b_vector"]
    from workloads import CONFIGS
    assert CONFIGS["mlp405b"].hidden * g405["bytes_per_element"] == g405["bytes_per_token_vector"]
    assert CONFIGS["mlp70b"].hidden == H
    assert CONFIGS["attn70b"].n_q_heads == golden["head_divisibility"]["n_q_heads"]
    assert CONFIGS["attn70b"].n_kv_heads == golden["head_divisibility"]["n_kv_heads"]


# ---------------------------------------------------------------- planted mistakes

def _pins_fail(monkeypatch, name, bad):
    """Plant ``bad`` in the oracle module and report whether a pin catches it."""
    monkeypatch.setattr(tp_oracle, name, bad)
    monkeypatch.setattr(oracle, name, bad, raising=False)
    checks = [test_linear_matches_fsum_bruteforce, test_mlp_block_matches_fsum_bruteforce,
              test_gelu_matches_torch_tanh_gelu_fp64, test_gelu_close_to_erf_gelu,
              test_gelu_identities, test_row_shard_partials_sum_to_unsplit,
              test_attn_projections_match_bruteforce]
    caught = 0
    for c in checks:
        try:
            c()
        except (AssertionError, ValueError, IndexError):
            caught += 1
    return caught


def test_planted_wrong_gelu_constant_is_caught(monkeypatch):
    def bad(z):
        z = np.asarray(z, dtype=np.float64)
        return 0.5 * z * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (z + 0.44715 * z ** 3)))
    assert _pins_fail(monkeypatch, "gelu_tanh", bad) >= 2


def test_planted_transposed_operand_is_caught(monkeypatch):
    real = tp_oracle.linear

    def bad(x, w, b=None):
        xf = oracle.to_f64(x)
        wf = oracle.to_f64(w)
        if wf.shape[0] == wf.shape[1]:
            wf = wf.T
        else:  # a plausible slip: reduce against the wrong axis of a reshaped weight
            wf = wf.reshape(wf.shape[1], wf.shape[0]).T
        y = xf @ wf.T
        return y if b is None else y + oracle.to_f64(b)[None, :]
    assert _pins_fail(monkeypatch, "linear", bad) >= 2
    assert tp_oracle.linear is bad
    monkeypatch.setattr(tp_oracle, "linear", real)


def test_planted_dropped_bias_is_caught(monkeypatch):
    def bad(partials, b):
        y = np.zeros_like(partials[0])
        for p in partials:
            y = y + p
        return y
    assert _pins_fail(monkeypatch, "shard_sum", bad) >= 1


def test_planted_dropped_partial_is_caught(monkeypatch):
    def bad(partials, b):
        y = np.zeros_like(partials[0])
        for p in partials[:-1]:
            y = y + p
        return y if b is None else y + oracle.to_f64(b)[None, :]
    assert _pins_fail(monkeypatch, "shard_sum", bad) >= 1


# ---------------------------------------------------------------- 8-bit weights

def _e4m3_codes(shape, seed):
    """Random finite E4M3 codes of both signs (NaN codes 0x7F / 0xFF excluded)."""
    g = torch.Generator().manual_seed(seed)
    mag = torch.randint(0, 0x7F, shape, generator=g, dtype=torch.int32)
    sign = torch.randint(0, 2, shape, generator=g, dtype=torch.int32) * 0x80
    return (mag | sign).to(torch.uint8)


def test_e4m3_landmark_values():
    # the E4M3 format's own landmarks: 1.0, the largest finite value 448, the
    # smallest normal 2^-6, the smallest subnormal 2^-9, and the NaN codes
    t = oracle.E4M3_TABLE
    assert t[0x38] == 1.0 and t[0xB8] == -1.0
    assert t[0x7E] == 448.0 and t[0xFE] == -448.0
    assert t[0x08] == 2.0 ** -6 and t[0x01] == 2.0 ** -9 and t[0x07] == 7 * 2.0 ** -9
    assert t[0x00] == 0.0 and math.copysign(1.0, t[0x80]) == -1.0
    assert math.isnan(t[0x7F]) and math.isnan(t[0xFF])
    pos = t[:0x7F]
    assert np.all(np.diff(pos) > 0)                 # codes 0..0x7E increase strictly
    assert np.array_equal(t[0x80:0xFF], -pos)       # the sign bit only negates


def test_e4m3_table_matches_torch_float8():
    # an independent decoder: torch's float8_e4m3fn
    ref = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn)
    ref = ref.to(torch.float64).numpy()
    t = oracle.E4M3_TABLE
    assert np.array_equal(np.isnan(ref), np.isnan(t))
    assert np.array_equal(ref[~np.isnan(ref)], t[~np.isnan(t)])


def test_w8_linear_matches_fsum_bruteforce():
    q = _e4m3_codes((6, 40), 11)
    sc = torch.rand(6, generator=torch.Generator().manual_seed(12)) * 0.01 + 1e-3
    x = _bf16_np((3, 40), 1.0, 13)
    b = _bf16_np((6,), 0.1, 14)
    w = np.array([[sc[n].item() * oracle.e4m3_value(int(q[n, k])) for k in range(40)]
                  for n in range(6)])
    got = oracle.linear(x, oracle.E4M3Weight(q, sc), b)
    assert _close(got, _fsum_linear(x, w, b), np.abs(got).max() + 1.0)


def test_w8_shards_equal_the_dequantised_weight():
    # column and row shards of an 8-bit weight slice codes and scales together
    q = _e4m3_codes((48, 64), 21)
    sc = torch.rand(48, generator=torch.Generator().manual_seed(22)) * 0.01
    wd = q.view(torch.float8_e4m3fn).to(torch.float64) * sc.to(torch.float64)[:, None]
    x = _bf16_np((5, 64), 1.0, 23)
    w8 = oracle.E4M3Weight(q, sc)
    for t in (1, 2, 4):
        a = oracle.colpar_linear(x, w8, None, t, "gelu_tanh")
        b = oracle.colpar_linear(x, wd.numpy(), None, t, "gelu_tanh")
        assert _close(a, b, np.abs(b).max() + 1.0)
        h = _bf16_np((5, 48), 1.0, 24 + t)
        wr = oracle.E4M3Weight(q.T.contiguous(), torch.ones(64))
        a = oracle.rowpar_linear(h, wr, None, t)
        b = oracle.rowpar_linear(h, q.T.contiguous().view(torch.float8_e4m3fn)
                                 .to(torch.float64).numpy(), None, t)
        assert _close(a, b, np.abs(b).max() + 1.0)


def test_planted_wrong_e4m3_bias_is_caught(monkeypatch):
    def bad_value(code):
        e = (code >> 3) & 0xF
        m = code & 0x7
        sign = -1.0 if code & 0x80 else 1.0
        if e == 0xF and m == 0x7:
            return math.nan
        if e == 0:
            return sign * (m / 8.0) * 2.0 ** -7
        return sign * (1.0 + m / 8.0) * 2.0 ** (e - 8)     # exponent bias 8, not 7
    bad = np.array([bad_value(c) for c in range(256)])
    monkeypatch.setattr(tp_oracle, "E4M3_TABLE", bad)
    monkeypatch.setattr(oracle, "E4M3_TABLE", bad)
    caught = 0
    for c in (test_e4m3_landmark_values, test_e4m3_table_matches_torch_float8,
              test_w8_shards_equal_the_dequantised_weight):
        try:
            c()
        except AssertionError:
            caught += 1
    assert caught >= 2
