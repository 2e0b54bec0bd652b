"""Pins of the backward-pass oracle against things other than itself (CPU only).

* central finite differences of the forward oracle (itself pinned by brute
  force in test_oracle.py): every gradient entry of a tiny block, for several t;
* torch autograd through torch's own tanh GeLU in float64 (a library routine);
* the closed form of the purely linear block: dx = dy W2 W1, dW1 = (dy W2)^T x,
  dW2 = dy^T (x W1^T);
* the identity g'(z) + g'(-z) = 1, the derivative of gelu(z) - gelu(-z) = z;
* the result does not depend on t, and the backward exchange is one [T, H]
  partial per shard;
* planted mistakes (in the oracle, on the CPU) that these pins must catch.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import tp_backward

pytestmark = pytest.mark.filterwarnings("ignore::DeprecationWarning")

T, H, F = 3, 5, 8
EPS = 1e-6


def _tiny(seed):
    rng = np.random.default_rng(seed)
    return {"x": rng.normal(0.0, 1.0, (T, H)), "w1": rng.normal(0.0, 0.5, (F, H)),
            "b1": rng.normal(0.0, 0.3, F), "w2": rng.normal(0.0, 0.5, (H, F)),
            "b2": rng.normal(0.0, 0.3, H), "dy": rng.normal(0.0, 1.0, (T, H))}


def _loss(p, t, act):
    y = oracle.mlp_block(p["x"], p["w1"], p["b1"], p["w2"], p["b2"], t, act)
    return float(np.sum(p["dy"] * y))


def _central_differences(p, t, act):
    """dL/dparam for L = sum(dy * y), one entry at a time, by central differences."""
    out = {}
    for name in ("x", "w1", "b1", "w2", "b2"):
        g = np.empty_like(p[name])
        for idx in np.ndindex(p[name].shape):
            q = {k: v.copy() for k, v in p.items()}
            q[name][idx] += EPS
            up = _loss(q, t, act)
            q[name][idx] -= 2 * EPS
            g[idx] = (up - _loss(q, t, act)) / (2 * EPS)
        out[name] = g
    return out


@pytest.mark.parametrize("act", ["gelu_tanh", "none"])
@pytest.mark.parametrize("t", [1, 2, 4])
def test_backward_matches_central_differences(t, act):
    p = _tiny(100 + t)
    g = oracle.mlp_block_backward(p["x"], p["w1"], p["b1"], p["w2"], p["dy"], t, act)
    fd = _central_differences(p, t, act)
    for mine, ref in (("dx", "x"), ("dw1", "w1"), ("db1", "b1"), ("dw2", "w2"), ("db2", "b2")):
        np.testing.assert_allclose(g[mine], fd[ref], rtol=1e-6, atol=1e-7, err_msg=mine)


def test_gelu_grad_matches_central_differences():
    z = np.linspace(-8.0, 8.0, 2001)
    fd = (oracle.gelu_tanh(z + EPS) - oracle.gelu_tanh(z - EPS)) / (2 * EPS)
    np.testing.assert_allclose(oracle.gelu_tanh_grad(z), fd, rtol=0, atol=1e-8)


def test_gelu_grad_matches_torch_autograd_fp64():
    z = torch.linspace(-8.0, 8.0, 4001, dtype=torch.float64, requires_grad=True)
    torch.nn.functional.gelu(z, approximate="tanh").sum().backward()
    np.testing.assert_allclose(oracle.gelu_tanh_grad(z.detach().numpy()), z.grad.numpy(),
                               rtol=0, atol=1e-14)


def test_gelu_grad_identities():
    z = np.linspace(-10.0, 10.0, 1001)
    g = oracle.gelu_tanh_grad
    np.testing.assert_allclose(g(z) + g(-z), 1.0, rtol=0, atol=1e-14)
    assert g(np.array([0.0]))[0] == 0.5
    # far from zero the GeLU is the identity or zero
    np.testing.assert_allclose(g(np.array([12.0, -12.0])), [1.0, 0.0], atol=1e-12)


def test_block_backward_matches_torch_autograd_fp64():
    p = _tiny(200)
    tp = {k: torch.tensor(v, dtype=torch.float64, requires_grad=True) for k, v in p.items()}
    z = tp["x"] @ tp["w1"].T + tp["b1"]
    y = torch.nn.functional.gelu(z, approximate="tanh") @ tp["w2"].T + tp["b2"]
    (y * tp["dy"]).sum().backward()
    g = oracle.mlp_block_backward(p["x"], p["w1"], p["b1"], p["w2"], p["dy"], 4, "gelu_tanh")
    for mine, ref in (("dx", "x"), ("dw1", "w1"), ("db1", "b1"), ("dw2", "w2"), ("db2", "b2")):
        np.testing.assert_allclose(g[mine], tp[ref].grad.numpy(), rtol=1e-12, atol=1e-13,
                                   err_msg=mine)


def test_linear_block_closed_form():
    p = _tiny(300)
    x, w1, w2, dy = p["x"], p["w1"], p["w2"], p["dy"]
    g = oracle.mlp_block_backward(x, w1, None, w2, dy, 2, "none")
    np.testing.assert_allclose(g["dx"], dy @ w2 @ w1, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(g["dw1"], (dy @ w2).T @ x, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(g["dw2"], dy.T @ (x @ w1.T), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(g["db1"], (dy @ w2).sum(axis=0), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(g["db2"], dy.sum(axis=0), rtol=0, atol=1e-15)


def test_backward_independent_of_tp_degree():
    rng = np.random.default_rng(400)
    x, dy = rng.normal(size=(6, 16)), rng.normal(size=(6, 16))
    w1, w2 = rng.normal(0, 0.3, (64, 16)), rng.normal(0, 0.3, (16, 64))
    b1 = rng.normal(0, 0.1, 64)
    ref = oracle.mlp_block_backward(x, w1, b1, w2, dy, 1)
    for t in (2, 4, 8, 16):
        g = oracle.mlp_block_backward(x, w1, b1, w2, dy, t)
        # equal up to rounding order: dx is a sum over shards, and the library
        # matmul blocks the weight-gradient slices differently from the whole
        for k in ("dx", "dw1", "db1", "dw2", "db2"):
            np.testing.assert_allclose(g[k], ref[k], rtol=1e-12, atol=1e-13, err_msg=k)


def test_backward_exchange_is_one_token_by_hidden_partial_per_shard():
    # the one backward exchange of the MLP carries, per shard, a [T, H]
    # partial: H * 2 bytes per token in 16-bit, the same 16 KB per token at
    # H = 8192 as the forward all-reduce
    p = _tiny(500)
    g = oracle.mlp_block_backward(p["x"], p["w1"], p["b1"], p["w2"], p["dy"], 4)
    assert len(g["dx_partials"]) == 4
    assert all(d.shape == (T, H) for d in g["dx_partials"])
    np.testing.assert_allclose(sum(g["dx_partials"]), g["dx"], rtol=1e-14, atol=1e-15)


def test_backward_accepts_bf16_torch_tensors_exactly():
    p = _tiny(600)
    tb = {k: torch.tensor(v).to(torch.bfloat16) for k, v in p.items()}
    exact = {k: v.to(torch.float64).numpy() for k, v in tb.items()}
    g = oracle.mlp_block_backward(tb["x"], tb["w1"], tb["b1"], tb["w2"], tb["dy"], 2)
    e = oracle.mlp_block_backward(exact["x"], exact["w1"], exact["b1"], exact["w2"],
                                  exact["dy"], 2)
    for k in ("dx", "dw1", "db1", "dw2", "db2"):
        np.testing.assert_array_equal(g[k], e[k])


def test_backward_rejects_mismatched_shapes():
    p = _tiny(700)
    with pytest.raises(ValueError):
        oracle.mlp_block_backward(p["x"], p["w1"], None, p["w2"].T, p["dy"], 2)
    with pytest.raises(ValueError):
        oracle.mlp_block_backward(p["x"], p["w1"], None, p["w2"], p["dy"], 3)


# ---------------------------------------------------------------- planted mistakes

def _pins_fail(monkeypatch, name, bad):
    """Plant ``bad`` in the backward oracle and count the pins that catch it."""
    monkeypatch.setattr(tp_backward, name, bad)
    checks = [lambda: test_backward_matches_central_differences(2, "gelu_tanh"),
              lambda: test_backward_matches_central_differences(4, "none"),
              test_block_backward_matches_torch_autograd_fp64,
              test_gelu_grad_matches_torch_autograd_fp64,
              test_gelu_grad_identities,
              test_linear_block_closed_form]
    caught = 0
    for c in checks:
        try:
            c()
        except (AssertionError, ValueError, IndexError):
            caught += 1
    return caught


def test_planted_dropped_gelu_derivative_term_is_caught(monkeypatch):
    def bad(z):  # only the first product-rule term
        z = np.asarray(z, dtype=np.float64)
        th = np.tanh(oracle.tp_oracle.SQRT_2_OVER_PI * (z + oracle.tp_oracle.GELU_CUBIC * z ** 3))
        return 0.5 * (1.0 + th)
    monkeypatch.setattr(oracle, "gelu_tanh_grad", bad)
    assert _pins_fail(monkeypatch, "gelu_tanh_grad", bad) >= 3


def test_planted_missing_backward_sum_is_caught(monkeypatch):
    def bad(partials, b):  # only the local shard's term, as if the all-reduce were skipped
        return partials[0].copy()
    assert _pins_fail(monkeypatch, "shard_sum", bad) >= 2


def test_planted_transposed_weight_gradient_is_caught(monkeypatch):
    real = tp_backward.mlp_block_backward

    def bad(x, w1, b1, w2, dy, t, act="gelu_tanh"):
        g = real(x, w1, b1, w2, dy, t, act)
        # dW2 taken as h^T dy ([F, H]) and forced back into the [H, F] layout
        g["dw2"] = g["dw2"].T.reshape(g["dw2"].shape)
        return g
    monkeypatch.setattr(oracle, "mlp_block_backward", bad)
    assert _pins_fail(monkeypatch, "mlp_block_backward", bad) >= 2


def test_planted_wrong_sign_is_caught(monkeypatch):
    def bad(z, act):
        return -tp_backward.gelu_tanh_grad(z) if act == "gelu_tanh" else -np.ones_like(z)
    assert _pins_fail(monkeypatch, "act_grad", bad) >= 2
