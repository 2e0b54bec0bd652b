"""fp64 CPU oracle of the tensor-parallel MLP block's backward pass.

TEST INFRASTRUCTURE ONLY, under the same rules as ``tp_oracle``: only the tests,
the package's ``smoke()`` entry and the benchmark's CPU-baseline / reference leg
may import it; no CUDA code imports or links it.

What it computes: for the block y = sum_s act(x W1_s^T + b1_s) W2[:, K_s]^T + b2
(``tp_oracle.mlp_block``) and an upstream gradient dy = dL/dy, the gradients
dL/dx, dL/dW1, dL/db1, dL/dW2, dL/db2 by the chain rule, each shard's share
computed where the split puts it.

Source: xingyuzhitong.com "Tensor vs Pipeline Parallelism", section "Tensor
parallelism: split inside each layer": the Megatron-LM split (first
feed-forward linear by columns, second by rows) needs two all-reduces per
layer in the forward pass and two more in the backward pass.  The pages do not
say what the backward ones carry.  Reading, from the structure of that split:
in the backward pass dy reaches every shard whole (the backward of a sum over
shards is a copy to each shard), each weight gradient lands on the shard that
owns the weight, and the one exchange of the MLP is the sum over shards of the
first layer's input gradient dx, since every column shard used all of x.  That
sum is taken in ascending shard order, each partial started from zero, like
the forward sum.

Steps, per shard s owning first-layer outputs F_s (rows of W1, columns of W2):
  z_s  = x W1_s^T + b1_s,  h_s = act(z_s)          (recomputed forward)
  dh_s = dy W2[:, F_s]                              (no exchange)
  dW2[:, F_s] = dy^T h_s
  dz_s = dh_s * act'(z_s)
  dW1_s = dz_s^T x,  db1_s = sum over tokens of dz_s
  dx_s = dz_s W1_s                                  (a full-size [T, H] partial)
then dx = ((dx_0 + dx_1) + ...) + dx_{t-1} and db2 = sum over tokens of dy.

act' for the tanh GeLU g(z) = 0.5 z (1 + tanh u), u = c (z + a z^3), is the
product and chain rules applied to that form:
  g'(z) = 0.5 (1 + tanh u) + 0.5 z (1 - tanh^2 u) c (1 + 3 a z^2).

Pinned by tests/test_oracle_backward.py against central finite differences of
the (separately pinned) forward oracle, torch autograd of torch's own tanh GeLU
in float64, the closed form of the purely linear block, the identity
g'(z) + g'(-z) = 1, and independence of the result from t; planted mistakes
(a dropped GeLU-derivative term, a missing backward sum, a transposed weight
gradient) must fail them.
"""
from __future__ import annotations

from typing import Dict, Optional

import numpy as np

from .tp_oracle import GELU_CUBIC, SQRT_2_OVER_PI, ArrayLike, apply_act, shard_ranges, shard_sum, to_f64


def gelu_tanh_grad(z: np.ndarray) -> np.ndarray:
    """d/dz of the tanh-form GeLU, elementwise, in float64 (formula in the module docstring)."""
    z = np.asarray(z, dtype=np.float64)
    th = np.tanh(SQRT_2_OVER_PI * (z + GELU_CUBIC * z * z * z))
    return 0.5 * (1.0 + th) + 0.5 * z * (1.0 - th * th) * SQRT_2_OVER_PI * (
        1.0 + 3.0 * GELU_CUBIC * z * z)


def act_grad(z: np.ndarray, act: str) -> np.ndarray:
    if act == "gelu_tanh":
        return gelu_tanh_grad(z)
    if act == "none":
        return np.ones_like(np.asarray(z, dtype=np.float64))
    raise ValueError(f"unknown activation {act!r}")


def mlp_block_backward(x: ArrayLike, w1: ArrayLike, b1: Optional[ArrayLike], w2: ArrayLike,
                       dy: ArrayLike, t: int, act: str = "gelu_tanh") -> Dict[str, object]:
    """Gradients of the tensor-parallel MLP block for the upstream gradient dy [T, H].

    Weights in their storage layout: w1 [F, H], w2 [H, F].  Returns a dict with
    ``dx`` [T, H], ``dw1`` [F, H], ``db1`` [F], ``dw2`` [H, F], ``db2`` [H]
    (db1 and db2 are the gradients a bias would get, also when none is
    passed) and ``dx_partials``, the t per-shard [T, H] terms whose sum is dx:
    the tensors the backward all-reduce carries.
    """
    xf, w1f, w2f, dyf = to_f64(x), to_f64(w1), to_f64(w2), to_f64(dy)
    T, H = xf.shape
    F = w1f.shape[0]
    if w1f.shape != (F, H) or w2f.shape != (H, F) or dyf.shape != (T, H):
        raise ValueError(f"shape mismatch x{xf.shape} w1{w1f.shape} w2{w2f.shape} dy{dyf.shape}")
    b1f = None if b1 is None else to_f64(b1)
    dw1 = np.empty((F, H))
    db1 = np.empty(F)
    dw2 = np.empty((H, F))
    partials = []
    for (f0, f1) in shard_ranges(F, t):
        z = xf @ w1f[f0:f1].T
        if b1f is not None:
            z = z + b1f[None, f0:f1]
        h = apply_act(z, act)
        dh = dyf @ w2f[:, f0:f1]
        dw2[:, f0:f1] = dyf.T @ h
        dz = dh * act_grad(z, act)
        dw1[f0:f1] = dz.T @ xf
        db1[f0:f1] = dz.sum(axis=0)
        partials.append(dz @ w1f[f0:f1])
    dx = shard_sum(partials, None)
    return {"dx": dx, "dw1": dw1, "db1": db1, "dw2": dw2, "db2": dyf.sum(axis=0),
            "dx_partials": partials}
