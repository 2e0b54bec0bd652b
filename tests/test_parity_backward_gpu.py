"""GPU parity of the MLP block's backward pass against the fp64 backward oracle.

tp_mlp_backward (through the C ABI) returns dx, dw1, db1, dw2 and db2 for an
upstream gradient dy; oracle.mlp_block_backward computes the same gradients by
the chain rule in float64 (pinned in test_oracle_backward.py).  Acceptance is
the forward's: relative L2 error <= 1e-2 and max |error| <= 2e-2 * max |ref|
per output.  The GPU keeps z, dz and h in bf16 between its kernels (relative
rounding error 2^-9 per element), far inside that bound.  Shapes: the tiny
block with biases, ragged sizes (a token count that is not a multiple of 64
feeds the weight-gradient contractions over tokens, and output tiles that
overhang the matrices), and the 70B-shaped layer at 64 tokens, t = 8.
"""
import numpy as np
import pytest
import torch

import oracle
import tensor_transformer_linear_column_b200 as tp
import workloads

pytestmark = pytest.mark.gpu

REL_L2 = 1e-2
MAX_ABS_FRAC = 2e-2


def _dev():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch.device("cuda", torch.cuda.current_device())


def _parity(y_gpu, ref, what):
    y = y_gpu.detach().to("cpu", torch.float64).numpy()
    r = np.asarray(ref, dtype=np.float64)
    assert y.shape == r.shape, (what, y.shape, r.shape)
    assert np.isfinite(y).all(), what
    err = y - r
    rel = np.linalg.norm(err) / max(np.linalg.norm(r), 1e-300)
    mx = np.abs(err).max()
    bound = MAX_ABS_FRAC * np.abs(r).max()
    assert rel <= REL_L2 and mx <= bound, f"{what}: rel_l2={rel:.3e} max_abs={mx:.3e} bound={bound:.3e}"


def _check_all(x, w1, b1, w2, dy, t, act, what):
    dev = _dev()
    ref = oracle.mlp_block_backward(x, w1, b1, w2, dy, t, act)
    g = tp.tp_mlp_backward(x.to(dev), w1.to(dev), None if b1 is None else b1.to(dev),
                           w2.to(dev), dy.to(dev), t, act)
    torch.cuda.synchronize()
    assert tp.tp_device_error_check() == tp.TP_OK
    for k in ("dx", "dw1", "db1", "dw2", "db2"):
        _parity(g[k], ref[k], f"{what} {k}")
    return g


def test_tiny_block_backward():
    cfg = workloads.CONFIGS["tiny"]
    d = workloads.mlp_inputs(cfg, 8)
    dy = workloads.random_bf16_small((8, cfg.hidden), 1.0, 21)
    _check_all(d["x"], d["w1"], d["b1"], d["w2"], dy, 2, "gelu_tanh", "tiny")


@pytest.mark.parametrize("T,H,F,t", [(100, 384, 1536, 4), (1, 256, 512, 2), (300, 192, 768, 3),
                                     (64, 640, 1280, 5)])
@pytest.mark.parametrize("act", ["gelu_tanh", "none"])
def test_ragged_backward(T, H, F, t, act):
    x = workloads.random_bf16_small((T, H), 1.0, 31 + T)
    w1 = workloads.random_bf16_small((F, H), 0.04, 32)
    b1 = workloads.random_bf16_small((F,), 0.05, 33)
    w2 = workloads.random_bf16_small((H, F), 0.04, 34)
    dy = workloads.random_bf16_small((T, H), 1.0, 35 + T)
    _check_all(x, w1, b1, w2, dy, t, act, f"T={T} H={H} F={F} t={t} {act}")


def test_backward_bit_identical_on_repeat():
    dev = _dev()
    x = workloads.random_bf16_small((130, 512), 1.0, 41).to(dev)
    w1 = workloads.random_bf16_small((2048, 512), 0.04, 42).to(dev)
    w2 = workloads.random_bf16_small((512, 2048), 0.04, 43).to(dev)
    dy = workloads.random_bf16_small((130, 512), 1.0, 44).to(dev)
    a = tp.tp_mlp_backward(x, w1, None, w2, dy, 4, "gelu_tanh")
    b = tp.tp_mlp_backward(x, w1, None, w2, dy, 4, "gelu_tanh")
    torch.cuda.synchronize()
    for k in a:
        assert torch.equal(a[k], b[k]), k


def test_mlp70b_backward_64_tokens():
    cfg = workloads.CONFIGS["mlp70b"]
    T = 64
    d = workloads.mlp_inputs(cfg, T)
    dy = workloads.normal_bf16((T, cfg.hidden), 1.0, 0, 200 + T)
    _check_all(d["x"], d["w1"], None, d["w2"], dy, 8, "gelu_tanh", "mlp70b T=64")
