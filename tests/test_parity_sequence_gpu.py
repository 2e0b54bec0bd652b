"""GPU parity of the sequence-parallel region against the fp64 oracle.

The row-parallel linear (tp_rowpar_gemm_reduce, whose on-chip shard sum is
the reduce-scatter and all-gather together) followed by tp_sp_add_rmsnorm
(residual add and RMSNorm of each token shard's rows) must match
oracle.sp_residual_norm (pinned in test_oracle_sequence.py) on both outputs,
r = residual + y and n = RMSNorm(r) * gamma, within the parity tolerance:
relative L2 <= 1e-2 and max |error| <= 2e-2 * max |ref|.
"""
import numpy as np
import pytest
import torch

import oracle
import tensor_transformer_linear_column_b200 as tp
import workloads

pytestmark = pytest.mark.gpu


def _dev():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch.device("cuda", torch.cuda.current_device())


def _parity(y_gpu, ref, what):
    y = y_gpu.detach().to("cpu", torch.float64).numpy()
    r = np.asarray(ref, dtype=np.float64)
    assert y.shape == r.shape and np.isfinite(y).all(), what
    err = y - r
    rel = np.linalg.norm(err) / max(np.linalg.norm(r), 1e-300)
    mx = np.abs(err).max()
    assert rel <= 1e-2 and mx <= 2e-2 * np.abs(r).max(), f"{what}: rel={rel:.3e} max={mx:.3e}"


@pytest.mark.parametrize("T,K,H,t", [(8, 1024, 256, 2), (64, 6656, 16384, 8),
                                     (48, 768, 192, 3), (200, 2048, 1024, 4)])
def test_rowpar_then_sp_region(T, K, H, t):
    dev = _dev()
    h = workloads.random_bf16_small((T, K), 1.0, 50 + T)
    w = workloads.random_bf16_small((H, K), 0.02, 51)
    b = workloads.random_bf16_small((H,), 0.05, 52)
    res = workloads.random_bf16_small((T, H), 1.0, 53 + T)
    gamma = (1.0 + workloads.random_bf16_small((H,), 0.1, 54).float()).to(torch.bfloat16)
    parts = oracle.rowpar_partials(h, w, t)
    r_ref, n_ref = oracle.sp_residual_norm(parts, b, res, gamma, t)
    y = tp.tp_rowpar_gemm_reduce(h.to(dev), w.to(dev), b.to(dev), t)
    r, n = tp.tp_sp_add_rmsnorm(y, res.to(dev), gamma.to(dev), t)
    torch.cuda.synchronize()
    assert tp.tp_device_error_check() == tp.TP_OK
    _parity(r, r_ref, f"r T={T} H={H} t={t}")
    _parity(n, n_ref, f"n T={T} H={H} t={t}")


def test_sp_region_bit_identical_on_repeat():
    dev = _dev()
    y = workloads.random_bf16_small((32, 4096), 1.0, 60).to(dev)
    res = workloads.random_bf16_small((32, 4096), 1.0, 61).to(dev)
    g = workloads.random_bf16_small((4096,), 1.0, 62).to(dev)
    a = tp.tp_sp_add_rmsnorm(y, res, g, 8)
    b = tp.tp_sp_add_rmsnorm(y, res, g, 8)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_sp405b_bench_workload_sampled_rows():
    # the bench workload (T = 8192 token rows of H = 16384, t = 8) in the
    # bench's launch configuration; the oracle checks 64 seeded rows
    dev = _dev()
    cfg = workloads.CONFIGS["sp405b"]
    T = cfg.tokens[0]
    d = workloads.sp_norm_inputs(cfg, T)
    rows = workloads.sample_rows(T, 64)
    r_ref, n_ref = oracle.sp_residual_norm([oracle.to_f64(d["y"][rows])], None,
                                           d["residual"][rows], d["gamma"], 1)
    prev = tp.tp_get_launch_options()
    tp.tp_set_launch_options(tp.TP_OPT_PDL | tp.TP_OPT_STATIC_WEIGHTS)
    try:
        r, n = tp.tp_sp_add_rmsnorm(d["y"].to(dev), d["residual"].to(dev), d["gamma"].to(dev),
                                    cfg.tp_degrees[0])
        torch.cuda.synchronize()
    finally:
        tp.tp_set_launch_options(prev)
    idx = torch.tensor(rows, device=dev)
    _parity(r[idx], r_ref, "sp405b r")
    _parity(n[idx], n_ref, "sp405b n")
    assert tp.tp_device_error_check() == tp.TP_OK


@pytest.mark.parametrize("T,H,t", [(1000, 8192, 8), (450, 12288, 2), (300, 4096, 3), (149, 16384, 1)])
def test_sp_region_wide_rows(T, H, t):
    # wide rows kept in registers between the sum of squares and the
    # normalisation (up to 64 values per thread), T rows in t token shards,
    # T not a multiple of the SM count
    dev = _dev()
    y = workloads.random_bf16_small((T, H), 1.0, 70 + T)
    res = workloads.random_bf16_small((T, H), 1.0, 71 + T)
    gamma = (1.0 + workloads.random_bf16_small((H,), 0.1, 72).float()).to(torch.bfloat16)
    r_ref, n_ref = oracle.sp_residual_norm([oracle.to_f64(y)], None, res, gamma, t)
    r, n = tp.tp_sp_add_rmsnorm(y.to(dev), res.to(dev), gamma.to(dev), t)
    torch.cuda.synchronize()
    assert tp.tp_device_error_check() == tp.TP_OK
    _parity(r, r_ref, f"r T={T} H={H}")
    _parity(n, n_ref, f"n T={T} H={H}")
