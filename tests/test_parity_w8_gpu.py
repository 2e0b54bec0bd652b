"""GPU parity of the 8-bit-weight calls (FP8 E4M3 codes with one fp32 scale per
output row) against the fp64 oracle, through the C ABI.

The oracle computes the same layer with the weight scale[n] * e4m3(q[n, k])
decoded exactly (oracle.E4M3Weight); the acceptance bound is the bf16 one
(relative L2 <= 1e-2, max |error| <= 2e-2 max |y_ref|): the GPU's products are
the bf16 kernel's, since every E4M3 value is a bf16 value.
"""
import numpy as np
import pytest
import torch

import oracle
import tensor_transformer_linear_column_b200 as tp
import workloads
from test_parity_gpu import BENCH_OPTIONS, _dev, _no_device_error, assert_parity, launch_options

pytestmark = pytest.mark.gpu


def _w8(shape, std, seed):
    w = workloads.random_bf16_small(shape, std, seed)
    return workloads.quantize_e4m3_rows(w)


W8_COL = [(1, 64, 64), (3, 576, 320), (5, 4096, 320), (17, 128, 1088), (63, 192, 256),
          (64, 1024, 512), (128, 256, 384), (5, 256, 20480), (3, 8192, 320), (9, 16384, 192),
          # two k-blocks per box with a K-split cluster (2 CTAs, and 8 above)
          (2, 4096, 16384)]


@pytest.mark.parametrize("T,K,N", W8_COL)
@pytest.mark.parametrize("act", ["none", "gelu_tanh"])
def test_w8_colpar(T, K, N, act):
    dev = _dev()
    x = workloads.random_bf16_small((T, K), 1.0, 7000 + T)
    q, sc = _w8((N, K), 0.05, 7100 + N)
    b = workloads.random_bf16_small((N,), 0.1, 7200 + N)
    ref = oracle.colpar_linear(x, oracle.E4M3Weight(q, sc), b, 1, act)
    with launch_options(BENCH_OPTIONS):
        y = tp.tp_colpar_gemm_gelu_w8(x.to(dev), q.to(dev), sc.to(dev), b.to(dev), 1, act)
    torch.cuda.synchronize()
    _no_device_error()
    assert_parity(y, ref, f"w8 colpar T={T} K={K} N={N} {act}")


W8_ROW = [(1, 512, 64, 1), (5, 512, 320, 2), (33, 1024, 256, 4), (64, 512, 128, 8),
          (2, 8192, 192, 2), (8, 2048, 1088, 8), (40, 1024, 256, 16), (6, 4096, 64, 16),
          # two k-blocks per box, clusters of 4 (2 CTAs per shard)
          (7, 8192, 8192, 2)]


@pytest.mark.parametrize("T,K,N,t", W8_ROW)
def test_w8_rowpar(T, K, N, t):
    dev = _dev()
    h = workloads.random_bf16_small((T, K), 0.5, 7300 + T)
    q, sc = _w8((N, K), 0.05, 7400 + N)
    b = workloads.random_bf16_small((N,), 0.1, 7500 + N)
    ref = oracle.rowpar_linear(h, oracle.E4M3Weight(q, sc), b, t)
    with launch_options(BENCH_OPTIONS):
        y = tp.tp_rowpar_gemm_reduce_w8(h.to(dev), q.to(dev), sc.to(dev), b.to(dev), t)
    torch.cuda.synchronize()
    _no_device_error()
    assert_parity(y, ref, f"w8 rowpar T={T} K={K} N={N} t={t}")


def test_w8_rowpar_more_than_two_shards_per_cta_is_unsupported():
    # t = 3 over K = 576: no power-of-two cluster splits 3 shards, so one CTA
    # would own all three; the 8-bit kernel drains at most two per CTA
    dev = _dev()
    h = workloads.random_bf16_small((7, 576), 0.5, 7307).to(dev)
    q, sc = _w8((192, 576), 0.05, 7492)
    with pytest.raises(tp.TPError) as e:
        tp.tp_rowpar_gemm_reduce_w8(h, q.to(dev), sc.to(dev), None, 3)
    assert e.value.status == tp.TP_ERR_UNSUPPORTED


def test_w8_mlp_unsupported_split_launches_nothing():
    # t = 3 over F = 576: the second layer would need three shards per CTA;
    # the call must refuse before its first layer writes the workspace
    dev = _dev()
    T, H, F = 5, 256, 576
    x = workloads.random_bf16_small((T, H), 1.0, 7700).to(dev)
    q1, s1 = _w8((F, H), 0.05, 7701)
    q2, s2 = _w8((H, F), 0.05, 7702)
    ws = torch.full((tp.tp_mlp_workspace_bytes(T, F),), 0x5A, dtype=torch.uint8, device=dev)
    out = torch.full((T, H), 7.0, dtype=torch.bfloat16, device=dev)
    with pytest.raises(tp.TPError) as e:
        tp.tp_mlp_forward_w8(x, q1.to(dev), s1.to(dev), None, q2.to(dev), s2.to(dev), None, 3,
                             "gelu_tanh", out=out, workspace=ws)
    assert e.value.status == tp.TP_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert bool((ws == 0x5A).all())
    assert bool((out == 7.0).all())


@pytest.fixture(scope="module")
def mlp70b_w8():
    cfg = workloads.CONFIGS["mlp70b_w8"]
    d = workloads.mlp_inputs(cfg, 1)
    q1, s1 = workloads.quantize_e4m3_rows(d["w1"])
    q2, s2 = workloads.quantize_e4m3_rows(d["w2"])
    dev = _dev()
    return cfg, (q1, s1, q2, s2), tuple(a.to(dev) for a in (q1, s1, q2, s2))


@pytest.mark.parametrize("t", [4, 8])
@pytest.mark.parametrize("T", [1, 16, 64])
def test_w8_mlp70b_decode(mlp70b_w8, T, t):
    dev = _dev()
    cfg, (q1, s1, q2, s2), (q1d, s1d, q2d, s2d) = mlp70b_w8
    x = workloads.mlp_x(cfg, T)
    ref = oracle.mlp_block(x, oracle.E4M3Weight(q1, s1), None, oracle.E4M3Weight(q2, s2), None,
                           t, "gelu_tanh")
    with launch_options(BENCH_OPTIONS):
        y = tp.tp_mlp_forward_w8(x.to(dev), q1d, s1d, None, q2d, s2d, None, t, "gelu_tanh")
    torch.cuda.synchronize()
    _no_device_error()
    assert_parity(y, ref, f"w8 mlp70b T={T} t={t}")


def test_w8_repeat_bit_identical(mlp70b_w8):
    dev = _dev()
    cfg, _, (q1d, s1d, q2d, s2d) = mlp70b_w8
    x = workloads.mlp_x(cfg, 16).to(dev)
    ys = [tp.tp_mlp_forward_w8(x, q1d, s1d, None, q2d, s2d, None, 8, "gelu_tanh")
          for _ in range(3)]
    torch.cuda.synchronize()
    for y in ys[1:]:
        assert torch.equal(y, ys[0])


def test_w8_power_of_two_scales_match_the_bf16_weight():
    # with scales that are powers of two, scale * e4m3(q) is a bf16 value and
    # the 8-bit call must agree with the bf16 call on that weight
    dev = _dev()
    T, K, N = 8, 2048, 512
    g = torch.Generator().manual_seed(7600)
    q = (torch.randint(0, 0x7F, (N, K), generator=g, dtype=torch.int32)
         | torch.randint(0, 2, (N, K), generator=g, dtype=torch.int32) * 0x80).to(torch.uint8)
    sc = 2.0 ** -torch.randint(4, 9, (N,), generator=g).to(torch.float32)
    w = (q.view(torch.float8_e4m3fn).to(torch.float32) * sc[:, None]).to(torch.bfloat16)
    x = workloads.random_bf16_small((T, K), 1.0, 7601)
    y8 = tp.tp_colpar_gemm_gelu_w8(x.to(dev), q.to(dev), sc.to(dev), None, 2, "gelu_tanh")
    y16 = tp.tp_colpar_gemm_gelu(x.to(dev), w.to(dev), None, 2, "gelu_tanh")
    torch.cuda.synchronize()
    assert_parity(y8, y16.double().cpu().numpy(), "w8 vs bf16 on the same weight")
    ref = oracle.colpar_linear(x, w, None, 2, "gelu_tanh")
    assert_parity(y8, ref, "w8 vs oracle")


def test_w8_decode_only():
    dev = _dev()
    x = torch.zeros((129, 256), dtype=torch.bfloat16, device=dev)
    q = torch.zeros((256, 256), dtype=torch.uint8, device=dev)
    sc = torch.ones(256, dtype=torch.float32, device=dev)
    with pytest.raises(tp.TPError) as e:
        tp.tp_colpar_gemm_gelu_w8(x, q, sc, None, 1)
    assert e.value.status == tp.TP_ERR_UNSUPPORTED
