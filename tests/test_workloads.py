"""The seeded input generator: deterministic, thread-count independent."""
import torch

import workloads


def test_chunked_draw_independent_of_threads(monkeypatch):
    monkeypatch.setattr(workloads, "CHUNK", 1000)
    a = workloads.normal_bf16((7, 1001), 0.02, seed=3, index=1, threads=1)
    b = workloads.normal_bf16((7, 1001), 0.02, seed=3, index=1, threads=5)
    assert a.dtype == torch.bfloat16 and a.shape == (7, 1001)
    assert torch.equal(a, b)
    c = workloads.normal_bf16((7, 1001), 0.02, seed=4, index=1, threads=1)
    assert not torch.equal(a, c)


def test_std_and_rounding():
    a = workloads.normal_bf16((1 << 16,), 0.02, seed=0, index=1)
    s = a.float().std().item()
    assert 0.019 < s < 0.021
    # values are exactly representable in bf16
    assert torch.equal(a.float().to(torch.bfloat16), a)


def test_tiny_x_is_fp32_rounded_once():
    cfg = workloads.CONFIGS["tiny"]
    d = workloads.mlp_inputs(cfg, 8)
    assert d["x_fp32"].dtype == torch.float32
    assert torch.equal(d["x_fp32"].to(torch.bfloat16), d["x"])
    assert d["b1"] is not None and d["b2"] is not None
    assert d["w1"].shape == (1024, 256) and d["w2"].shape == (256, 1024)


def test_sample_rows():
    r = workloads.sample_rows(8192, 64, seed=0)
    assert r == sorted(set(r)) and len(r) == 64 and all(0 <= i < 8192 for i in r)
    assert r == workloads.sample_rows(8192, 64, seed=0)
