"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Acceptance (bf16 in, fp32 accumulate, bf16 out): relative L2 error <= 1e-2 and
max |error| <= 2e-2 * max |y_ref|, on the full output, or on 64 seeded rows
for the two prefill workloads (rows are independent, so the oracle computes
only those rows).  Both kernel paths are exercised: the weight-streaming
(decode) kernels and the persistent tiled (prefill) kernels, forced through
tp_set_decode_max_tokens.
"""
import contextlib

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


def assert_parity(y_gpu, y_ref, what=""):
    y = y_gpu.detach().to("cpu", torch.float64).numpy()
    r = np.asarray(y_ref, dtype=np.float64)
    assert y.shape == r.shape, (what, y.shape, r.shape)
    assert np.isfinite(y).all(), what
    err = y - r
    rel = np.linalg.norm(err) / max(np.linalg.norm(r), 1e-300)
    mx = np.abs(err).max()
    bound = MAX_ABS_FRAC * np.abs(r).max()
    assert rel <= REL_L2 and mx <= bound, f"{what}: rel_l2={rel:.3e} max_abs={mx:.3e} bound={bound:.3e}"
    return rel, mx


@contextlib.contextmanager
def kernel_path(name):
    """Force one kernel: "stream" (tensor-core weight streaming, T <= 128) or
    "tiled" (persistent tensor-core GEMM)."""
    prev = tp.tp_get_decode_max_tokens()
    tp.tp_set_decode_max_tokens(0 if name == "tiled" else 128)
    try:
        yield
    finally:
        tp.tp_set_decode_max_tokens(prev)


def paths_for(T, K, shard_k=None):
    """Kernels that can serve a call of T tokens."""
    return ["stream", "tiled"] if T <= 128 else ["tiled"]


@contextlib.contextmanager
def launch_options(flags):
    prev = tp.tp_get_launch_options()
    tp.tp_set_launch_options(flags)
    try:
        yield
    finally:
        tp.tp_set_launch_options(prev)


# the launch configuration bench.py times: PDL with static-weight prefetch
BENCH_OPTIONS = tp.TP_OPT_PDL | tp.TP_OPT_STATIC_WEIGHTS


def _no_device_error():
    assert tp.tp_device_error_check() == tp.TP_OK


def _cuda(t, dev):
    return None if t is None else t.to(dev).contiguous()


# ---------------------------------------------------------------- tiny block

@pytest.mark.parametrize("path", ["stream", "tiled"])
def test_tiny_mlp_block(path):
    dev = _dev()
    cfg = workloads.CONFIGS["tiny"]
    d = workloads.mlp_inputs(cfg, 8)
    ref = oracle.mlp_block(d["x"], d["w1"], d["b1"], d["w2"], d["b2"], 2, "gelu_tanh")
    g = {k: _cuda(v, dev) for k, v in d.items() if k != "x_fp32"}
    with kernel_path(path):
        y = tp.tp_mlp_forward(g["x"], g["w1"], g["b1"], g["w2"], g["b2"], 2, "gelu_tanh")
        h = tp.tp_colpar_gemm_gelu(g["x"], g["w1"], g["b1"], 2, "gelu_tanh")
        y2 = tp.tp_rowpar_gemm_reduce(h, g["w2"], g["b2"], 2)
    torch.cuda.synchronize()
    _no_device_error()
    assert_parity(y, ref, f"tiny mlp {path}")
    assert torch.equal(y, y2)
    assert_parity(h, oracle.colpar_linear(d["x"], d["w1"], d["b1"], 2, "gelu_tanh"), "tiny colpar")


# ---------------------------------------------------------------- square projection

@pytest.fixture(scope="module")
def sq_weights():
    cfg = workloads.CONFIGS["sq4096"]
    d = workloads.proj_inputs(cfg, 1)
    return cfg, d["w"]


@pytest.mark.parametrize("path", ["stream", "tiled"])
@pytest.mark.parametrize("T", [1, 8, 64])
def test_sq4096_colpar(sq_weights, T, path):
    dev = _dev()
    cfg, w = sq_weights
    x = workloads.proj_inputs(cfg, T)["x"]
    ref = oracle.colpar_linear(x, w, None, 2, "none")
    with kernel_path(path), launch_options(BENCH_OPTIONS):
        y = tp.tp_colpar_gemm_gelu(x.to(dev), w.to(dev), None, 2, "none")
    torch.cuda.synchronize()
    _no_device_error()
    assert_parity(y, ref, f"sq4096 T={T} {path}")


# ---------------------------------------------------------------- ragged shapes, both paths

RAGGED_COL = [(1, 64, 64), (2, 768, 64), (3, 576, 320), (3, 256, 1088), (5, 4096, 320),
              (8, 512, 64), (17, 128, 1088), (63, 192, 256), (65, 64, 320),
              (128, 256, 384), (130, 320, 576), (200, 256, 1024), (257, 128, 320),
              (300, 64, 1088), (5, 256, 20480), (40, 128, 20480),
              # long per-CTA streams: two k-blocks per TMA box, an odd number of stages
              (3, 8192, 320), (9, 16384, 192)]


@pytest.mark.parametrize("T,K,N", RAGGED_COL)
@pytest.mark.parametrize("act", ["none", "gelu_tanh"])
def test_colpar_ragged(T, K, N, act):
    dev = _dev()
    x = workloads.random_bf16_small((T, K), 1.0, 1000 + T)
    w = workloads.random_bf16_small((N, K), 0.05, 2000 + N)
    b = workloads.random_bf16_small((N,), 0.1, 3000 + N)
    ref = oracle.colpar_linear(x, w, b, 1, act)
    for path in paths_for(T, K):
        with kernel_path(path):
            y = tp.tp_colpar_gemm_gelu(x.to(dev), w.to(dev), b.to(dev), 1, act)
        torch.cuda.synchronize()
        assert_parity(y, ref, f"colpar T={T} K={K} N={N} {act} {path}")
    _no_device_error()


RAGGED_ROW = [(1, 512, 64, 1), (5, 512, 320, 2), (33, 1024, 256, 4), (64, 512, 128, 8),
              (128, 1024, 192, 4), (129, 2048, 320, 8), (300, 512, 64, 4), (7, 576, 192, 3),
              (40, 1024, 256, 16), (2, 4096, 128, 2), (3, 768, 320, 3), (6, 4096, 64, 16),
              (8, 2048, 1088, 8), (1, 256, 64, 1), (2, 8192, 192, 2)]


@pytest.mark.parametrize("T,K,N,t", RAGGED_ROW)
def test_rowpar_ragged(T, K, N, t):
    dev = _dev()
    h = workloads.random_bf16_small((T, K), 0.5, 4000 + T)
    w = workloads.random_bf16_small((N, K), 0.05, 5000 + N)
    b = workloads.random_bf16_small((N,), 0.1, 6000 + N)
    ref = oracle.rowpar_linear(h, w, b, t)
    for path in paths_for(T, K, K // t):
        with kernel_path(path):
            y = tp.tp_rowpar_gemm_reduce(h.to(dev), w.to(dev), b.to(dev), t)
        torch.cuda.synchronize()
        assert_parity(y, ref, f"rowpar T={T} K={K} N={N} t={t} {path}")
    _no_device_error()


@pytest.mark.parametrize("path", ["stream", "tiled"])
def test_rowpar_equals_sum_of_single_shard_calls(path):
    # the all-reduce property: the fused t-shard call matches the shards'
    # separately computed partials summed (up to rounding of those partials)
    dev = _dev()
    T, K, N, t = 24, 2048, 256, 4
    h = workloads.random_bf16_small((T, K), 0.5, 71)
    w = workloads.random_bf16_small((N, K), 0.05, 72)
    ks = K // t
    with kernel_path(path):
        y = tp.tp_rowpar_gemm_reduce(h.to(dev), w.to(dev), None, t)
        parts = [tp.tp_rowpar_gemm_reduce(h[:, s * ks:(s + 1) * ks].contiguous().to(dev),
                                          w[:, s * ks:(s + 1) * ks].contiguous().to(dev), None, 1)
                 for s in range(t)]
    torch.cuda.synchronize()
    summed = sum(p.double() for p in parts)
    assert_parity(y, summed.cpu().numpy(), "fused sum vs separate partials")
    assert_parity(y, oracle.rowpar_linear(h, w, None, t), "fused sum vs oracle")


def test_colpar_result_independent_of_tp_degree():
    dev = _dev()
    x = workloads.random_bf16_small((7, 512), 1.0, 81).to(dev)
    w = workloads.random_bf16_small((1024, 512), 0.05, 82).to(dev)
    for path in ("stream", "tiled"):
        with kernel_path(path):
            ys = [tp.tp_colpar_gemm_gelu(x, w, None, t, "gelu_tanh") for t in (1, 2, 4, 8, 16)]
        torch.cuda.synchronize()
        for y in ys[1:]:
            assert torch.equal(y, ys[0])


# ---------------------------------------------------------------- 70B-shaped MLP decode

@pytest.fixture(scope="module")
def mlp70b():
    cfg = workloads.CONFIGS["mlp70b"]
    d = workloads.mlp_inputs(cfg, 1)
    dev = _dev()
    return cfg, d["w1"], d["w2"], d["w1"].to(dev), d["w2"].to(dev)


@pytest.mark.parametrize("t", [4, 8])
@pytest.mark.parametrize("T", [1, 16, 64])
def test_mlp70b_decode(mlp70b, T, t):
    dev = _dev()
    cfg, w1, w2, w1d, w2d = mlp70b
    x = workloads.mlp_x(cfg, T)
    ref = oracle.mlp_block(x, w1, None, w2, None, t, "gelu_tanh")
    with launch_options(BENCH_OPTIONS):
        y = tp.tp_mlp_forward(x.to(dev), w1d, None, w2d, None, t, "gelu_tanh")
    torch.cuda.synchronize()
    _no_device_error()
    assert_parity(y, ref, f"mlp70b T={T} t={t}")


def test_mlp70b_tp4_vs_tp8_differ_only_in_rounding(mlp70b):
    dev = _dev()
    cfg, w1, w2, w1d, w2d = mlp70b
    x = workloads.mlp_x(cfg, 16).to(dev)
    y4 = tp.tp_mlp_forward(x, w1d, None, w2d, None, 4, "gelu_tanh")
    y8 = tp.tp_mlp_forward(x, w1d, None, w2d, None, 8, "gelu_tanh")
    torch.cuda.synchronize()
    assert_parity(y4, y8.double().cpu().numpy(), "t=4 vs t=8")


# ---------------------------------------------------------------- prefill, sampled rows

def test_attn70b_prefill_sampled_rows():
    dev = _dev()
    cfg = workloads.CONFIGS["attn70b"]
    T = cfg.tokens[0]
    d = workloads.attn_inputs(cfg, T)
    rows = workloads.sample_rows(T, cfg.sample_rows)
    q_ref = oracle.attn_qkv(d["x"][rows], d["w_qkv"], None, cfg.n_q_heads, cfg.n_kv_heads,
                            cfg.head_dim, 8)
    o_ref = oracle.attn_out(d["ctx"][rows], d["w_o"], None, cfg.n_q_heads, cfg.head_dim, 8)
    with launch_options(BENCH_OPTIONS):
        qkv, y = tp.tp_attn_proj_forward(d["x"].to(dev), d["w_qkv"].to(dev), None,
                                         d["ctx"].to(dev), d["w_o"].to(dev), None,
                                         cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim, 8)
    torch.cuda.synchronize()
    _no_device_error()
    idx = torch.tensor(rows, device=dev)
    assert_parity(qkv[idx], q_ref, "attn70b qkv")
    assert_parity(y[idx], o_ref, "attn70b out")
    assert torch.isfinite(y.float()).all() and torch.isfinite(qkv.float()).all()


@pytest.fixture(scope="module")
def attn70b_weights():
    cfg = workloads.CONFIGS["attn70b"]
    d = workloads.attn_inputs(cfg, 1, with_bias=True)
    return cfg, d


@pytest.mark.parametrize("T", [1, 16, 64])
@pytest.mark.parametrize("bias", [False, True])
def test_attn70b_decode_projections(attn70b_weights, T, bias):
    # decode-shaped calls of the attention projections on the 70B head layout
    # (64 query / 8 key-value heads of 128, t = 8): both go through the
    # weight-streaming kernel -- QKV N = 10240 column-parallel, O-projection
    # over nctx = 8192 with 8 head-group shards of 1024
    dev = _dev()
    cfg, d = attn70b_weights
    nq, nkv, hd = cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim
    x = workloads.random_bf16_small((T, cfg.hidden), 1.0, 300 + T)
    ctx = workloads.random_bf16_small((T, nq * hd), 1.0, 400 + T)
    b_qkv = d["b_qkv"] if bias else None
    b_o = d["b_o"] if bias else None
    q_ref = oracle.attn_qkv(x, d["w_qkv"], b_qkv, nq, nkv, hd, 8)
    o_ref = oracle.attn_out(ctx, d["w_o"], b_o, nq, hd, 8)
    with launch_options(BENCH_OPTIONS):
        qkv, y = tp.tp_attn_proj_forward(x.to(dev), d["w_qkv"].to(dev), _cuda(b_qkv, dev),
                                         ctx.to(dev), d["w_o"].to(dev), _cuda(b_o, dev),
                                         nq, nkv, hd, 8)
    torch.cuda.synchronize()
    _no_device_error()
    assert_parity(qkv, q_ref, f"attn70b decode qkv T={T}")
    assert_parity(y, o_ref, f"attn70b decode out T={T}")


def test_mlp405b_prefill_sampled_rows():
    dev = _dev()
    cfg = workloads.CONFIGS["mlp405b"]
    T = cfg.tokens[0]
    d = workloads.mlp_inputs(cfg, T)
    rows = workloads.sample_rows(T, cfg.sample_rows)
    ref = oracle.mlp_block(d["x"][rows], d["w1"], None, d["w2"], None, 8, "gelu_tanh")
    with launch_options(BENCH_OPTIONS):
        y = tp.tp_mlp_forward(d["x"].to(dev), d["w1"].to(dev), None, d["w2"].to(dev), None, 8,
                              "gelu_tanh")
    torch.cuda.synchronize()
    _no_device_error()
    assert_parity(y[torch.tensor(rows, device=dev)], ref, "mlp405b rows")
    assert torch.isfinite(y.float()).all()


# ---------------------------------------------------------------- determinism

@pytest.mark.parametrize("path", ["stream", "tiled"])
def test_repeat_and_launch_order_bit_identical(path):
    dev = _dev()
    T, H, F, t = 40, 1024, 4096, 4
    x = workloads.random_bf16_small((T, H), 1.0, 91).to(dev)
    w1 = workloads.random_bf16_small((F, H), 0.03, 92).to(dev)
    w2 = workloads.random_bf16_small((H, F), 0.03, 93).to(dev)
    b2 = workloads.random_bf16_small((H,), 0.1, 94).to(dev)
    other_x = workloads.random_bf16_small((300, H), 1.0, 95).to(dev)
    with kernel_path(path):
        ref = tp.tp_mlp_forward(x, w1, None, w2, b2, t, "gelu_tanh")
        outs = []
        for i in range(5):
            outs.append(tp.tp_mlp_forward(x, w1, None, w2, b2, t, "gelu_tanh"))
        # interleave other work on a second stream, then run again
        s2 = torch.cuda.Stream()
        with torch.cuda.stream(s2):
            for i in range(3):
                tp.tp_colpar_gemm_gelu(other_x, w1, None, 4, "gelu_tanh")
        outs.append(tp.tp_mlp_forward(x, w1, None, w2, b2, t, "gelu_tanh"))
        with torch.cuda.stream(s2):
            outs.append(tp.tp_mlp_forward(x, w1, None, w2, b2, t, "gelu_tanh"))
    torch.cuda.synchronize()
    _no_device_error()
    for o in outs:
        assert torch.equal(o, ref)


# ---------------------------------------------------------------- bounds: canaries

@pytest.mark.parametrize("T", [1, 3, 17, 63, 129])
def test_outputs_write_nothing_outside_their_bounds(T):
    dev = _dev()
    K, N, t = 256, 320, 2
    x = workloads.random_bf16_small((T, K), 1.0, 11).to(dev)
    w = workloads.random_bf16_small((N, K), 0.05, 12).to(dev)
    pad = 4096
    for path in paths_for(T, K, K // t):
        buf = torch.empty((pad + T * N + pad,), dtype=torch.bfloat16, device=dev)
        buf.view(torch.int16).fill_(0x7FC1)  # a NaN bit pattern
        out = buf[pad:pad + T * N].view(T, N)
        with kernel_path(path):
            tp.tp_colpar_gemm_gelu(x, w, None, t, "gelu_tanh", out=out)
            h = tp.tp_rowpar_gemm_reduce(x, w[:, :K].contiguous(), None, t)
        torch.cuda.synchronize()
        head = buf[:pad].view(torch.int16)
        tail = buf[pad + T * N:].view(torch.int16)
        assert bool((head == 0x7FC1).all()) and bool((tail == 0x7FC1).all()), path
        assert torch.isfinite(out.float()).all()
        assert torch.isfinite(h.float()).all()
    _no_device_error()


# ---------------------------------------------------------------- launch options (PDL)


ALL_OPTIONS = [0, tp.TP_OPT_PDL, tp.TP_OPT_PDL | tp.TP_OPT_STATIC_WEIGHTS]


@pytest.mark.parametrize("T", [5, 64, 200])
def test_launch_options_do_not_change_results(T):
    dev = _dev()
    H, F, t = 512, 2048, 4
    x = workloads.random_bf16_small((T, H), 1.0, 301).to(dev)
    w1 = workloads.random_bf16_small((F, H), 0.04, 302).to(dev)
    w2 = workloads.random_bf16_small((H, F), 0.04, 303).to(dev)
    b1 = workloads.random_bf16_small((F,), 0.05, 304).to(dev)
    outs = []
    for flags in ALL_OPTIONS:
        with launch_options(flags):
            outs.append(tp.tp_mlp_forward(x, w1, b1, w2, None, t, "gelu_tanh"))
    torch.cuda.synchronize()
    _no_device_error()
    for o in outs[1:]:
        assert torch.equal(o, outs[0])
    ref = oracle.mlp_block(x.cpu(), w1.cpu(), b1.cpu(), w2.cpu(), None, t, "gelu_tanh")
    assert_parity(outs[-1], ref, f"options T={T}")


@pytest.mark.parametrize("path", ["stream", "tiled"])
def test_dependent_chain_under_programmatic_launch(path):
    # each call reads the previous call's output: the kernels must not read
    # activations before the producing kernel finished, whatever the options
    dev = _dev()
    T, K = {"stream": (16, 1024), "tiled": (192, 1024)}[path]
    w = workloads.random_bf16_small((K, K), 1.0 / 32, 401).to(dev)
    x0 = workloads.random_bf16_small((T, K), 1.0, 402).to(dev)
    steps = 12
    with kernel_path(path):
        with launch_options(0):
            ref = x0
            for _ in range(steps):
                ref = tp.tp_colpar_gemm_gelu(ref, w, None, 2, "gelu_tanh")
                torch.cuda.synchronize()
        for flags in ALL_OPTIONS[1:]:
            with launch_options(flags):
                y = x0
                bufs = [torch.empty_like(x0) for _ in range(2)]
                for i in range(steps):
                    y = tp.tp_colpar_gemm_gelu(y, w, None, 2, "gelu_tanh", out=bufs[i % 2])
                torch.cuda.synchronize()
            assert torch.equal(y, ref), flags
    _no_device_error()


def test_graph_replayed_decode_step_matches_eager(sq_weights):
    # the default bench step (T = 1, 8, 64 on the 4096 x 4096 projection, weights
    # rotated per call) captured in a CUDA graph gives the eager results bit for bit
    dev = _dev()
    cfg, w = sq_weights
    ws = [w.to(dev), (w.to(dev).float() * 0.5).to(torch.bfloat16)]
    xs = {T: workloads.proj_inputs(cfg, T)["x"].to(dev) for T in (1, 8, 64)}
    outs = {T: torch.empty((T, 4096), dtype=torch.bfloat16, device=dev) for T in xs}
    with launch_options(BENCH_OPTIONS):
        eager = {}
        for j, T in enumerate(xs):
            eager[T] = tp.tp_colpar_gemm_gelu(xs[T], ws[j % 2], None, 2, "none")
        s = torch.cuda.Stream()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for j, T in enumerate(xs):
                tp.tp_colpar_gemm_gelu(xs[T], ws[j % 2], None, 2, "none", out=outs[T])
        for _ in range(3):
            g.replay()
    torch.cuda.synchronize()
    _no_device_error()
    for T in xs:
        assert torch.equal(outs[T], eager[T])
    assert_parity(outs[64], oracle.colpar_linear(xs[64].cpu(), w, None, 2, "none"), "graph T=64")


def test_binding_checks_dtype_and_device_before_the_library():
    # no launch happens in any of these: the binding refuses first
    dev = _dev()
    x = torch.zeros(8, 256, dtype=torch.float32, device=dev)
    w = torch.zeros(1024, 256, dtype=torch.bfloat16, device=dev)
    with pytest.raises(TypeError):
        tp.tp_colpar_gemm_gelu(x, w, None, 2)
    xb = x.to(torch.bfloat16)
    with pytest.raises(ValueError):
        tp.tp_colpar_gemm_gelu(xb, w.cpu(), None, 2)
    with pytest.raises(ValueError):
        tp.tp_colpar_gemm_gelu(xb.cpu(), w, None, 2)
