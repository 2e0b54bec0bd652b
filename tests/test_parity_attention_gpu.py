"""GPU parity of the attention core (decode over a per-head KV cache) against
the fp64 attention oracle.

tp_attn_decode appends the new tokens' keys and values to the caches and
computes ctx for them; oracle.attn_core does the same shard by shard in
float64 (pinned in test_oracle_attention.py).  Inputs are the exact bf16
values both receive.  Acceptance: relative L2 error <= 1e-2 and max |error|
<= 2e-2 * max |ref| on ctx (the GPU rounds the softmax weights to bf16 for the
weighted sum of values: relative error 2^-9 per weight), and bit-exact cache
contents: the appended rows equal qkv's K and V columns and nothing else in
the caches changes.  Cache rows past the visible keys are filled with NaN, so
a read of any of them would show.  Shapes: the 70B head layout (64 query / 8
key-value heads of 128, t = 8) at cache lengths on and off the 128-key block
boundary, several new-token counts (one and several token groups), and other
grouped-query ratios.
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
D = 128


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


def _case(nq, nkv, t, past, T, q_scale=1.0, seed=0, max_extra=37):
    """Seeded qkv, caches (NaN past the cached rows) and the oracle's result."""
    nqkv = (nq + 2 * nkv) * D
    qkv = workloads.random_bf16_small((T, nqkv), 1.0, 1000 + seed)
    if q_scale != 1.0:
        qkv[:, :nq * D] = (qkv[:, :nq * D].float() * q_scale).to(torch.bfloat16)
    max_len = past + T + max_extra
    nan = torch.tensor(float("nan"), dtype=torch.bfloat16)
    kc = torch.full((nkv, max_len, D), nan, dtype=torch.bfloat16)
    vc = torch.full((nkv, max_len, D), nan, dtype=torch.bfloat16)
    if past > 0:
        kc[:, :past] = workloads.random_bf16_small((nkv, past, D), 1.0, 2000 + seed)
        vc[:, :past] = workloads.random_bf16_small((nkv, past, D), 1.0, 3000 + seed)
    kh = nkv // t
    cache = [(kc[s * kh:(s + 1) * kh, :past], vc[s * kh:(s + 1) * kh, :past]) for s in range(t)]
    ctx_ref, grown = oracle.attn_core(qkv, nq, nkv, D, t, cache)
    return qkv, kc, vc, ctx_ref, grown


def _run(nq, nkv, t, past, T, **kw):
    dev = _dev()
    qkv, kc, vc, ctx_ref, grown = _case(nq, nkv, t, past, T, **kw)
    kd, vd = kc.to(dev), vc.to(dev)
    ctx = tp.tp_attn_decode(qkv.to(dev), kd, vd, past, nq, nkv, D, t)
    torch.cuda.synchronize()
    assert tp.tp_device_error_check() == tp.TP_OK
    what = f"nq={nq} nkv={nkv} t={t} past={past} T={T}"
    _parity(ctx, ctx_ref, what)
    # the caches: cached rows untouched, new rows = K / V columns of qkv, the
    # rest untouched (still NaN)
    kh = nkv // t
    k_new = torch.from_numpy(np.concatenate([g[0] for g in grown], axis=0)).to(torch.bfloat16)
    v_new = torch.from_numpy(np.concatenate([g[1] for g in grown], axis=0)).to(torch.bfloat16)
    kg, vg = kd.cpu(), vd.cpu()
    assert torch.equal(kg[:, :past + T].view(torch.int16), k_new.view(torch.int16)), what
    assert torch.equal(vg[:, :past + T].view(torch.int16), v_new.view(torch.int16)), what
    assert torch.equal(kg[:, past + T:].view(torch.int16), kc[:, past + T:].view(torch.int16))
    assert torch.equal(vg[:, past + T:].view(torch.int16), vc[:, past + T:].view(torch.int16))
    assert kh * t == nkv
    return ctx


@pytest.mark.parametrize("past,T", [(0, 1), (1, 1), (127, 1), (128, 1), (1000, 4), (8191, 1),
                                    (300, 5), (4095, 16), (5000, 33), (20000, 2)])
def test_attn_decode_70b_heads(past, T):
    _run(64, 8, 8, past, T)


@pytest.mark.parametrize("past,T", [(513, 1), (2047, 3)])
def test_attn_decode_peaked_softmax(past, T):
    # large scores: most weight on a few keys (exercises the max subtraction)
    _run(64, 8, 8, past, T, q_scale=6.0, seed=5)


@pytest.mark.parametrize("nq,nkv,t,past,T", [(32, 32, 4, 700, 2), (16, 1, 1, 900, 3),
                                             (8, 2, 2, 129, 9), (4, 4, 1, 0, 40)])
def test_attn_decode_other_head_ratios(nq, nkv, t, past, T):
    _run(nq, nkv, t, past, T, seed=nq + T)


def test_attn_decode_bit_identical_on_repeat():
    dev = _dev()
    qkv, kc, vc, _, _ = _case(64, 8, 8, 3000, 2, seed=9)
    q = qkv.to(dev)
    k1, v1 = kc.to(dev), vc.to(dev)
    k2, v2 = kc.to(dev), vc.to(dev)
    a = tp.tp_attn_decode(q, k1, v1, 3000, 64, 8, D, 8)
    b = tp.tp_attn_decode(q, k2, v2, 3000, 64, 8, D, 8)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_attn_decode_chained_steps_match_one_prefill():
    # three decode steps through the cache give the oracle's one-shot result
    dev = _dev()
    nq, nkv, t = 64, 8, 8
    qkv, kc, vc, _, _ = _case(nq, nkv, t, 1200, 3, seed=11)
    kd, vd = kc.to(dev), vc.to(dev)
    outs = [tp.tp_attn_decode(qkv[i:i + 1].to(dev), kd, vd, 1200 + i, nq, nkv, D, t)
            for i in range(3)]
    torch.cuda.synchronize()
    kh = nkv // t
    cache = [(kc[s * kh:(s + 1) * kh, :1200], vc[s * kh:(s + 1) * kh, :1200]) for s in range(t)]
    ref, _ = oracle.attn_core(qkv, nq, nkv, D, t, cache)
    _parity(torch.cat(outs, 0), ref, "three chained steps")


def test_attn_decode_bench_workload_sizes():
    # the bench workload itself: 64K cached tokens of the 70B head layout,
    # T = 1, 2, 4, in the launch configuration bench.py times (programmatic
    # dependent launch with static-weight prefetch), against the oracle
    dev = _dev()
    cfg = workloads.CONFIGS["attn70b_decode"]
    nq, nkv, t = cfg.n_q_heads, cfg.n_kv_heads, cfg.tp_degrees[0]
    k, v = workloads.attn_decode_cache(cfg)
    kh = nkv // t
    cache = [(k[s * kh:(s + 1) * kh], v[s * kh:(s + 1) * kh]) for s in range(t)]
    max_len = cfg.past + max(cfg.tokens)
    kd = torch.empty((nkv, max_len, D), dtype=torch.bfloat16, device=dev)
    vd = torch.empty_like(kd)
    prev = tp.tp_get_launch_options()
    tp.tp_set_launch_options(tp.TP_OPT_PDL | tp.TP_OPT_STATIC_WEIGHTS)
    try:
        for T in cfg.tokens:
            kd[:, :cfg.past].copy_(k)
            vd[:, :cfg.past].copy_(v)
            qkv = workloads.attn_decode_qkv(cfg, T)
            ref, _ = oracle.attn_core(qkv, nq, nkv, D, t, cache)
            ctx = tp.tp_attn_decode(qkv.to(dev), kd, vd, cfg.past, nq, nkv, D, t)
            torch.cuda.synchronize()
            _parity(ctx, ref, f"bench workload T={T}")
    finally:
        tp.tp_set_launch_options(prev)
    assert tp.tp_device_error_check() == tp.TP_OK
