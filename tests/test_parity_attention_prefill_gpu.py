"""GPU parity of the attention core for many new tokens (tp_attn_prefill)
against the fp64 attention oracle.

tp_attn_prefill appends the new tokens' keys and values to the caches and
computes ctx with the causal grouped-query softmax; oracle.attn_core does the
same shard by shard in float64 (pinned in test_oracle_attention.py).  Inputs
are the exact bf16 values both receive.  Acceptance as for decode: relative L2
error <= 1e-2 and max |error| <= 2e-2 * max |ref| on ctx (the softmax weights
are rounded to bf16 for the weighted sum of values), and bit-exact caches (the
appended rows equal qkv's K and V columns; every other row is unchanged).
Cache rows past the visible keys are NaN, so a read of any of them would show.

Shapes: the 70B head layout (64 query / 8 key-value heads of 128, t = 8) with
token counts on and off the 128-row tile and key-block boundaries, prompts
after a cache (chunked prefill), other grouped-query ratios (including a
ratio that is not a power of two), one token, peaked and growing scores that
make the running maximum move, and the full 4096-token workload on sampled
(token, head) rows.
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


def _case(nq, nkv, t, past, T, q_scale=1.0, k_ramp=0.0, seed=0, max_extra=29):
    """Seeded qkv, caches (NaN past the cached rows) and the oracle's result.
    k_ramp > 0 scales key j (cached and new) by 1 + k_ramp * j / 128, so later
    key blocks carry larger scores and the running maximum keeps rising."""
    nqkv = (nq + 2 * nkv) * D
    qkv = workloads.random_bf16_small((T, nqkv), 1.0, 5000 + seed)
    if q_scale != 1.0:
        qkv[:, :nq * D] = (qkv[:, :nq * D].float() * q_scale).to(torch.bfloat16)
    max_len = past + T + max_extra
    nan = torch.tensor(float("nan"), dtype=torch.bfloat16)
    kc = torch.full((nkv, max_len, D), nan, dtype=torch.bfloat16)
    vc = torch.full((nkv, max_len, D), nan, dtype=torch.bfloat16)
    if past > 0:
        kc[:, :past] = workloads.random_bf16_small((nkv, past, D), 1.0, 6000 + seed)
        vc[:, :past] = workloads.random_bf16_small((nkv, past, D), 1.0, 7000 + seed)
    if k_ramp > 0.0:
        ramp = 1.0 + k_ramp * torch.arange(past + T, dtype=torch.float32) / 128.0
        if past > 0:
            kc[:, :past] = (kc[:, :past].float() * ramp[:past, None]).to(torch.bfloat16)
        kcols = qkv[:, nq * D:(nq + nkv) * D].float() * ramp[past:, None]
        qkv[:, nq * D:(nq + nkv) * D] = kcols.to(torch.bfloat16)
    kh = nkv // t
    cache = [(kc[s * kh:(s + 1) * kh, :past], vc[s * kh:(s + 1) * kh, :past]) for s in range(t)]
    ctx_ref, grown = oracle.attn_core(qkv, nq, nkv, D, t, cache)
    return qkv, kc, vc, ctx_ref, grown


def _check_caches(kd, vd, kc, vc, grown, past, T, what):
    k_new = torch.from_numpy(np.concatenate([g[0] for g in grown], axis=0)).to(torch.bfloat16)
    v_new = torch.from_numpy(np.concatenate([g[1] for g in grown], axis=0)).to(torch.bfloat16)
    kg, vg = kd.cpu(), vd.cpu()
    assert torch.equal(kg[:, :past + T].view(torch.int16), k_new.view(torch.int16)), what
    assert torch.equal(vg[:, :past + T].view(torch.int16), v_new.view(torch.int16)), what
    assert torch.equal(kg[:, past + T:].view(torch.int16), kc[:, past + T:].view(torch.int16)), what
    assert torch.equal(vg[:, past + T:].view(torch.int16), vc[:, past + T:].view(torch.int16)), what


def _run(nq, nkv, t, past, T, **kw):
    dev = _dev()
    qkv, kc, vc, ctx_ref, grown = _case(nq, nkv, t, past, T, **kw)
    kd, vd = kc.to(dev), vc.to(dev)
    ctx = tp.tp_attn_prefill(qkv.to(dev), kd, vd, past, nq, nkv, D, t)
    torch.cuda.synchronize()
    assert tp.tp_device_error_check() == tp.TP_OK
    what = f"nq={nq} nkv={nkv} t={t} past={past} T={T} {kw}"
    _parity(ctx, ctx_ref, what)
    _check_caches(kd, vd, kc, vc, grown, past, T, what)
    return ctx


@pytest.mark.parametrize("T", [1, 2, 127, 128, 129, 255, 256, 300, 515])
def test_attn_prefill_70b_heads_prompt(T):
    _run(64, 8, 8, 0, T)


@pytest.mark.parametrize("past,T", [(1, 130), (127, 64), (128, 128), (1000, 200), (4095, 33),
                                    (2500, 600)])
def test_attn_prefill_70b_heads_after_cache(past, T):
    _run(64, 8, 8, past, T, seed=past + T)


@pytest.mark.parametrize("nq,nkv,t,past,T", [(32, 32, 4, 5, 77), (16, 1, 1, 0, 256),
                                             (8, 2, 2, 129, 517), (12, 4, 2, 100, 250),
                                             (4, 4, 1, 37, 1), (24, 8, 8, 0, 384)])
def test_attn_prefill_other_head_ratios(nq, nkv, t, past, T):
    _run(nq, nkv, t, past, T, seed=nq + T)


@pytest.mark.parametrize("past,T", [(0, 700), (300, 400)])
def test_attn_prefill_peaked_softmax(past, T):
    # large scores: most weight on a few keys (the maximum subtraction matters)
    _run(16, 2, 2, past, T, q_scale=6.0, seed=3)


@pytest.mark.parametrize("past,T", [(0, 1024), (640, 300)])
def test_attn_prefill_growing_scores_move_the_maximum(past, T):
    # later keys are larger, so most key blocks raise the running maximum past
    # the threshold at which O and l are rescaled
    _run(8, 1, 1, past, T, q_scale=2.0, k_ramp=1.0, seed=4)


def test_attn_prefill_bit_identical_on_repeat():
    dev = _dev()
    qkv, kc, vc, _, _ = _case(64, 8, 8, 200, 333, seed=9)
    q = qkv.to(dev)
    k1, v1 = kc.to(dev), vc.to(dev)
    k2, v2 = kc.to(dev), vc.to(dev)
    a = tp.tp_attn_prefill(q, k1, v1, 200, 64, 8, D, 8)
    b = tp.tp_attn_prefill(q, k2, v2, 200, 64, 8, D, 8)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_attn_prefill_chunks_match_one_prompt():
    # a 700-token prompt in three chunks through the cache gives the oracle's
    # one-shot result (and the same caches)
    dev = _dev()
    nq, nkv, t = 64, 8, 8
    qkv, kc, vc, ref, grown = _case(nq, nkv, t, 0, 700, seed=11)
    kd, vd = kc.to(dev), vc.to(dev)
    outs, start = [], 0
    for n in (256, 300, 144):
        outs.append(tp.tp_attn_prefill(qkv[start:start + n].to(dev), kd, vd, start, nq, nkv, D, t))
        start += n
    torch.cuda.synchronize()
    _parity(torch.cat(outs, 0), ref, "three chunks")
    _check_caches(kd, vd, kc, vc, grown, 0, 700, "three chunks")


def test_attn_prefill_then_decode_continue_the_same_cache():
    # prefill 400 tokens, then two decode steps over the cache it wrote
    dev = _dev()
    nq, nkv, t = 64, 8, 8
    qkv, kc, vc, ref, _ = _case(nq, nkv, t, 0, 402, seed=12)
    kd, vd = kc.to(dev), vc.to(dev)
    a = tp.tp_attn_prefill(qkv[:400].to(dev), kd, vd, 0, nq, nkv, D, t)
    b = tp.tp_attn_decode(qkv[400:401].to(dev), kd, vd, 400, nq, nkv, D, t)
    c = tp.tp_attn_decode(qkv[401:402].to(dev), kd, vd, 401, nq, nkv, D, t)
    torch.cuda.synchronize()
    _parity(torch.cat([a, b, c], 0), ref, "prefill + two decode steps")


def test_attn_prefill_bench_workload_sampled_rows():
    # the bench workload itself (a 4096-token prompt, 64 query / 8 key-value
    # heads, t = 8) in the launch configuration bench.py times; 48 seeded
    # (token, head) rows, tile edges included, against the oracle's one-head
    # attention over the keys each token sees
    dev = _dev()
    cfg = workloads.CONFIGS["attn70b_prefill"]
    nq, nkv, t = cfg.n_q_heads, cfg.n_kv_heads, cfg.tp_degrees[0]
    T = cfg.tokens[0]
    qkv = workloads.attn_decode_qkv(cfg, T)
    kd = torch.empty((nkv, T, D), dtype=torch.bfloat16, device=dev)
    vd = torch.empty_like(kd)
    prev = tp.tp_get_launch_options()
    tp.tp_set_launch_options(tp.TP_OPT_PDL | tp.TP_OPT_STATIC_WEIGHTS)
    try:
        ctx = tp.tp_attn_prefill(qkv.to(dev), kd, vd, 0, nq, nkv, D, t).cpu()
    finally:
        tp.tp_set_launch_options(prev)
    assert tp.tp_device_error_check() == tp.TP_OK
    rng = np.random.default_rng(0)
    toks = sorted(set([0, 127, 128, 2047, 4095] + list(rng.choice(T, 43, replace=False))))
    q64 = qkv.double().numpy()
    G = nq // nkv
    rows, refs = [], []
    for i in toks:
        h = int(rng.integers(nq))
        g = h // G
        q = q64[i:i + 1, h * D:(h + 1) * D]
        k = q64[:i + 1, (nq + g) * D:(nq + g + 1) * D]
        v = q64[:i + 1, (nq + nkv + g) * D:(nq + nkv + g + 1) * D]
        refs.append(oracle.attend_head(q, k, v, i)[0])
        rows.append(ctx[i, h * D:(h + 1) * D])
    _parity(torch.stack(rows), np.stack(refs), "bench workload sampled rows")
    # the caches hold every token's K and V columns
    kcols = qkv[:, nq * D:(nq + nkv) * D].reshape(T, nkv, D).transpose(0, 1)
    assert torch.equal(kd.cpu().view(torch.int16), kcols.contiguous().view(torch.int16))


def test_attn_prefill_after_cache_many_items_per_cta_sampled_rows():
    # 70B heads, a 2900-token chunk after 1500 cached tokens: 23 tiles x 32
    # head pairs, about five work items per SM of different lengths, a ragged
    # last tile; 40 seeded (token, head) rows against the oracle's one-head
    # attention over the cached and new keys each token sees
    dev = _dev()
    nq, nkv, t, past, T = 64, 8, 8, 1500, 2900
    nqkv = (nq + 2 * nkv) * D
    qkv = workloads.random_bf16_small((T, nqkv), 1.0, 5151)
    max_len = past + T + 7
    kc = torch.zeros((nkv, max_len, D), dtype=torch.bfloat16)
    vc = torch.zeros((nkv, max_len, D), dtype=torch.bfloat16)
    kc[:, :past] = workloads.random_bf16_small((nkv, past, D), 1.0, 6151)
    vc[:, :past] = workloads.random_bf16_small((nkv, past, D), 1.0, 7151)
    kd, vd = kc.to(dev), vc.to(dev)
    ctx = tp.tp_attn_prefill(qkv.to(dev), kd, vd, past, nq, nkv, D, t).cpu()
    assert tp.tp_device_error_check() == tp.TP_OK
    rng = np.random.default_rng(1)
    toks = sorted(set([0, 127, 128, 2815, 2816, T - 1] + list(rng.choice(T, 34, replace=False))))
    q64 = qkv.double().numpy()
    kc64, vc64 = kc.double().numpy(), vc.double().numpy()
    G = nq // nkv
    rows, refs = [], []
    for i in toks:
        h = int(rng.integers(nq))
        g = h // G
        q = q64[i:i + 1, h * D:(h + 1) * D]
        k = np.concatenate([kc64[g, :past], q64[:i + 1, (nq + g) * D:(nq + g + 1) * D]])
        v = np.concatenate([vc64[g, :past], q64[:i + 1, (nq + nkv + g) * D:(nq + nkv + g + 1) * D]])
        refs.append(oracle.attend_head(q, k, v, past + i)[0])
        rows.append(ctx[i, h * D:(h + 1) * D])
    _parity(torch.stack(rows), np.stack(refs), "after-cache chunk, sampled rows")
