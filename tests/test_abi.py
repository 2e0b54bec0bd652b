"""The C ABI without a GPU: the library loads, exports every function the
header declares, and rejects bad arguments on the host before any CUDA call.

Only invalid argument combinations are passed here (with fake, never
dereferenced pointers); each returns its error code before the library
touches the CUDA runtime.
"""
import ctypes
import os
import re
import subprocess

import pytest

import tensor_transformer_linear_column_b200 as tp
from tensor_transformer_linear_column_b200 import build_lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tp_block.h")

GOOD = 0x10000          # 16-byte aligned fake device address, never dereferenced
ODD = 0x10008 + 1       # misaligned


@pytest.fixture(scope="module")
def lib():
    build_lib.build()
    return tp.load()


def _header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(tp_[a-z0-9_]+)\s*\(", text)
    return sorted(set(names))


def _header_enum(name):
    text = open(HEADER).read()
    return {k: int(v) for k, v in re.findall(rf"\b({name}[A-Z0-9_]*)\s*=\s*(\d+)", text)}


def test_header_declares_the_four_block_calls():
    fns = _header_functions()
    for f in ("tp_colpar_gemm_gelu", "tp_rowpar_gemm_reduce", "tp_mlp_forward",
              "tp_attn_proj_forward"):
        assert f in fns


def test_library_exports_every_declared_symbol(lib):
    declared = _header_functions()
    out = subprocess.run(["nm", "-D", "--defined-only", build_lib.LIB_PATH],
                         capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s+(\w+)$", out, flags=re.M))
    for name in declared:
        assert name in exported, name
        assert hasattr(lib, name)
    assert set(tp.SIGNATURES) == set(declared)


def test_status_and_act_codes_match_header():
    st = _header_enum("TP_ERR_")
    st.update(_header_enum("TP_OK"))
    for k, v in st.items():
        assert getattr(tp, k) == v
    for k, v in _header_enum("TP_ACT_").items():
        assert getattr(tp, k) == v


def test_status_strings(lib):
    for code in range(0, 9):
        s = tp.status_string(code)
        assert isinstance(s, str) and s and s != "unknown status"
    assert tp.status_string(99) == "unknown status"


def test_workspace_bytes(lib):
    assert tp.tp_mlp_workspace_bytes(1, 64) == 256
    assert tp.tp_mlp_workspace_bytes(8, 1024) == 8 * 1024 * 2
    assert tp.tp_mlp_workspace_bytes(3, 64) == 512
    assert tp.tp_mlp_workspace_bytes(0, 64) == 0
    assert tp.tp_mlp_workspace_bytes(8192, 53248) == 8192 * 53248 * 2


def _colpar(lib, x=GOOD, w=GOOD, b=None, T=8, K=256, N=1024, t=2, act=0, out=GOOD):
    return lib.tp_colpar_gemm_gelu(x, w, b, T, K, N, t, act, out, None)


def _rowpar(lib, h=GOOD, w=GOOD, b=None, T=8, K=1024, N=256, t=2, out=GOOD):
    return lib.tp_rowpar_gemm_reduce(h, w, b, T, K, N, t, out, None)


def test_colpar_rejects_bad_arguments(lib):
    assert _colpar(lib, x=None) == tp.TP_ERR_NULL
    assert _colpar(lib, w=None) == tp.TP_ERR_NULL
    assert _colpar(lib, out=None) == tp.TP_ERR_NULL
    assert _colpar(lib, x=ODD) == tp.TP_ERR_ALIGN
    assert _colpar(lib, b=ODD) == tp.TP_ERR_ALIGN
    assert _colpar(lib, T=0) == tp.TP_ERR_SHAPE
    assert _colpar(lib, T=-3) == tp.TP_ERR_SHAPE
    assert _colpar(lib, K=100) == tp.TP_ERR_SHAPE
    assert _colpar(lib, N=1000) == tp.TP_ERR_SHAPE
    assert _colpar(lib, act=7) == tp.TP_ERR_UNSUPPORTED
    assert _colpar(lib, t=0) == tp.TP_ERR_TP_DEGREE
    assert _colpar(lib, N=4096, t=3) == tp.TP_ERR_TP_DEGREE


def test_rowpar_rejects_bad_arguments(lib):
    assert _rowpar(lib, h=None) == tp.TP_ERR_NULL
    assert _rowpar(lib, w=ODD) == tp.TP_ERR_ALIGN
    assert _rowpar(lib, T=0) == tp.TP_ERR_SHAPE
    assert _rowpar(lib, t=3) == tp.TP_ERR_TP_DEGREE          # 1024 % 3 != 0
    assert _rowpar(lib, t=32) == tp.TP_ERR_TP_DEGREE         # shard width 32 < 64
    assert _rowpar(lib, t=-1) == tp.TP_ERR_TP_DEGREE


def test_w8_calls_reject_bad_arguments(lib):
    # every check here runs before any CUDA call, so no device is needed
    def col(x=GOOD, w=GOOD, sc=GOOD, T=8, K=256, N=1024, t=2, act=0):
        return lib.tp_colpar_gemm_gelu_w8(x, w, sc, None, T, K, N, t, act, GOOD, None)

    def row(h=GOOD, w=GOOD, sc=GOOD, T=8, K=1024, N=256, t=2):
        return lib.tp_rowpar_gemm_reduce_w8(h, w, sc, None, T, K, N, t, GOOD, None)

    def mlp(sc1=GOOD, sc2=GOOD, T=8, t=2, ws=GOOD, ws_bytes=1 << 20):
        return lib.tp_mlp_forward_w8(GOOD, GOOD, sc1, None, GOOD, sc2, None, T, 256, 1024, t, 1,
                                     GOOD, ws, ws_bytes, None)
    assert col(sc=None) == tp.TP_ERR_NULL
    assert col(w=None) == tp.TP_ERR_NULL
    assert col(sc=ODD) == tp.TP_ERR_ALIGN
    assert col(w=ODD) == tp.TP_ERR_ALIGN
    assert col(K=100) == tp.TP_ERR_SHAPE
    assert col(t=3) == tp.TP_ERR_TP_DEGREE
    assert col(act=9) == tp.TP_ERR_UNSUPPORTED
    assert col(T=129) == tp.TP_ERR_UNSUPPORTED        # decode path only
    assert row(sc=None) == tp.TP_ERR_NULL
    assert row(t=32) == tp.TP_ERR_TP_DEGREE
    assert row(T=200) == tp.TP_ERR_UNSUPPORTED
    assert mlp(sc2=None) == tp.TP_ERR_NULL
    assert mlp(sc1=ODD) == tp.TP_ERR_ALIGN
    assert mlp(t=3) == tp.TP_ERR_TP_DEGREE
    assert mlp(T=129) == tp.TP_ERR_UNSUPPORTED
    assert mlp(ws=None) == tp.TP_ERR_WORKSPACE


def test_mlp_rejects_bad_arguments(lib):
    def call(ws=GOOD, ws_bytes=1 << 20, t=2, F=1024, act=1, x=GOOD):
        return lib.tp_mlp_forward(x, GOOD, None, GOOD, None, 8, 256, F, t, act, GOOD, ws,
                                  ws_bytes, None)
    assert call(x=None) == tp.TP_ERR_NULL
    assert call(ws=None) == tp.TP_ERR_WORKSPACE
    assert call(ws_bytes=8 * 1024 * 2 - 1) == tp.TP_ERR_WORKSPACE
    assert call(ws=ODD) == tp.TP_ERR_ALIGN
    assert call(t=3) == tp.TP_ERR_TP_DEGREE
    assert call(t=32) == tp.TP_ERR_TP_DEGREE
    assert call(act=5) == tp.TP_ERR_UNSUPPORTED
    assert call(F=1000) == tp.TP_ERR_SHAPE


def test_backward_rejects_bad_arguments(lib):
    def call(x=GOOD, dy=GOOD, dx=GOOD, dw1=GOOD, dw2=GOOD, db1=None, ws=GOOD,
             ws_bytes=1 << 22, T=8, H=256, F=1024, t=2, act=1):
        return lib.tp_mlp_backward(x, GOOD, None, GOOD, dy, T, H, F, t, act, dx, dw1, db1, dw2,
                                   None, ws, ws_bytes, None)
    assert tp.tp_mlp_backward_workspace_bytes(8, 1024) == 3 * 8 * 1024 * 2
    assert tp.tp_mlp_backward_workspace_bytes(3, 64) == 3 * 512
    assert tp.tp_mlp_backward_workspace_bytes(0, 64) == 0
    assert call(x=None) == tp.TP_ERR_NULL
    assert call(dy=None) == tp.TP_ERR_NULL
    assert call(dw2=None) == tp.TP_ERR_NULL
    assert call(dx=ODD) == tp.TP_ERR_ALIGN
    assert call(db1=ODD) == tp.TP_ERR_ALIGN
    assert call(T=0) == tp.TP_ERR_SHAPE
    assert call(H=100) == tp.TP_ERR_SHAPE
    assert call(act=4) == tp.TP_ERR_UNSUPPORTED
    assert call(t=3) == tp.TP_ERR_TP_DEGREE
    assert call(t=32) == tp.TP_ERR_TP_DEGREE
    assert call(ws=None) == tp.TP_ERR_WORKSPACE
    assert call(ws_bytes=3 * 8 * 1024 * 2 - 1) == tp.TP_ERR_WORKSPACE
    assert call(ws=ODD) == tp.TP_ERR_ALIGN


def test_attn_decode_rejects_bad_arguments(lib):
    def call(qkv=GOOD, kc=GOOD, ctx=GOOD, T=1, past=10, max_len=64, nq=64, nkv=8, d=128, t=8,
             ws=GOOD, ws_bytes=1 << 24):
        return lib.tp_attn_decode(qkv, kc, GOOD, T, past, max_len, nq, nkv, d, t, ctx, ws,
                                  ws_bytes, None)
    assert tp.tp_attn_decode_workspace_bytes(1, 10, 64, 8, 128) > 0
    assert tp.tp_attn_decode_workspace_bytes(1, 10, 64, 8, 64) == 0      # d must be 128
    assert tp.tp_attn_decode_workspace_bytes(1, 10, 24, 8, 128) == 0     # G = 3
    assert call(qkv=None) == tp.TP_ERR_NULL
    assert call(kc=ODD) == tp.TP_ERR_ALIGN
    assert call(T=0) == tp.TP_ERR_SHAPE
    assert call(past=60, T=5) == tp.TP_ERR_SHAPE                       # past + T > max_len
    assert call(nq=60) == tp.TP_ERR_SHAPE                              # nkv does not divide nq
    assert call(d=64) == tp.TP_ERR_UNSUPPORTED
    assert call(nq=24) == tp.TP_ERR_UNSUPPORTED                        # G = 3
    assert call(t=3) == tp.TP_ERR_TP_DEGREE
    assert call(t=16) == tp.TP_ERR_TP_DEGREE                           # 8 kv heads: t <= 8
    assert call(ws=None) == tp.TP_ERR_WORKSPACE
    assert call(ws_bytes=tp.tp_attn_decode_workspace_bytes(1, 10, 64, 8, 128) - 1) == \
        tp.TP_ERR_WORKSPACE


def test_attn_prefill_rejects_bad_arguments(lib):
    def call(qkv=GOOD, kc=GOOD, vc=GOOD, ctx=GOOD, T=300, past=10, max_len=512, nq=64, nkv=8,
             d=128, t=8):
        return lib.tp_attn_prefill(qkv, kc, vc, T, past, max_len, nq, nkv, d, t, ctx, None)
    assert call(qkv=None) == tp.TP_ERR_NULL
    assert call(vc=None) == tp.TP_ERR_NULL
    assert call(ctx=None) == tp.TP_ERR_NULL
    assert call(kc=ODD) == tp.TP_ERR_ALIGN
    assert call(ctx=ODD) == tp.TP_ERR_ALIGN
    assert call(T=0) == tp.TP_ERR_SHAPE
    assert call(past=-1) == tp.TP_ERR_SHAPE
    assert call(past=300, T=300) == tp.TP_ERR_SHAPE                    # past + T > max_len
    assert call(nq=60) == tp.TP_ERR_SHAPE                              # nkv does not divide nq
    assert call(T=65536 * 128, max_len=65536 * 128 + 10) == tp.TP_ERR_SHAPE  # > 65535 tiles
    assert call(d=64) == tp.TP_ERR_UNSUPPORTED
    assert call(t=3) == tp.TP_ERR_TP_DEGREE
    assert call(t=16) == tp.TP_ERR_TP_DEGREE                           # 8 kv heads: t <= 8


def test_sp_norm_rejects_bad_arguments(lib):
    def call(y=GOOD, g=GOOD, T=16, H=256, t=4, eps=1e-5, r=GOOD):
        return lib.tp_sp_add_rmsnorm(y, GOOD, g, T, H, t, eps, r, GOOD, None)
    assert call(y=None) == tp.TP_ERR_NULL
    assert call(g=None) == tp.TP_ERR_NULL
    assert call(r=ODD) == tp.TP_ERR_ALIGN
    assert call(T=0) == tp.TP_ERR_SHAPE
    assert call(H=100) == tp.TP_ERR_SHAPE
    assert call(eps=-1.0) == tp.TP_ERR_SHAPE
    assert call(eps=float("nan")) == tp.TP_ERR_SHAPE
    assert call(t=3) == tp.TP_ERR_TP_DEGREE        # 16 tokens do not split 3 ways
    assert call(t=0) == tp.TP_ERR_TP_DEGREE


def test_attention_head_rules_from_the_pages(lib, golden):
    g = golden["head_divisibility"]

    def call(t, nq=g["n_q_heads"], nkv=g["n_kv_heads"], d=128):
        return lib.tp_attn_proj_forward(GOOD, GOOD, None, GOOD, GOOD, None, 16, 8192, nq, nkv,
                                        d, t, GOOD, GOOD, None)
    for t in g["tp_degrees_that_fail"]:
        assert call(t) == tp.TP_ERR_TP_DEGREE
    # more shards than key-value heads would need replicated heads: rejected
    assert call(16) == tp.TP_ERR_TP_DEGREE
    assert call(0) == tp.TP_ERR_TP_DEGREE
    # a head group narrower than 64 columns cannot be a shard here
    assert call(8, nq=8, nkv=8, d=32) == tp.TP_ERR_TP_DEGREE
    assert call(1, d=6) == tp.TP_ERR_SHAPE                   # (64 + 16) * 6 columns


def test_decode_threshold_setting(lib):
    prev = tp.tp_get_decode_max_tokens()
    try:
        assert lib.tp_set_decode_max_tokens(-1) == tp.TP_ERR_UNSUPPORTED
        assert lib.tp_set_decode_max_tokens(129) == tp.TP_ERR_UNSUPPORTED
        tp.tp_set_decode_max_tokens(0)
        assert tp.tp_get_decode_max_tokens() == 0
        tp.tp_set_decode_max_tokens(128)
        assert tp.tp_get_decode_max_tokens() == 128
    finally:
        tp.tp_set_decode_max_tokens(prev)


def test_python_binding_rejects_host_tensors():
    # host pointers handed to a kernel would fault: every wrapper refuses
    # non-CUDA inputs before it reaches the library
    import torch
    bf = torch.bfloat16
    x = torch.zeros(8, 256, dtype=bf)
    w1, w2 = torch.zeros(1024, 256, dtype=bf), torch.zeros(256, 1024, dtype=bf)
    q1, q2 = torch.zeros(1024, 256, dtype=torch.uint8), torch.zeros(256, 1024, dtype=torch.uint8)
    s1, s2 = torch.ones(1024), torch.ones(256)
    h = torch.zeros(8, 1024, dtype=bf)
    calls = [
        lambda: tp.tp_colpar_gemm_gelu(x, w1, None, 2),
        lambda: tp.tp_rowpar_gemm_reduce(h, w2, None, 2),
        lambda: tp.tp_mlp_forward(x, w1, None, w2, None, 2),
        lambda: tp.tp_mlp_forward_noalloc(x, w1, None, w2, None, 2),
        lambda: tp.tp_colpar_gemm_gelu_w8(x, q1, s1, None, 2),
        lambda: tp.tp_rowpar_gemm_reduce_w8(h, q2, s2, None, 2),
        lambda: tp.tp_mlp_forward_w8(x, q1, s1, None, q2, s2, None, 2),
        lambda: tp.tp_attn_proj_forward(x, torch.zeros(384, 256, dtype=bf), None,
                                        torch.zeros(8, 256, dtype=bf),
                                        torch.zeros(256, 256, dtype=bf), None, 4, 1, 64, 1),
    ]
    for c in calls:
        with pytest.raises(ValueError, match="CUDA tensors"):
            c()


def test_launch_options_setting(lib):
    prev = tp.tp_get_launch_options()
    try:
        assert prev & tp.TP_OPT_PDL  # on by default
        assert lib.tp_set_launch_options(4) == tp.TP_ERR_UNSUPPORTED
        assert tp.tp_get_launch_options() == prev
        tp.tp_set_launch_options(tp.TP_OPT_PDL | tp.TP_OPT_STATIC_WEIGHTS)
        assert tp.tp_get_launch_options() == 3
        tp.tp_set_launch_options(0)
        assert tp.tp_get_launch_options() == 0
    finally:
        tp.tp_set_launch_options(prev)


# ---------------------------------------------------------------- launch plans (host only)

def test_stream_plan_of_the_sq4096_decode_launches():
    # the launches the GPU made for the 4096 x 4096 decode step (T = 1, 8, 64),
    # as an ncu capture recorded them: 32 n-tiles x clusters of 8 CTAs along K,
    # dynamic shared memory per CTA in bytes
    expected = {1: (256, 8, 58512), 8: (256, 8, 60560), 64: (256, 8, 109712)}
    for T, (grid, cluster, smem) in expected.items():
        p = tp.tp_stream_plan(T, 4096, 4096)
        assert p["grid_x"] * p["cluster"] == grid
        assert p["cluster"] == cluster
        assert p["smem_bytes"] == smem


def test_stream_plan_ring_depths_of_the_70b_decode():
    # 8-bit codes are converted into tensor memory, so a stage holds only the
    # code tiles + x; two k-blocks per box (16 KB requests) where four such
    # stages fit the ring's budget
    for T, stages, kpb in ((1, 5, 2), (16, 5, 2), (64, 6, 1)):
        p = tp.tp_stream_plan(T, 8192, 28672, 1, w8=True)
        assert p["stages"] == stages and p["kblocks_per_box"] == kpb, (T, p)
        t_pad = (T + 15) // 16 * 16
        assert p["stage_bytes"] == kpb * (64 + t_pad) * 64 * 2
    # bf16 up-projection at T = 1: two k-blocks per box, three boxes in flight
    p = tp.tp_stream_plan(1, 8192, 28672)
    assert p["kblocks_per_box"] == 2 and p["stages"] == 3


@pytest.mark.parametrize("w8", [False, True])
def test_stream_plan_invariants(w8):
    sms, max_smem = tp.B200_SMS, tp.B200_MAX_SMEM
    checked = 0
    for T in (1, 2, 15, 16, 17, 33, 64, 65, 100, 128):
        for K, N in ((64, 64), (256, 1088), (4096, 4096), (8192, 28672), (28672, 8192),
                     (16384, 192), (576, 320)):
            for shards in (1, 2, 3, 4, 8, 16):
                if K % shards or (K // shards) % 64:
                    continue
                try:
                    p = tp.tp_stream_plan(T, K, N, shards, w8)
                except tp.TPError as e:
                    assert e.status == tp.TP_ERR_UNSUPPORTED
                    continue
                checked += 1
                t_pad = (T + 15) // 16 * 16
                assert p["grid_x"] == (N + 127) // 128
                assert p["cluster"] in (1, 2, 4, 8)
                if p["cluster"] >= shards:
                    assert p["jsplit"] * shards == p["cluster"] and p["shards_per_cta"] == 1
                else:
                    assert p["jsplit"] == 1 and p["shards_per_cta"] * p["cluster"] == shards
                    assert t_pad <= 64  # the running sum of several shards lives in registers
                assert 2 <= p["stages"] <= (12 if w8 else 8)
                assert p["kblocks_per_box"] in (1, 2)
                w_row = 64 if w8 else 128  # bytes per weight row of a k-block
                assert p["stage_bytes"] == p["kblocks_per_box"] * (w_row + t_pad) * 128
                # the CTAs an SM can hold never need more TMEM than it has:
                # two accumulator regions (+ four 32-column A slots for 8-bit)
                tcols = max(32, 1 << (t_pad - 1).bit_length())
                need = 2 * tcols + (128 if w8 else 0)
                alloc = 1 << (need - 1).bit_length()
                by_regs = 2 if p["shards_per_cta"] > 1 else 3
                by_smem = (228 * 1024) // (p["smem_bytes"] + 1024)
                assert min(by_regs, by_smem) * alloc <= 512, (T, K, N, shards, w8, p)
                assert p["smem_bytes"] <= max_smem
                assert p["smem_bytes"] >= p["stages"] * p["stage_bytes"]
                if w8:
                    assert p["shards_per_cta"] <= 2
                    assert p["kblocks_per_box"] == 1 or p["shards_per_cta"] == 1
                # every CTA resident at once whenever some cluster shape allows it
                if p["grid_x"] * p["cluster"] > 2 * sms:
                    assert p["cluster"] == 1 or shards > 1
    assert checked > 100


def test_stream_plan_errors(lib):
    with pytest.raises(tp.TPError) as e:
        tp.tp_stream_plan(129, 4096, 4096)
    assert e.value.status == tp.TP_ERR_UNSUPPORTED
    with pytest.raises(tp.TPError) as e:  # 8-bit: three shards would share one CTA
        tp.tp_stream_plan(5, 576, 256, 3, w8=True)
    assert e.value.status == tp.TP_ERR_UNSUPPORTED
    assert tp.tp_stream_plan(5, 576, 256, 3)["shards_per_cta"] == 3  # bf16 takes it
    with pytest.raises(tp.TPError) as e:
        tp.tp_stream_plan(8, 4096, 4096, 3)
    assert e.value.status == tp.TP_ERR_TP_DEGREE
    with pytest.raises(tp.TPError) as e:
        tp.tp_stream_plan(8, 100, 4096)
    assert e.value.status == tp.TP_ERR_SHAPE
    assert lib.tp_stream_plan(8, 4096, 4096, 1, 0, 148, 232448, None) == tp.TP_ERR_NULL
