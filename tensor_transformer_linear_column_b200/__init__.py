"""Python binding of libtp_block.so (include/tp_block.h): argument marshalling only.

Every function here takes torch tensors that already live on the current CUDA
device, checks dtype / device / contiguity, and passes raw pointers, sizes and
the current stream to the C ABI of the same name.  All arithmetic runs in the
library's CUDA kernels; there is no fallback of any kind: if the shared library
is missing or fails to load, the first call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

from .build_lib import LIB_PATH

TP_OK = 0
TP_ERR_NULL = 1
TP_ERR_ALIGN = 2
TP_ERR_SHAPE = 3
TP_ERR_TP_DEGREE = 4
TP_ERR_WORKSPACE = 5
TP_ERR_UNSUPPORTED = 6
TP_ERR_CUDA = 7
TP_ERR_DEVICE_TIMEOUT = 8

TP_ACT_NONE = 0
TP_ACT_GELU_TANH = 1

TP_OPT_PDL = 1
TP_OPT_STATIC_WEIGHTS = 2

ACTS = {"none": TP_ACT_NONE, "gelu_tanh": TP_ACT_GELU_TANH}

# name -> (restype, argtypes) of every symbol declared in include/tp_block.h
_P = ctypes.c_void_p
_I = ctypes.c_int
_Z = ctypes.c_size_t
SIGNATURES = {
    "tp_colpar_gemm_gelu": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _P, _P]),
    "tp_rowpar_gemm_reduce": (_I, [_P, _P, _P, _I, _I, _I, _I, _P, _P]),
    "tp_mlp_workspace_bytes": (_Z, [_I, _I]),
    "tp_mlp_forward": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _Z, _P]),
    "tp_attn_proj_forward": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P]),
    "tp_mlp_forward_noalloc": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P]),
    "tp_mlp_backward_workspace_bytes": (_Z, [_I, _I]),
    "tp_attn_decode_workspace_bytes": (_Z, [_I, _I, _I, _I, _I]),
    "tp_sp_add_rmsnorm": (_I, [_P, _P, _P, _I, _I, _I, ctypes.c_float, _P, _P, _P]),
    "tp_attn_decode": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _P, _Z, _P]),
    "tp_attn_prefill": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _P]),
    "tp_mlp_backward": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _Z,
                             _P]),
    "tp_colpar_gemm_gelu_w8": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P]),
    "tp_rowpar_gemm_reduce_w8": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _P, _P]),
    "tp_mlp_forward_w8": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _Z, _P]),
    "tp_status_string": (ctypes.c_char_p, [_I]),
    "tp_last_cuda_error": (ctypes.c_char_p, []),
    "tp_device_error_check": (_I, []),
    "tp_diag_bounded_wait": (_I, [ctypes.c_uint, _P, _P]),
    "tp_set_decode_max_tokens": (_I, [_I]),
    "tp_get_decode_max_tokens": (_I, []),
    "tp_set_launch_options": (_I, [ctypes.c_uint]),
    "tp_get_launch_options": (ctypes.c_uint, []),
    "tp_stream_plan": (_I, [_I, _I, _I, _I, _I, _I, _I, _P]),
}


class StreamPlan(ctypes.Structure):
    """tp_stream_plan_t of include/tp_block.h."""
    _fields_ = [(name, ctypes.c_int) for name in (
        "grid_x", "cluster", "jsplit", "shards_per_cta", "stages", "kblocks_per_box",
        "stage_bytes", "smem_bytes", "l2_ahead")]


# a B200: 148 multiprocessors, 227 KB of opt-in shared memory per block
B200_SMS = 148
B200_MAX_SMEM = 232448


class TPError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = f"{where}: status {status} ({status_string(status)})"
        if status == TP_ERR_CUDA:
            msg += f": {load().tp_last_cuda_error().decode()}"
        super().__init__(msg)


_lib: Optional[ctypes.CDLL] = None


def library_path() -> str:
    return LIB_PATH


def load() -> ctypes.CDLL:
    """Load the shared library (raises if it is absent: build it first)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing; build it with "
                "`python -m tensor_transformer_linear_column_b200.build_lib`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def status_string(status: int) -> str:
    return load().tp_status_string(int(status)).decode()


def _ptr(t: Optional[torch.Tensor], name: str, dev: torch.device) -> Optional[int]:
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != torch.bfloat16:
        raise TypeError(f"{name} must be bfloat16, got {t.dtype}")
    if t.device != dev:
        raise ValueError(f"{name} is on {t.device}, expected {dev}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _ptr_typed(t: Optional[torch.Tensor], name: str, dev: torch.device,
               dtype: torch.dtype) -> Optional[int]:
    """Like _ptr for the 8-bit weight bytes (uint8) and their fp32 scales."""
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.device != dev:
        raise ValueError(f"{name} is on {t.device}, expected {dev}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _device(t: torch.Tensor) -> torch.device:
    """The device of a call: that of its first tensor, which must be the current
    CUDA device (the library launches there; a host or other-device pointer
    handed to a kernel would fault)."""
    if not isinstance(t, torch.Tensor) or t.device.type != "cuda":
        raise ValueError("inputs must be CUDA tensors")
    cur = torch.cuda.current_device()
    if t.device.index != cur:
        raise ValueError(f"inputs are on {t.device} but the current device is cuda:{cur}; "
                         f"call under torch.cuda.device({t.device.index})")
    return t.device


def _stream(stream: Optional[torch.cuda.Stream]) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if stream.device.index != torch.cuda.current_device():
        raise ValueError(f"stream is on {stream.device}, not the current device")
    return stream.cuda_stream


def _check(status: int, where: str) -> None:
    if status != TP_OK:
        raise TPError(status, where)


def _act(act) -> int:
    return ACTS[act] if isinstance(act, str) else int(act)


def tp_colpar_gemm_gelu(x: torch.Tensor, w: torch.Tensor, b: Optional[torch.Tensor],
                        tp_degree: int, act="none", out: Optional[torch.Tensor] = None,
                        stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """out[T, N] = act(x[T, K] @ w[N, K]^T + b) with the output split in tp_degree shards."""
    T, K = x.shape
    N = w.shape[0]
    if w.shape[1] != K:
        raise ValueError("w must be [N, K]")
    dev = _device(x)
    if out is None:
        out = torch.empty((T, N), dtype=torch.bfloat16, device=dev)
    st = load().tp_colpar_gemm_gelu(_ptr(x, "x", dev), _ptr(w, "w", dev), _ptr(b, "b", dev),
                                    T, K, N, int(tp_degree), _act(act), _ptr(out, "out", dev),
                                    _stream(stream))
    _check(st, "tp_colpar_gemm_gelu")
    return out


def tp_rowpar_gemm_reduce(h: torch.Tensor, w: torch.Tensor, b: Optional[torch.Tensor],
                          tp_degree: int, out: Optional[torch.Tensor] = None,
                          stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """out[T, N] = sum_s h[:, K_s] @ w[:, K_s]^T + b over tp_degree shards of K."""
    T, K = h.shape
    N = w.shape[0]
    if w.shape[1] != K:
        raise ValueError("w must be [N, K]")
    dev = _device(h)
    if out is None:
        out = torch.empty((T, N), dtype=torch.bfloat16, device=dev)
    st = load().tp_rowpar_gemm_reduce(_ptr(h, "h", dev), _ptr(w, "w", dev), _ptr(b, "b", dev),
                                      T, K, N, int(tp_degree), _ptr(out, "out", dev),
                                      _stream(stream))
    _check(st, "tp_rowpar_gemm_reduce")
    return out


def tp_mlp_workspace_bytes(T: int, F: int) -> int:
    return int(load().tp_mlp_workspace_bytes(int(T), int(F)))


def tp_mlp_forward(x: torch.Tensor, w1: torch.Tensor, b1: Optional[torch.Tensor],
                   w2: torch.Tensor, b2: Optional[torch.Tensor], tp_degree: int,
                   act="gelu_tanh", out: Optional[torch.Tensor] = None,
                   workspace: Optional[torch.Tensor] = None,
                   stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """The tensor-parallel MLP block y = sum_s act(x W1_s^T + b1_s) W2[:, s]^T + b2."""
    T, H = x.shape
    F = w1.shape[0]
    if w1.shape[1] != H or tuple(w2.shape) != (H, F):
        raise ValueError("w1 must be [F, H] and w2 [H, F]")
    dev = _device(x)
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    need = tp_mlp_workspace_bytes(T, F)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    if workspace.device != dev or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous tensor on the same device")
    ws_bytes = workspace.numel() * workspace.element_size()
    st = load().tp_mlp_forward(_ptr(x, "x", dev), _ptr(w1, "w1", dev), _ptr(b1, "b1", dev),
                               _ptr(w2, "w2", dev), _ptr(b2, "b2", dev), T, H, F,
                               int(tp_degree), _act(act), _ptr(out, "out", dev),
                               workspace.data_ptr(), ws_bytes, _stream(stream))
    _check(st, "tp_mlp_forward")
    return out


def tp_mlp_backward_workspace_bytes(T: int, F: int) -> int:
    return int(load().tp_mlp_backward_workspace_bytes(int(T), int(F)))


def tp_mlp_backward(x: torch.Tensor, w1: torch.Tensor, b1: Optional[torch.Tensor],
                    w2: torch.Tensor, dy: torch.Tensor, tp_degree: int, act="gelu_tanh",
                    with_bias_grads: bool = True, workspace: Optional[torch.Tensor] = None,
                    stream: Optional[torch.cuda.Stream] = None) -> dict:
    """Gradients of the tensor-parallel MLP block for the upstream gradient dy:
    {"dx", "dw1", "db1", "dw2", "db2"} (the bias gradients only if asked)."""
    T, H = x.shape
    F = w1.shape[0]
    if w1.shape[1] != H or tuple(w2.shape) != (H, F) or tuple(dy.shape) != (T, H):
        raise ValueError("w1 must be [F, H], w2 [H, F] and dy [T, H]")
    dev = _device(x)
    out = {"dx": torch.empty((T, H), dtype=torch.bfloat16, device=dev),
           "dw1": torch.empty((F, H), dtype=torch.bfloat16, device=dev),
           "dw2": torch.empty((H, F), dtype=torch.bfloat16, device=dev),
           "db1": torch.empty((F,), dtype=torch.bfloat16, device=dev) if with_bias_grads else None,
           "db2": torch.empty((H,), dtype=torch.bfloat16, device=dev) if with_bias_grads else None}
    need = tp_mlp_backward_workspace_bytes(T, F)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    if workspace.device != dev or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous tensor on the same device")
    st = load().tp_mlp_backward(
        _ptr(x, "x", dev), _ptr(w1, "w1", dev), _ptr(b1, "b1", dev), _ptr(w2, "w2", dev),
        _ptr(dy, "dy", dev), T, H, F, int(tp_degree), _act(act), _ptr(out["dx"], "dx", dev),
        _ptr(out["dw1"], "dw1", dev), _ptr(out["db1"], "db1", dev), _ptr(out["dw2"], "dw2", dev),
        _ptr(out["db2"], "db2", dev), workspace.data_ptr(),
        workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "tp_mlp_backward")
    return out


def tp_colpar_gemm_gelu_w8(x: torch.Tensor, w8: torch.Tensor, w_scale: torch.Tensor,
                           b: Optional[torch.Tensor], tp_degree: int, act="none",
                           out: Optional[torch.Tensor] = None,
                           stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """tp_colpar_gemm_gelu with an 8-bit weight: w8 [N, K] E4M3 bytes (uint8) and
    w_scale [N] fp32, W[n, k] = w_scale[n] * e4m3(w8[n, k])."""
    T, K = x.shape
    N = w8.shape[0]
    if w8.shape[1] != K or tuple(w_scale.shape) != (N,):
        raise ValueError("w8 must be [N, K] and w_scale [N]")
    dev = _device(x)
    if out is None:
        out = torch.empty((T, N), dtype=torch.bfloat16, device=dev)
    st = load().tp_colpar_gemm_gelu_w8(
        _ptr(x, "x", dev), _ptr_typed(w8, "w8", dev, torch.uint8),
        _ptr_typed(w_scale, "w_scale", dev, torch.float32), _ptr(b, "b", dev), T, K, N,
        int(tp_degree), _act(act), _ptr(out, "out", dev), _stream(stream))
    _check(st, "tp_colpar_gemm_gelu_w8")
    return out


def tp_rowpar_gemm_reduce_w8(h: torch.Tensor, w8: torch.Tensor, w_scale: torch.Tensor,
                             b: Optional[torch.Tensor], tp_degree: int,
                             out: Optional[torch.Tensor] = None,
                             stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """tp_rowpar_gemm_reduce with an 8-bit weight (see tp_colpar_gemm_gelu_w8)."""
    T, K = h.shape
    N = w8.shape[0]
    if w8.shape[1] != K or tuple(w_scale.shape) != (N,):
        raise ValueError("w8 must be [N, K] and w_scale [N]")
    dev = _device(h)
    if out is None:
        out = torch.empty((T, N), dtype=torch.bfloat16, device=dev)
    st = load().tp_rowpar_gemm_reduce_w8(
        _ptr(h, "h", dev), _ptr_typed(w8, "w8", dev, torch.uint8),
        _ptr_typed(w_scale, "w_scale", dev, torch.float32), _ptr(b, "b", dev), T, K, N,
        int(tp_degree), _ptr(out, "out", dev), _stream(stream))
    _check(st, "tp_rowpar_gemm_reduce_w8")
    return out


def tp_mlp_forward_w8(x: torch.Tensor, w1: torch.Tensor, s1: torch.Tensor,
                      b1: Optional[torch.Tensor], w2: torch.Tensor, s2: torch.Tensor,
                      b2: Optional[torch.Tensor], tp_degree: int, act="gelu_tanh",
                      out: Optional[torch.Tensor] = None,
                      workspace: Optional[torch.Tensor] = None,
                      stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """tp_mlp_forward with 8-bit weights: w1 [F, H] and w2 [H, F] E4M3 bytes,
    s1 [F] and s2 [H] fp32 row scales."""
    T, H = x.shape
    F = w1.shape[0]
    if w1.shape[1] != H or tuple(w2.shape) != (H, F):
        raise ValueError("w1 must be [F, H] and w2 [H, F]")
    if tuple(s1.shape) != (F,) or tuple(s2.shape) != (H,):
        raise ValueError("s1 must be [F] and s2 [H]")
    dev = _device(x)
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    need = tp_mlp_workspace_bytes(T, F)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    if workspace.device != dev or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous tensor on the same device")
    ws_bytes = workspace.numel() * workspace.element_size()
    st = load().tp_mlp_forward_w8(
        _ptr(x, "x", dev), _ptr_typed(w1, "w1", dev, torch.uint8),
        _ptr_typed(s1, "s1", dev, torch.float32), _ptr(b1, "b1", dev),
        _ptr_typed(w2, "w2", dev, torch.uint8), _ptr_typed(s2, "s2", dev, torch.float32),
        _ptr(b2, "b2", dev), T, H, F, int(tp_degree), _act(act), _ptr(out, "out", dev),
        workspace.data_ptr(), ws_bytes, _stream(stream))
    _check(st, "tp_mlp_forward_w8")
    return out


TP_NOALLOC_SCRATCH_BYTES = 4 * 1024 * 1024


def tp_mlp_forward_noalloc(x: torch.Tensor, w1: torch.Tensor, b1: Optional[torch.Tensor],
                           w2: torch.Tensor, b2: Optional[torch.Tensor], tp_degree: int,
                           act="gelu_tanh", out: Optional[torch.Tensor] = None,
                           stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """tp_mlp_forward without a workspace, for callers that cannot allocate device
    memory: h lives in the library's own TP_NOALLOC_SCRATCH_BYTES device array,
    shared by every call on the device (calls that may overlap on the GPU race)."""
    T, H = x.shape
    F = w1.shape[0]
    if w1.shape[1] != H or tuple(w2.shape) != (H, F):
        raise ValueError("w1 must be [F, H] and w2 [H, F]")
    dev = _device(x)
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    st = load().tp_mlp_forward_noalloc(_ptr(x, "x", dev), _ptr(w1, "w1", dev),
                                       _ptr(b1, "b1", dev), _ptr(w2, "w2", dev),
                                       _ptr(b2, "b2", dev), T, H, F, int(tp_degree), _act(act),
                                       _ptr(out, "out", dev), _stream(stream))
    _check(st, "tp_mlp_forward_noalloc")
    return out


def tp_attn_proj_forward(x: torch.Tensor, w_qkv: torch.Tensor, b_qkv: Optional[torch.Tensor],
                         ctx: torch.Tensor, w_o: torch.Tensor, b_o: Optional[torch.Tensor],
                         n_q_heads: int, n_kv_heads: int, head_dim: int, tp_degree: int,
                         qkv_out: Optional[torch.Tensor] = None,
                         out: Optional[torch.Tensor] = None,
                         stream: Optional[torch.cuda.Stream] = None):
    """(qkv, y): the head-split QKV projection and the row-parallel output projection."""
    T, H = x.shape
    dev = _device(x)
    nqkv = (n_q_heads + 2 * n_kv_heads) * head_dim
    if qkv_out is None:
        qkv_out = torch.empty((T, nqkv), dtype=torch.bfloat16, device=dev)
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    st = load().tp_attn_proj_forward(_ptr(x, "x", dev), _ptr(w_qkv, "w_qkv", dev),
                                     _ptr(b_qkv, "b_qkv", dev), _ptr(ctx, "ctx", dev),
                                     _ptr(w_o, "w_o", dev), _ptr(b_o, "b_o", dev), T, H,
                                     int(n_q_heads), int(n_kv_heads), int(head_dim),
                                     int(tp_degree), _ptr(qkv_out, "qkv_out", dev),
                                     _ptr(out, "out", dev), _stream(stream))
    _check(st, "tp_attn_proj_forward")
    return qkv_out, out


def tp_attn_decode_workspace_bytes(T: int, past: int, n_q_heads: int, n_kv_heads: int,
                                   head_dim: int) -> int:
    return int(load().tp_attn_decode_workspace_bytes(int(T), int(past), int(n_q_heads),
                                                     int(n_kv_heads), int(head_dim)))


def tp_attn_decode(qkv: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, past: int,
                   n_q_heads: int, n_kv_heads: int, head_dim: int, tp_degree: int,
                   ctx: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                   stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """ctx [T, nq d] of T new tokens (qkv [T, (nq + 2 nkv) d]) over the caches
    k_cache, v_cache [nkv, max_len, d] holding `past` tokens; appends the new
    tokens' keys and values to the caches in place."""
    T = qkv.shape[0]
    if qkv.shape[1] != (n_q_heads + 2 * n_kv_heads) * head_dim:
        raise ValueError("qkv must be [T, (nq + 2 nkv) d]")
    if k_cache.dim() != 3 or tuple(k_cache.shape) != tuple(v_cache.shape) or \
            k_cache.shape[0] != n_kv_heads or k_cache.shape[2] != head_dim:
        raise ValueError("caches must be [nkv, max_len, d]")
    dev = _device(qkv)
    if ctx is None:
        ctx = torch.empty((T, n_q_heads * head_dim), dtype=torch.bfloat16, device=dev)
    need = tp_attn_decode_workspace_bytes(T, past, n_q_heads, n_kv_heads, head_dim)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    if workspace.device != dev or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous tensor on the same device")
    st = load().tp_attn_decode(_ptr(qkv, "qkv", dev), _ptr(k_cache, "k_cache", dev),
                               _ptr(v_cache, "v_cache", dev), T, int(past), k_cache.shape[1],
                               int(n_q_heads), int(n_kv_heads), int(head_dim), int(tp_degree),
                               _ptr(ctx, "ctx", dev), workspace.data_ptr(),
                               workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "tp_attn_decode")
    return ctx


def tp_attn_prefill(qkv: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, past: int,
                    n_q_heads: int, n_kv_heads: int, head_dim: int, tp_degree: int,
                    ctx: Optional[torch.Tensor] = None,
                    stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """The attention core for many new tokens at once (a prompt or a chunk of
    one): ctx [T, nq d] of qkv [T, (nq + 2 nkv) d] over the caches k_cache,
    v_cache [nkv, max_len, d] holding `past` tokens; appends the new tokens'
    keys and values to the caches in place.  Needs no workspace."""
    T = qkv.shape[0]
    if qkv.shape[1] != (n_q_heads + 2 * n_kv_heads) * head_dim:
        raise ValueError("qkv must be [T, (nq + 2 nkv) d]")
    if k_cache.dim() != 3 or tuple(k_cache.shape) != tuple(v_cache.shape) or \
            k_cache.shape[0] != n_kv_heads or k_cache.shape[2] != head_dim:
        raise ValueError("caches must be [nkv, max_len, d]")
    dev = _device(qkv)
    if ctx is None:
        ctx = torch.empty((T, n_q_heads * head_dim), dtype=torch.bfloat16, device=dev)
    st = load().tp_attn_prefill(_ptr(qkv, "qkv", dev), _ptr(k_cache, "k_cache", dev),
                                _ptr(v_cache, "v_cache", dev), T, int(past), k_cache.shape[1],
                                int(n_q_heads), int(n_kv_heads), int(head_dim), int(tp_degree),
                                _ptr(ctx, "ctx", dev), _stream(stream))
    _check(st, "tp_attn_prefill")
    return ctx


def tp_sp_add_rmsnorm(y: torch.Tensor, residual: torch.Tensor, gamma: torch.Tensor,
                      tp_degree: int, eps: float = 1e-5, r_out: Optional[torch.Tensor] = None,
                      n_out: Optional[torch.Tensor] = None,
                      stream: Optional[torch.cuda.Stream] = None):
    """(r, n): r = residual + y, n = RMSNorm(r) * gamma, by token shards of T / t."""
    T, H = y.shape
    if tuple(residual.shape) != (T, H) or tuple(gamma.shape) != (H,):
        raise ValueError("residual must be [T, H] and gamma [H]")
    dev = _device(y)
    if r_out is None:
        r_out = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    if n_out is None:
        n_out = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    st = load().tp_sp_add_rmsnorm(_ptr(y, "y", dev), _ptr(residual, "residual", dev),
                                  _ptr(gamma, "gamma", dev), T, H, int(tp_degree), float(eps),
                                  _ptr(r_out, "r_out", dev), _ptr(n_out, "n_out", dev),
                                  _stream(stream))
    _check(st, "tp_sp_add_rmsnorm")
    return r_out, n_out


def tp_device_error_check() -> int:
    """Synchronise, then read and clear the kernels' device-side error word."""
    return int(load().tp_device_error_check())


def tp_diag_bounded_wait(limit_us: int, result: torch.Tensor,
                         stream: Optional[torch.cuda.Stream] = None) -> None:
    """Diagnostic: a kernel whose bounded waits run out on purpose (result: int32[3]
    on the current device; see include/tp_block.h)."""
    dev = _device(result)
    if result.dtype != torch.int32 or result.numel() < 3 or not result.is_contiguous():
        raise ValueError("result must be a contiguous int32 tensor of at least 3 elements")
    if result.device != dev:
        raise ValueError("result must be on the current device")
    _check(load().tp_diag_bounded_wait(int(limit_us), result.data_ptr(), _stream(stream)),
           "tp_diag_bounded_wait")


def tp_set_decode_max_tokens(max_tokens: int) -> None:
    _check(load().tp_set_decode_max_tokens(int(max_tokens)), "tp_set_decode_max_tokens")


def tp_get_decode_max_tokens() -> int:
    return int(load().tp_get_decode_max_tokens())


def tp_stream_plan(T: int, K: int, N: int, row_shards: int = 1, w8: bool = False,
                   sms: int = B200_SMS, max_smem: int = B200_MAX_SMEM) -> dict:
    """The weight-streaming kernel's launch for one layer (host arithmetic, no GPU
    needed); raises TPError (e.g. TP_ERR_UNSUPPORTED) when it would not stream."""
    plan = StreamPlan()
    st = load().tp_stream_plan(int(T), int(K), int(N), int(row_shards), 1 if w8 else 0,
                               int(sms), int(max_smem), ctypes.addressof(plan))
    _check(st, "tp_stream_plan")
    return {name: getattr(plan, name) for name, _ in StreamPlan._fields_}


def tp_set_launch_options(flags: int) -> None:
    """TP_OPT_PDL | TP_OPT_STATIC_WEIGHTS (see include/tp_block.h)."""
    _check(load().tp_set_launch_options(int(flags)), "tp_set_launch_options")


def tp_get_launch_options() -> int:
    return int(load().tp_get_launch_options())
