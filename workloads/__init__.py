"""Seeded synthetic inputs for the tensor-parallel transformer block.

This module is shared by the CPU oracle's tests, the CUDA parity tests and the
benchmark.  It only draws random numbers and rounds them to the storage type
(bf16); it holds none of the block's arithmetic.

Recipe (one place, so every consumer sees the same bits):

* every tensor is drawn from N(0, 1) in fp32 with ``torch.randn`` on the CPU,
  scaled by its standard deviation, then rounded to bf16 (round-to-nearest-even,
  ``Tensor.to(torch.bfloat16)``);
* a tensor is drawn in chunks of ``CHUNK`` elements; chunk ``c`` of tensor
  ``index`` under ``seed`` uses its own ``torch.Generator`` seeded with
  ``((seed * 1000 + index) << 24) + c``, so the values do not depend on how many
  threads draw them;
* weights are stored ``[out_features, in_features]`` row-major (the layer
  computes ``x @ weight.T``, as in the column-linear example of the
  iloveeagents.com page, "Example" section), so the math-orientation shape
  ``W1[H, F]`` is held as a ``[F, H]`` array.

Shapes and standard deviations are the five workloads the block is measured
on; see ``CONFIGS``.

8-bit weights (``quantize_e4m3_rows``): a drawn bf16 weight is stored as FP8
E4M3 codes with one fp32 scale per output row, scale[n] = max_k |w[n, k]| / 448
(448 is the largest finite E4M3 value) and q[n, k] = E4M3(w[n, k] / scale[n]),
rounded to nearest by ``Tensor.to(torch.float8_e4m3fn)``.  The layer then uses
the weight scale[n] * e4m3(q[n, k]); the oracle and the GPU both receive q and
the scales.
"""
from __future__ import annotations

import concurrent.futures as _cf
import dataclasses
import os
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np
import torch

CHUNK = 1 << 24

# tensor indices inside one workload (part of the seed derivation)
IDX_X, IDX_W1, IDX_B1, IDX_W2, IDX_B2 = 0, 1, 2, 3, 4
IDX_QKV_W, IDX_CTX, IDX_O_W, IDX_QKV_B, IDX_O_B = 1, 2, 3, 4, 5


def _chunk_seed(seed: int, index: int, chunk: int) -> int:
    return ((seed * 1000 + index) << 24) + chunk


def normal_bf16(shape: Sequence[int], std: float, seed: int, index: int,
                threads: Optional[int] = None) -> torch.Tensor:
    """Draw a bf16 CPU tensor ~ N(0, std^2) with the chunked recipe above."""
    numel = 1
    for s in shape:
        numel *= int(s)
    out = torch.empty(numel, dtype=torch.bfloat16)
    nchunks = (numel + CHUNK - 1) // CHUNK

    def fill(c: int) -> None:
        lo = c * CHUNK
        hi = min(numel, lo + CHUNK)
        g = torch.Generator().manual_seed(_chunk_seed(seed, index, c))
        v = torch.randn(hi - lo, generator=g, dtype=torch.float32)
        if std != 1.0:
            v.mul_(std)
        out[lo:hi] = v.to(torch.bfloat16)

    if nchunks <= 1:
        for c in range(nchunks):
            fill(c)
    else:
        n = threads or min(nchunks, max(1, (os.cpu_count() or 1)))
        with _cf.ThreadPoolExecutor(max_workers=n) as ex:
            list(ex.map(fill, range(nchunks)))
    return out.view(*[int(s) for s in shape])


def normal_fp32(shape: Sequence[int], std: float, seed: int, index: int) -> torch.Tensor:
    """fp32 draw with the same recipe (no rounding); used for the tiny block's fp32 x."""
    numel = 1
    for s in shape:
        numel *= int(s)
    assert numel <= CHUNK
    g = torch.Generator().manual_seed(_chunk_seed(seed, index, 0))
    v = torch.randn(numel, generator=g, dtype=torch.float32)
    if std != 1.0:
        v.mul_(std)
    return v.view(*[int(s) for s in shape])


@dataclasses.dataclass(frozen=True)
class MLPConfig:
    """A column-parallel -> GeLU -> row-parallel MLP block."""
    name: str
    hidden: int            # H
    ffn: int               # F
    tokens: Tuple[int, ...]  # T values measured
    tp_degrees: Tuple[int, ...]
    act: str               # "gelu_tanh" | "none"
    w_std: float
    b_std: Optional[float]  # None -> the workload has no biases
    x_fp32: bool = False   # x drawn in fp32 and rounded by the caller
    sample_rows: Optional[int] = None  # oracle checks this many seeded rows
    weights: str = "bf16"  # "bf16", or "e4m3": 8-bit weights with row scales


@dataclasses.dataclass(frozen=True)
class ProjConfig:
    """A single column-parallel projection (no second layer)."""
    name: str
    k: int
    n: int
    tokens: Tuple[int, ...]
    tp_degrees: Tuple[int, ...]
    act: str
    w_std: float


@dataclasses.dataclass(frozen=True)
class AttnConfig:
    """QKV projection split by heads + row-parallel output projection."""
    name: str
    hidden: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    tokens: Tuple[int, ...]
    tp_degrees: Tuple[int, ...]
    w_std: float
    sample_rows: Optional[int] = None


@dataclasses.dataclass(frozen=True)
class AttnDecodeConfig:
    """The attention core: new tokens over a per-head KV cache holding `past`
    earlier tokens (decode: a few new tokens over a long cache; prefill: a
    whole prompt, usually with no cache)."""
    name: str
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    past: int               # cached tokens before the new ones
    tokens: Tuple[int, ...]  # new tokens per call, one call per entry
    tp_degrees: Tuple[int, ...]


@dataclasses.dataclass(frozen=True)
class SPNormConfig:
    """The sequence-parallel region after a row-parallel linear: residual add
    and RMSNorm of every token row, by token shards."""
    name: str
    hidden: int
    tokens: Tuple[int, ...]
    tp_degrees: Tuple[int, ...]


CONFIGS: Dict[str, object] = {
    # x[8,256] fp32, W1[256->1024], W2[1024->256] N(0,0.02), biases N(0,0.01), t=2
    "tiny": MLPConfig("tiny", hidden=256, ffn=1024, tokens=(8,), tp_degrees=(2,),
                      act="gelu_tanh", w_std=0.02, b_std=0.01, x_fp32=True),
    # W[4096,4096] split column-wise into 2 shards of 2048 outputs; decode T in {1,8,64}
    "sq4096": ProjConfig("sq4096", k=4096, n=4096, tokens=(1, 8, 64), tp_degrees=(2,),
                         act="none", w_std=0.02),
    # Llama-3-70B-shaped MLP decode
    "mlp70b": MLPConfig("mlp70b", hidden=8192, ffn=28672, tokens=(1, 16, 64),
                        tp_degrees=(4, 8), act="gelu_tanh", w_std=0.02, b_std=None),
    # the backward pass of the 70B-shaped MLP over a 4096-token batch (training)
    "mlp70b_bwd": MLPConfig("mlp70b_bwd", hidden=8192, ffn=28672, tokens=(4096,),
                            tp_degrees=(8,), act="gelu_tanh", w_std=0.02, b_std=None,
                            sample_rows=64),
    # the same MLP with 8-bit (E4M3, per-row scale) weights, decode
    "mlp70b_w8": MLPConfig("mlp70b_w8", hidden=8192, ffn=28672, tokens=(1, 16, 64),
                           tp_degrees=(4, 8), act="gelu_tanh", w_std=0.02, b_std=None,
                           weights="e4m3"),
    # Llama-3-70B-shaped attention projections, prefill
    "attn70b": AttnConfig("attn70b", hidden=8192, n_q_heads=64, n_kv_heads=8,
                          head_dim=128, tokens=(4096,), tp_degrees=(8,), w_std=0.02,
                          sample_rows=64),
    # the attention core between the 70B projections, decode over a 64K-token cache
    "attn70b_decode": AttnDecodeConfig("attn70b_decode", n_q_heads=64, n_kv_heads=8,
                                       head_dim=128, past=65536, tokens=(1, 2, 4),
                                       tp_degrees=(8,)),
    # the attention core between the 70B projections, prefill: a 4096-token
    # prompt, causal over itself (no cached tokens)
    "attn70b_prefill": AttnDecodeConfig("attn70b_prefill", n_q_heads=64, n_kv_heads=8,
                                        head_dim=128, past=0, tokens=(4096,),
                                        tp_degrees=(8,)),
    # the sequence-parallel region of the 405B-shaped block in prefill
    "sp405b": SPNormConfig("sp405b", hidden=16384, tokens=(8192,), tp_degrees=(8,)),
    # 405B-shaped MLP prefill; the oracle checks 64 seeded rows
    "mlp405b": MLPConfig("mlp405b", hidden=16384, ffn=53248, tokens=(8192,),
                         tp_degrees=(8,), act="gelu_tanh", w_std=0.01, b_std=None,
                         sample_rows=64),
}


def x_index(T: int) -> int:
    """Tensor index of the activations for a T-token batch (one draw per T)."""
    return 100 + int(T)


def mlp_inputs(cfg: MLPConfig, T: int, seed: int = 0, with_bias: Optional[bool] = None
               ) -> Dict[str, Optional[torch.Tensor]]:
    """x [T,H], w1 [F,H], b1 [F], w2 [H,F], b2 [H] as bf16 CPU tensors."""
    H, F = cfg.hidden, cfg.ffn
    if cfg.x_fp32:
        x32 = normal_fp32((T, H), 1.0, seed, IDX_X)
        x = x32.to(torch.bfloat16)
    else:
        x32 = None
        x = normal_bf16((T, H), 1.0, seed, x_index(T))
    w1 = normal_bf16((F, H), cfg.w_std, seed, IDX_W1)
    w2 = normal_bf16((H, F), cfg.w_std, seed, IDX_W2)
    use_b = (cfg.b_std is not None) if with_bias is None else with_bias
    b_std = cfg.b_std if cfg.b_std is not None else 0.01
    b1 = normal_bf16((F,), b_std, seed, IDX_B1) if use_b else None
    b2 = normal_bf16((H,), b_std, seed, IDX_B2) if use_b else None
    return {"x": x, "x_fp32": x32, "w1": w1, "b1": b1, "w2": w2, "b2": b2}


def mlp_x(cfg: MLPConfig, T: int, seed: int = 0) -> torch.Tensor:
    """Only the activations of mlp_inputs (same draw), without the weights."""
    if cfg.x_fp32:
        return normal_fp32((T, cfg.hidden), 1.0, seed, IDX_X).to(torch.bfloat16)
    return normal_bf16((T, cfg.hidden), 1.0, seed, x_index(T))


def proj_inputs(cfg: ProjConfig, T: int, seed: int = 0, with_bias: bool = False
                ) -> Dict[str, Optional[torch.Tensor]]:
    """x [T,K], w [N,K] (and an optional b [N]) as bf16 CPU tensors."""
    x = normal_bf16((T, cfg.k), 1.0, seed, x_index(T))
    w = normal_bf16((cfg.n, cfg.k), cfg.w_std, seed, IDX_W1)
    b = normal_bf16((cfg.n,), 0.01, seed, IDX_B1) if with_bias else None
    return {"x": x, "w": w, "b": b}


def attn_inputs(cfg: AttnConfig, T: int, seed: int = 0, with_bias: bool = False
                ) -> Dict[str, Optional[torch.Tensor]]:
    """x [T,H], w_qkv [(nq+2nkv)d, H], ctx [T, nq d], w_o [H, nq d] as bf16."""
    H, d = cfg.hidden, cfg.head_dim
    nqkv = (cfg.n_q_heads + 2 * cfg.n_kv_heads) * d
    nctx = cfg.n_q_heads * d
    x = normal_bf16((T, H), 1.0, seed, x_index(T))
    w_qkv = normal_bf16((nqkv, H), cfg.w_std, seed, IDX_QKV_W)
    ctx = normal_bf16((T, nctx), 1.0, seed, IDX_CTX)
    w_o = normal_bf16((H, nctx), cfg.w_std, seed, IDX_O_W)
    b_qkv = normal_bf16((nqkv,), 0.01, seed, IDX_QKV_B) if with_bias else None
    b_o = normal_bf16((H,), 0.01, seed, IDX_O_B) if with_bias else None
    return {"x": x, "w_qkv": w_qkv, "b_qkv": b_qkv, "ctx": ctx, "w_o": w_o, "b_o": b_o}


def attn_decode_qkv(cfg: AttnDecodeConfig, T: int, seed: int = 0) -> torch.Tensor:
    """qkv [T, (nq + 2 nkv) d] of T new tokens, N(0, 1) bf16 (the projections'
    outputs have no fixed scale; unit variance keeps the scores q.k / sqrt(d)
    of order one)."""
    nqkv = (cfg.n_q_heads + 2 * cfg.n_kv_heads) * cfg.head_dim
    return normal_bf16((T, nqkv), 1.0, seed, 500 + int(T))


def attn_decode_cache(cfg: AttnDecodeConfig, seed: int = 0) -> Tuple[torch.Tensor, torch.Tensor]:
    """The caches k, v [nkv, past, d] of the cached tokens, N(0, 1) bf16."""
    shape = (cfg.n_kv_heads, cfg.past, cfg.head_dim)
    return normal_bf16(shape, 1.0, seed, 601), normal_bf16(shape, 1.0, seed, 602)


def sp_norm_inputs(cfg: SPNormConfig, T: int, seed: int = 0) -> Dict[str, torch.Tensor]:
    """y (the row-parallel output) and the residual [T, H] ~ N(0, 1), and
    gamma [H] ~ 1 + N(0, 0.1^2), bf16."""
    y = normal_bf16((T, cfg.hidden), 1.0, seed, 700 + int(T))
    res = normal_bf16((T, cfg.hidden), 1.0, seed, 800 + int(T))
    gamma = (1.0 + normal_bf16((cfg.hidden,), 0.1, seed, 701).float()).to(torch.bfloat16)
    return {"y": y, "residual": res, "gamma": gamma}


def mlp_dy(cfg: MLPConfig, T: int, seed: int = 0) -> torch.Tensor:
    """The upstream gradient dy [T, H] of the block's output, N(0, 1) bf16."""
    return normal_bf16((T, cfg.hidden), 1.0, seed, 900 + int(T))


def quantize_e4m3_rows(w: torch.Tensor, rows_per_chunk: int = 2048
                       ) -> Tuple[torch.Tensor, torch.Tensor]:
    """8-bit storage of a [N, K] weight (recipe in the module docstring):
    returns (q [N, K] uint8 E4M3 codes, scale [N] float32)."""
    n = int(w.shape[0])
    q = torch.empty(tuple(w.shape), dtype=torch.uint8)
    scale = torch.empty(n, dtype=torch.float32)
    for r0 in range(0, n, rows_per_chunk):
        r1 = min(n, r0 + rows_per_chunk)
        wf = w[r0:r1].to(torch.float32)
        amax = wf.abs().amax(dim=1)
        sc = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
        q[r0:r1] = (wf / sc[:, None]).to(torch.float8_e4m3fn).view(torch.uint8)
        scale[r0:r1] = sc
    return q, scale


def sample_rows(T: int, count: int, seed: int = 0) -> List[int]:
    """Seeded, sorted, distinct row indices for checks on a row sample."""
    rng = np.random.default_rng(seed)
    return sorted(int(i) for i in rng.choice(T, size=min(count, T), replace=False))


def random_bf16_small(shape: Sequence[int], std: float, seed: int) -> torch.Tensor:
    """Small bf16 tensor for unit tests (one generator, no chunking)."""
    g = torch.Generator().manual_seed(int(seed))
    return (torch.randn(*shape, generator=g) * std).to(torch.bfloat16)
