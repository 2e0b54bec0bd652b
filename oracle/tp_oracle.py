"""fp64 CPU oracle for the tensor-parallel transformer block.

TEST INFRASTRUCTURE ONLY.  Only the tests, the package's ``smoke()`` entry and
the benchmark's CPU-baseline / reference leg may import this module.  The CUDA
path neither imports nor links it, and it imports nothing from the CUDA path;
the two share only the seeded input generator in ``workloads``.

What it computes is the plain definition, in float64, with no blocking of any
reduction, fusion or reordering beyond what the method itself states:

* a column-parallel linear layer: the weight's output features are cut into
  ``t`` contiguous shards; each shard computes ``x @ W_s.T`` on its slice of the
  outputs, and the slices side by side are the layer output (iloveeagents.com,
  "Detail" TP=2 diagram and "Example" ``TensorParallelColumnLinear``;
  xingyuzhitong.com, "Tensor parallelism: split inside each layer");
* a row-parallel linear layer: the second weight is cut along its input
  features; each shard yields a full-size partial from its slice of the
  activations, and the partials are summed (the all-reduce) -- same passages,
  plus drpranayjha.com "How does tensor parallelism split a layer?" and the
  aidolsgroup.com glossary "Full definition";
* the MLP block: column-parallel first linear, elementwise GeLU, row-parallel
  second linear; the attention block's projections: QKV split by heads
  (column-parallel) and the output projection split by head groups
  (row-parallel) (xingyuzhitong.com, "Tensor parallelism"; drpranayjha.com,
  "How does tensor parallelism split a layer?").

Readings where the pages are silent (the pages name no activation, bias or
precision): GeLU is the tanh form 0.5 z (1 + tanh(sqrt(2/pi) (z + 0.044715
z^3))); biases are optional and added once -- to each output feature in the
column-parallel layer, and once after the shard sum in the row-parallel layer;
inputs are the exact bf16 values the GPU receives, upcast to float64; the
intermediate activation h is NOT rounded to bf16 here.  Row-parallel partials
are each started from zero and summed in ascending shard order (the pages only
say splitting changes the order of sums, drpranayjha.com "Short answers":
"Does splitting a model change its answers?").

Memory: large weights are upcast to float64 a block of *output features* at a
time.  That only bounds memory; every output element is still one dot product
over its full reduction dimension.

8-bit weights (drpranayjha.com "AI Infrastructure series, Part 5", "Reason 2":
decode reads 8-bit weights): an ``E4M3Weight`` holds FP8 E4M3 codes and one
scale per output row, W[n, k] = scale[n] * e4m3(q[n, k]); every function here
that takes a weight also takes one, and reads it through its exact float64
values (the E4M3 code table is written out from the format's definition in
``e4m3_value``).

Pinned by tests/test_oracle.py against: brute-force math.fsum dot products on
tiny inputs, torch's own tanh-GeLU in float64 and the erf GeLU (a different
formula that the tanh form approximates), the odd-part identity of GeLU, the
shard-sum and shard-concatenation invariants for every t, special cases
(identity weights, one-hot inputs, t = 1), and, for 8-bit weights, the E4M3
format's landmark values and torch's own float8_e4m3fn decoding.
"""
from __future__ import annotations

import math
from typing import List, Optional, Sequence, Tuple, Union

import numpy as np

try:  # the oracle accepts torch CPU tensors (bf16) as well as numpy arrays
    import torch
except Exception:  # pragma: no cover - torch is always present in this repo
    torch = None

ArrayLike = Union[np.ndarray, "torch.Tensor"]

SQRT_2_OVER_PI = math.sqrt(2.0 / math.pi)
GELU_CUBIC = 0.044715

# output features upcast per block (memory bound only; see module docstring)
_OUT_BLOCK = 2048


def e4m3_value(code: int) -> float:
    """The value of one FP8 E4M3 code ("E4M3FN"): 1 sign bit, 4 exponent bits
    with bias 7, 3 mantissa bits; exponent field 0 is subnormal (m/8 * 2^-6);
    there are no infinities and S.1111.111 is NaN."""
    sign = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return math.nan
    if e == 0:
        return sign * (m / 8.0) * 2.0 ** -6
    return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)


E4M3_TABLE = np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)


class E4M3Weight:
    """An 8-bit weight [N, K]: codes q (uint8) and row scales (float32),
    W[n, k] = scale[n] * e4m3(q[n, k]).  Slicing by rows, or by rows and
    columns, gives the matching sub-weight; ``to_f64`` decodes it exactly."""

    def __init__(self, q: ArrayLike, scale: ArrayLike):
        self.q = q
        self.scale = scale
        self.shape = tuple(int(d) for d in q.shape)

    def __getitem__(self, idx):
        rows = idx[0] if isinstance(idx, tuple) else idx
        return E4M3Weight(self.q[idx], self.scale[rows])

    def dequant(self) -> np.ndarray:
        if torch is not None and isinstance(self.q, torch.Tensor):
            codes = self.q.detach().to("cpu").numpy()
        else:
            codes = np.asarray(self.q)
        sc = to_f64(self.scale)
        return E4M3_TABLE[codes.astype(np.int64)] * sc[:, None]


def to_f64(a: ArrayLike) -> np.ndarray:
    """Exact upcast of a bf16/fp32/fp64 tensor or array (or an 8-bit weight)
    to a float64 ndarray."""
    if isinstance(a, E4M3Weight):
        return a.dequant()
    if torch is not None and isinstance(a, torch.Tensor):
        return a.detach().to("cpu").to(torch.float64).numpy()
    return np.asarray(a, dtype=np.float64)


def gelu_tanh(z: np.ndarray) -> np.ndarray:
    """tanh-form GeLU, elementwise, in float64 (reading stated in the module docstring)."""
    z = np.asarray(z, dtype=np.float64)
    return 0.5 * z * (1.0 + np.tanh(SQRT_2_OVER_PI * (z + GELU_CUBIC * z * z * z)))


def apply_act(z: np.ndarray, act: str) -> np.ndarray:
    if act == "gelu_tanh":
        return gelu_tanh(z)
    if act == "none":
        return z
    raise ValueError(f"unknown activation {act!r}")


def linear(x: ArrayLike, w: ArrayLike, b: Optional[ArrayLike] = None) -> np.ndarray:
    """y[r, j] = sum_k x[r, k] * w[j, k] + b[j]; w is stored [out, in].

    The layer of the iloveeagents.com "Example" computes ``x @ weight.T`` with
    ``weight`` shaped (out_features, in_features); this is that product in
    float64, one full-length dot product per output element.
    """
    xf = to_f64(x)
    n_out = int(w.shape[0])
    if xf.ndim != 2 or int(w.shape[1]) != xf.shape[1]:
        raise ValueError(f"shape mismatch x{tuple(xf.shape)} w{tuple(w.shape)}")
    y = np.empty((xf.shape[0], n_out), dtype=np.float64)
    for j0 in range(0, n_out, _OUT_BLOCK):
        j1 = min(n_out, j0 + _OUT_BLOCK)
        wf = to_f64(w[j0:j1])
        y[:, j0:j1] = xf @ wf.T
    if b is not None:
        y += to_f64(b)[None, :]
    return y


def shard_ranges(n: int, t: int) -> List[Tuple[int, int]]:
    """The t contiguous, equal shards [s n/t, (s+1) n/t) of a dimension of size n.

    iloveeagents.com "Example": ``tp_out_features = out_features // tp_world_size``;
    an uneven split is rejected rather than truncated.
    """
    if t < 1 or n % t != 0:
        raise ValueError(f"tp degree {t} does not divide {n}")
    step = n // t
    return [(s * step, (s + 1) * step) for s in range(t)]


def colpar_linear(x: ArrayLike, w: ArrayLike, b: Optional[ArrayLike], t: int,
                  act: str = "none") -> np.ndarray:
    """Column-parallel linear: shard s owns output features [s N/t, (s+1) N/t).

    Each shard computes act(x @ W_s.T + b_s) on its own slice with no exchange;
    the slices side by side are the output (iloveeagents.com "Detail" and
    "Example"; xingyuzhitong.com "Tensor parallelism").  The activation is
    elementwise, so it is applied per shard before any exchange.
    """
    n = int(w.shape[0])
    parts = []
    for (j0, j1) in shard_ranges(n, t):
        z = linear(x, w[j0:j1], None if b is None else b[j0:j1])
        parts.append(apply_act(z, act))
    return np.concatenate(parts, axis=1)


def rowpar_partials(h: ArrayLike, w: ArrayLike, t: int) -> List[np.ndarray]:
    """Row-parallel shard partials P_s = h[:, K_s] @ W[:, K_s].T, each from zero.

    The second matrix is split by rows of the math-orientation weight, i.e. by
    its input features (xingyuzhitong.com "Tensor parallelism"; drpranayjha.com
    "How does tensor parallelism split a layer?"); every shard produces a
    full-size [T, N] partial.
    """
    hf = to_f64(h)
    k = int(w.shape[1])
    if hf.shape[1] != k:
        raise ValueError(f"shape mismatch h{tuple(hf.shape)} w{tuple(w.shape)}")
    out = []
    for (k0, k1) in shard_ranges(k, t):
        out.append(linear(hf[:, k0:k1], w[:, k0:k1], None))
    return out


def shard_sum(partials: Sequence[np.ndarray], b: Optional[ArrayLike]) -> np.ndarray:
    """The all-reduce: ((P_0 + P_1) + ...) + P_{t-1}, then the bias once.

    The partial outputs are summed (aidolsgroup.com "Full definition";
    xingyuzhitong.com "Tensor parallelism": the partial results are combined by
    an all-reduce).
    """
    y = np.zeros_like(partials[0])
    for p in partials:
        y = y + p
    if b is not None:
        y = y + to_f64(b)[None, :]
    return y


def rowpar_linear(h: ArrayLike, w: ArrayLike, b: Optional[ArrayLike], t: int) -> np.ndarray:
    """Row-parallel linear followed by the sum of its t partials."""
    return shard_sum(rowpar_partials(h, w, t), b)


def mlp_block(x: ArrayLike, w1: ArrayLike, b1: Optional[ArrayLike], w2: ArrayLike,
              b2: Optional[ArrayLike], t: int, act: str = "gelu_tanh") -> np.ndarray:
    """y = sum_s act(x W1_s^T + b1_s) W2[:, s]^T + b2: the tensor-parallel MLP block.

    xingyuzhitong.com "Tensor parallelism": the first linear layer of the
    feed-forward block is split by columns and the second by rows;
    drpranayjha.com "How does tensor parallelism split a layer?".  Column shard
    s of W1 feeds exactly row shard s of W2, so the activation needs no exchange.
    """
    h = colpar_linear(x, w1, b1, t, act)
    return rowpar_linear(h, w2, b2, t)


def heads_divisible(n_q_heads: int, n_kv_heads: int, t: int) -> bool:
    """t must divide the query and key-value head counts.

    xingyuzhitong.com "Tensor parallelism" (the degree is limited by the number
    of attention heads or key-value heads, which must divide evenly) and
    "What the serving engines expose"; drpranayjha.com "How does tensor
    parallelism split a layer?" (64 query heads: groups of 2, 4 or 8 work, 3 or
    6 do not).  Replicating key-value heads past their count is not modelled.
    """
    return t >= 1 and n_q_heads % t == 0 and n_kv_heads % t == 0


def qkv_shard_columns(n_q_heads: int, n_kv_heads: int, head_dim: int, t: int,
                      s: int) -> np.ndarray:
    """Output columns of the fused [Q | K | V] projection owned by head shard s.

    Shard s holds query heads [s nq/t, (s+1) nq/t) and key-value heads
    [s nkv/t, (s+1) nkv/t) of both K and V (heads distributed among GPUs,
    xingyuzhitong.com "Tensor parallelism").  Layout: columns are Q heads, then K
    heads, then V heads, each head ``head_dim`` wide.
    """
    if not heads_divisible(n_q_heads, n_kv_heads, t):
        raise ValueError("tp degree must divide both head counts")
    d = head_dim
    qh, kh = n_q_heads // t, n_kv_heads // t
    q0 = s * qh * d
    k0 = n_q_heads * d + s * kh * d
    v0 = (n_q_heads + n_kv_heads) * d + s * kh * d
    return np.concatenate([np.arange(q0, q0 + qh * d), np.arange(k0, k0 + kh * d),
                           np.arange(v0, v0 + kh * d)])


def attn_qkv(x: ArrayLike, w_qkv: ArrayLike, b_qkv: Optional[ArrayLike], n_q_heads: int,
             n_kv_heads: int, head_dim: int, t: int) -> np.ndarray:
    """qkv = x W_qkv^T (+ b), computed shard by shard (heads split over t) and
    returned in the unsharded [Q | K | V] column order."""
    n = int(w_qkv.shape[0])
    if n != (n_q_heads + 2 * n_kv_heads) * head_dim:
        raise ValueError("w_qkv rows must be (nq + 2 nkv) * head_dim")
    xf = to_f64(x)
    out = np.empty((xf.shape[0], n), dtype=np.float64)
    for s in range(t):
        cols = qkv_shard_columns(n_q_heads, n_kv_heads, head_dim, t, s)
        b_s = None if b_qkv is None else _take_rows(b_qkv, cols)
        out[:, cols] = linear(xf, _take_rows(w_qkv, cols), b_s)
    return out


def _take_rows(a: ArrayLike, idx: np.ndarray):
    """Rows ``idx`` of a numpy array or torch tensor (a gather, no arithmetic)."""
    if torch is not None and isinstance(a, torch.Tensor):
        return a[torch.as_tensor(idx, dtype=torch.long)]
    return np.asarray(a)[idx]


def attn_out(ctx: ArrayLike, w_o: ArrayLike, b_o: Optional[ArrayLike], n_q_heads: int,
             head_dim: int, t: int) -> np.ndarray:
    """y = b_o + sum_s ctx[:, heads of s] W_o[:, heads of s]^T: the output
    projection split by rows (head groups of nq/t heads), partials summed."""
    if int(w_o.shape[1]) != n_q_heads * head_dim:
        raise ValueError("w_o columns must be nq * head_dim")
    if n_q_heads % t != 0:
        raise ValueError("tp degree must divide the query head count")
    return rowpar_linear(ctx, w_o, b_o, t)
