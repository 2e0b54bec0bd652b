"""fp64 CPU oracle of the head-sharded attention core with a per-shard KV cache.

TEST INFRASTRUCTURE ONLY, under the same rules as ``tp_oracle``: only the tests,
the package's ``smoke()`` entry and the benchmark's CPU-baseline / reference leg
may import it; no CUDA code imports or links it.

Where it sits: between the QKV projection (``tp_oracle.attn_qkv``, columns
[Q heads | K heads | V heads]) and the output projection (``tp_oracle.attn_out``,
which reads ctx as [T, nq * d], query-head-major).

Sources: attention heads are distributed among the tensor-parallel GPUs, so each
holds a slice of the layer and its share of the KV cache (xingyuzhitong.com
"Tensor vs Pipeline Parallelism", section "Tensor parallelism: split inside
each layer", and its list of consequences); each GPU holds 1/N of the KV cache
(drpranayjha.com "AI Infrastructure series, Part 5", section "How does tensor
parallelism split a layer?"); the head counts must divide by the degree, and
grouped-query models with eight key-value heads cap it near eight without
replicating cache (xingyuzhitong.com, section "What the serving engines
expose").

The pages give no formula for attention itself.  Readings (plainest standard
ones): scaled dot-product attention, scores q.k / sqrt(d), softmax over keys,
causal (a token sees the cache and the tokens up to itself); grouped-query
attention with query head h reading key-value head h // (nq / nkv) (contiguous
groups); no positional rotation (the pages name none; a rotary embedding would
act on q and k before this step and does not change how the heads shard).

Computation, per shard s (query heads [s nq/t, (s+1) nq/t), key-value heads
[s nkv/t, (s+1) nkv/t)) and per query head h of that shard, g = h // (nq/nkv):
  K_all = [cache_K[g]; new K of head g],  V_all likewise   ([P + T, d])
  for new token i (position P + i): s_j = q_i . K_all[j] / sqrt(d) for
  j <= P + i; p = softmax(s) (shifted by its maximum); ctx_i = sum_j p_j V_all[j].
The shard returns its ctx columns and its grown cache; no exchange is needed
(every query head's key-value head lives on the same shard when t divides both
head counts).

Pinned by tests/test_oracle_attention.py against pure-Python brute force
(``math.exp``, ``math.fsum``), torch's scaled_dot_product_attention in float64,
special cases (one key, equal scores), chunked prefill through the cache equal
to one-shot prefill, independence from t, and planted mistakes.
"""
from __future__ import annotations

import math
from typing import List, Optional, Sequence, Tuple

import numpy as np

from .tp_oracle import ArrayLike, heads_divisible, to_f64


def _split_qkv(qkv: np.ndarray, nq: int, nkv: int, d: int):
    """[T, (nq + 2 nkv) d] -> q [nq, T, d], k [nkv, T, d], v [nkv, T, d]."""
    T = qkv.shape[0]
    if qkv.shape[1] != (nq + 2 * nkv) * d:
        raise ValueError("qkv columns must be (nq + 2 nkv) * head_dim")
    q = qkv[:, : nq * d].reshape(T, nq, d).transpose(1, 0, 2)
    k = qkv[:, nq * d: (nq + nkv) * d].reshape(T, nkv, d).transpose(1, 0, 2)
    v = qkv[:, (nq + nkv) * d:].reshape(T, nkv, d).transpose(1, 0, 2)
    return q, k, v


def attend_head(q: np.ndarray, k_all: np.ndarray, v_all: np.ndarray, past: int) -> np.ndarray:
    """Causal scaled dot-product attention of one head: q [T, d] at positions
    past .. past + T - 1 over k_all, v_all [past + T, d]; returns [T, d]."""
    T, d = q.shape
    out = np.empty((T, d))
    for i in range(T):
        n = past + i + 1                      # keys this token may see
        s = (k_all[:n] @ q[i]) / math.sqrt(d)
        p = np.exp(s - s.max())
        p = p / p.sum()
        out[i] = p @ v_all[:n]
    return out


def empty_cache(t: int, n_kv_heads: int, head_dim: int) -> List[Tuple[np.ndarray, np.ndarray]]:
    """Per-shard KV caches with no tokens: shard s holds [nkv/t, 0, d] for K and V."""
    kh = n_kv_heads // t
    return [(np.zeros((kh, 0, head_dim)), np.zeros((kh, 0, head_dim))) for _ in range(t)]


def attn_core(qkv: ArrayLike, n_q_heads: int, n_kv_heads: int, head_dim: int, t: int,
              cache: Optional[Sequence[Tuple[ArrayLike, ArrayLike]]] = None
              ) -> Tuple[np.ndarray, List[Tuple[np.ndarray, np.ndarray]]]:
    """ctx [T, nq * d] for new tokens qkv [T, (nq + 2 nkv) d], shard by shard.

    ``cache``: per shard s a pair (K, V), each [nkv/t, P, d] -- the keys and
    values of the P earlier tokens of this shard's key-value heads (None: no
    earlier tokens).  Returns ctx and the per-shard caches grown by the T new
    tokens.
    """
    if not heads_divisible(n_q_heads, n_kv_heads, t):
        raise ValueError("tp degree must divide both head counts")
    nq, nkv, d = n_q_heads, n_kv_heads, head_dim
    qkvf = to_f64(qkv)
    T = qkvf.shape[0]
    q, k, v = _split_qkv(qkvf, nq, nkv, d)
    if cache is None:
        cache = empty_cache(t, nkv, d)
    if len(cache) != t:
        raise ValueError("one (K, V) cache per shard")
    group = nq // nkv
    qh, kh = nq // t, nkv // t
    ctx = np.empty((T, nq * d))
    grown = []
    for s in range(t):
        ck, cv = to_f64(cache[s][0]), to_f64(cache[s][1])
        if ck.shape[0] != kh or cv.shape != ck.shape or ck.shape[2] != d:
            raise ValueError(f"shard {s} cache must be [{kh}, P, {d}] for K and V")
        past = ck.shape[1]
        k_s = np.concatenate([ck, k[s * kh:(s + 1) * kh]], axis=1)
        v_s = np.concatenate([cv, v[s * kh:(s + 1) * kh]], axis=1)
        for h in range(s * qh, (s + 1) * qh):
            g = h // group - s * kh           # key-value head, local to the shard
            ctx[:, h * d:(h + 1) * d] = attend_head(q[h], k_s[g], v_s[g], past)
        grown.append((k_s, v_s))
    return ctx, grown
