"""fp64 CPU oracle of sequence parallelism inside the tensor-parallel group.

TEST INFRASTRUCTURE ONLY, under the same rules as ``tp_oracle``: only the tests,
the package's ``smoke()`` entry and the benchmark's CPU-baseline / reference leg
may import it; no CUDA code imports or links it.

Source: drpranayjha.com "AI Infrastructure series, Part 5", section "What about
MoE models and very long prompts?": sequence parallelism, a Megatron-LM feature
related to context parallelism, splits the parts of a layer that tensor
parallelism leaves whole -- normalisation and dropout -- along the sequence,
inside the same tensor-parallel group, to save activation memory.

Readings (the pages give no formulas for this step):

* where it sits: between the row-parallel linear of one sublayer and the
  column-parallel linear of the next.  The all-reduce of the row-parallel
  partials is taken as its two halves: a reduce-scatter that leaves shard s
  the summed rows of its tokens [s T/t, (s+1) T/t), and an all-gather of the
  normalised rows before the next column-parallel linear, which needs every
  token.  T must divide by t, like every other split here.
* what the whole-layer part computes per token: the residual connection and
  the normalisation of a pre-norm Llama-shaped block, r = x + y (the new
  residual stream) and n = RMSNorm(r) = r / sqrt(mean_j r_j^2 + eps) * gamma;
  RMSNorm is the normalisation of the Llama-shaped models the workloads use;
  eps = 1e-5.  Dropout is the identity at inference and is not modelled.
* order: the reduce-scatter sums the shard partials in ascending shard order,
  each from zero, then adds the bias once, exactly like the forward all-reduce
  (``tp_oracle.shard_sum``), restricted to the shard's rows.

Pinned by tests/test_oracle_sequence.py against: the all-reduce it replaces
(reduce-scatter then all-gather gives ``shard_sum`` exactly), torch's own
``rms_norm`` in float64, ``math.fsum`` brute force on a tiny case, the
closed-form invariants of RMSNorm (unit root-mean-square output for gamma = 1
and eps = 0; invariance to positive scaling of a row), independence from t,
and planted mistakes.
"""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

import numpy as np

from .tp_oracle import ArrayLike, shard_ranges, to_f64

RMS_EPS = 1e-5


def rms_norm(r: ArrayLike, gamma: ArrayLike, eps: float = RMS_EPS) -> np.ndarray:
    """n[i, j] = r[i, j] / sqrt(mean_j r[i, j]^2 + eps) * gamma[j], row by row."""
    rf = to_f64(r)
    g = to_f64(gamma)
    ms = (rf * rf).mean(axis=1, keepdims=True)
    return rf / np.sqrt(ms + eps) * g[None, :]


def token_shards(T: int, t: int) -> List[Tuple[int, int]]:
    """The t contiguous, equal token ranges [s T/t, (s+1) T/t) of a sequence."""
    return shard_ranges(T, t)


def reduce_scatter(partials: Sequence[np.ndarray], b: Optional[ArrayLike], t: int
                   ) -> List[np.ndarray]:
    """Shard s's rows of ((P_0 + P_1) + ...) + P_{t-1} + b: the first half of
    the all-reduce, leaving each shard only its own tokens."""
    T = partials[0].shape[0]
    bias = None if b is None else to_f64(b)
    out = []
    for (r0, r1) in token_shards(T, t):
        y = np.zeros_like(partials[0][r0:r1])
        for p in partials:
            y = y + p[r0:r1]
        if bias is not None:
            y = y + bias[None, :]
        out.append(y)
    return out


def all_gather(pieces: Sequence[np.ndarray]) -> np.ndarray:
    """The second half: every shard's rows, in token order."""
    return np.concatenate(list(pieces), axis=0)


def sp_residual_norm(partials: Sequence[np.ndarray], b: Optional[ArrayLike],
                     residual: ArrayLike, gamma: ArrayLike, t: int, eps: float = RMS_EPS
                     ) -> Tuple[np.ndarray, np.ndarray]:
    """The sequence-parallel region after a row-parallel linear.

    Shard s receives its tokens' summed rows (reduce-scatter), adds its slice of
    the residual stream and normalises those rows alone; the all-gather then
    returns (r, n) for the whole sequence: r = residual + y, n = RMSNorm(r).
    """
    res = to_f64(residual)
    T = res.shape[0]
    ys = reduce_scatter(partials, b, t)
    rs, ns = [], []
    for (r0, r1), y in zip(token_shards(T, t), ys):
        r = res[r0:r1] + y
        rs.append(r)
        ns.append(rms_norm(r, gamma, eps))
    return all_gather(rs), all_gather(ns)
