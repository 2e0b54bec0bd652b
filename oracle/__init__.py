"""fp64 CPU oracle of the tensor-parallel block -- test infrastructure only.

Importable only from the tests, ``__graft_entry__.smoke()`` and the benchmark's
CPU-baseline / reference leg.  The CUDA product path never touches it.
"""
from .tp_oracle import (  # noqa: F401
    E4M3_TABLE,
    E4M3Weight,
    apply_act,
    attn_out,
    attn_qkv,
    colpar_linear,
    e4m3_value,
    gelu_tanh,
    heads_divisible,
    linear,
    mlp_block,
    qkv_shard_columns,
    rowpar_linear,
    rowpar_partials,
    shard_ranges,
    shard_sum,
    to_f64,
)
from .tp_attention import attend_head, attn_core, empty_cache  # noqa: F401
from .tp_backward import act_grad, gelu_tanh_grad, mlp_block_backward  # noqa: F401
from .tp_sequence import (  # noqa: F401
    RMS_EPS,
    all_gather,
    reduce_scatter,
    rms_norm,
    sp_residual_norm,
    token_shards,
)
