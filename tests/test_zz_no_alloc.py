"""The allocation-free MLP call, for callers that cannot allocate device memory
(plugin hosts that pass only inputs and outputs, processes whose device memory
belongs to another allocator, loops that cannot take cudaMalloc's implicit
synchronisation).

tp_mlp_forward_noalloc keeps the activation between the two layers in the
library's own static device array instead of a caller workspace.  It runs the
same kernels with the same launch geometry as tp_mlp_forward (the workspace
entry point), so these tests call both through the C ABI and require the two
results to be bit-identical, on two calls in a row, on both kernel paths (a
stale or misaligned read of the array would shift a few ulps, which a
tolerance would hide); each result is also held to the parity tolerance used
everywhere else against the fp64 oracle.  Sizes past the array must be
refused.  This file is collected last on purpose.
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


def _close(y, ref, what):
    a = y.double().cpu().numpy()
    r = ref.double().cpu().numpy()
    err = a - r
    rel = np.linalg.norm(err) / np.linalg.norm(r)
    mx = np.abs(err).max()
    assert np.isfinite(a).all(), what
    assert rel <= REL_L2 and mx <= MAX_ABS_FRAC * np.abs(r).max(), \
        f"{what}: rel_l2={rel:.3e} max_abs={mx:.3e}"


@pytest.mark.parametrize("T,H,F,t", [(16, 1024, 4096, 4),      # streaming kernels
                                     (64, 512, 32768, 8),      # h exactly fills the array
                                     (300, 768, 2048, 2)])     # tiled kernels
def test_noalloc_matches_workspace_call_twice(T, H, F, t):
    assert torch.cuda.is_available()
    dev = torch.device("cuda", torch.cuda.current_device())
    w1 = workloads.random_bf16_small((F, H), 0.03, 11).to(dev)
    b1 = workloads.random_bf16_small((F,), 0.05, 12).to(dev)
    w2 = workloads.random_bf16_small((H, F), 0.03, 13).to(dev)
    b2 = workloads.random_bf16_small((H,), 0.05, 14).to(dev)
    for call in range(2):  # the second call must not see the first call's h
        x = workloads.random_bf16_small((T, H), 1.0, 100 + call).to(dev)
        ref = tp.tp_mlp_forward(x, w1, b1, w2, b2, t, "gelu_tanh")
        y = tp.tp_mlp_forward_noalloc(x, w1, b1, w2, b2, t, "gelu_tanh")
        torch.cuda.synchronize()
        assert torch.equal(y, ref), f"call {call} T={T} F={F}: not bit-identical"
        if call == 0:
            exact = oracle.mlp_block(x.cpu(), w1.cpu(), b1.cpu(), w2.cpu(), b2.cpu(), t,
                                     "gelu_tanh")
            _close(y, torch.from_numpy(exact), f"call {call} T={T} F={F} vs oracle")
    assert tp.tp_device_error_check() == tp.TP_OK


def test_noalloc_refuses_sizes_beyond_its_array():
    dev = torch.device("cuda", torch.cuda.current_device())
    H, F = 64, 32768
    T = tp.TP_NOALLOC_SCRATCH_BYTES // (2 * F) + 1
    x = torch.zeros((T, H), dtype=torch.bfloat16, device=dev)
    w1 = torch.zeros((F, H), dtype=torch.bfloat16, device=dev)
    w2 = torch.zeros((H, F), dtype=torch.bfloat16, device=dev)
    with pytest.raises(tp.TPError) as e:
        tp.tp_mlp_forward_noalloc(x, w1, None, w2, None, 8, "gelu_tanh")
    assert e.value.status == tp.TP_ERR_WORKSPACE
