"""The bounded-wait timeout path on the GPU, without a fault or a hang.

Every wait in the library's kernels is bounded: past its limit it records an
error in the device-side error word, raises its CTA's abort flag and returns,
and tp_device_error_check() reports TP_ERR_DEVICE_TIMEOUT once, then clears
the word.  tp_diag_bounded_wait launches one CTA whose two roles wait on
barriers nothing arrives on (a flag that nothing sets): the first with a 1 ms
limit, the second with the normal one-second limit but the shared abort flag.
"""
import pytest
import torch

import tensor_transformer_linear_column_b200 as tp

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_reports_and_clears():
    dev = torch.device("cuda", torch.cuda.current_device())
    assert tp.tp_device_error_check() == tp.TP_OK  # nothing pending
    res = torch.full((4,), -1, dtype=torch.int32, device=dev)
    tp.tp_diag_bounded_wait(1000, res)
    assert tp.tp_device_error_check() == tp.TP_ERR_DEVICE_TIMEOUT
    assert tp.tp_device_error_check() == tp.TP_OK  # the word was cleared
    r = res.cpu().tolist()
    assert r[0] == 0 and r[1] == 0, r  # both waits gave up
    # the second role left through the shared abort flag, long before its own
    # one-second limit (it waited about as long as the first one's 1 ms)
    assert 0 < r[2] < 100_000_000, r


def test_kernels_still_work_after_a_timeout():
    # the context stays usable: a block call after the diagnostic is correct
    dev = torch.device("cuda", torch.cuda.current_device())
    res = torch.zeros((4,), dtype=torch.int32, device=dev)
    tp.tp_diag_bounded_wait(200, res)
    assert tp.tp_device_error_check() == tp.TP_ERR_DEVICE_TIMEOUT
    g = torch.Generator().manual_seed(5)
    x = (torch.randn(16, 512, generator=g)).to(torch.bfloat16).to(dev)
    w = (torch.randn(1024, 512, generator=g) * 0.05).to(torch.bfloat16).to(dev)
    y = tp.tp_colpar_gemm_gelu(x, w, None, 2, "none")
    torch.cuda.synchronize()
    ref = x.double() @ w.double().T
    err = (y.double() - ref).norm() / ref.norm()
    assert err.item() < 1e-2
    assert tp.tp_device_error_check() == tp.TP_OK


def test_diag_rejects_bad_arguments():
    dev = torch.device("cuda", torch.cuda.current_device())
    res = torch.zeros((4,), dtype=torch.int32, device=dev)
    lib = tp.load()
    assert lib.tp_diag_bounded_wait(0, res.data_ptr(), None) == tp.TP_ERR_UNSUPPORTED
    assert lib.tp_diag_bounded_wait(2_000_000, res.data_ptr(), None) == tp.TP_ERR_UNSUPPORTED
    assert lib.tp_diag_bounded_wait(1000, None, None) == tp.TP_ERR_NULL
    assert lib.tp_diag_bounded_wait(1000, res.data_ptr() + 4, None) == tp.TP_ERR_ALIGN
