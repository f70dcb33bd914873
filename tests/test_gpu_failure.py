"""Failure detection without a GPU fault: a bounded device-side wait runs out
(its mbarrier never completes), the kernel records HBL_ERR_TIMEOUT and exits,
the host reads the status, and the context keeps working afterwards."""
import numpy as np
import pytest
import torch

import oracle
import parity
from hadamard_bit_quant_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def H():
    from hadamard_bit_quant_b200 import build, hbl
    build.build()
    hbl.lib()
    return hbl


def test_bounded_wait_times_out_and_reports(H):
    assert H.hbl_get_device_error() == 0                  # clean start
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    H.hbl_selftest_wait_timeout(2000, flag)               # 2 ms limit
    assert H.hbl_get_device_error() == 5                  # HBL_ERR_TIMEOUT
    assert flag.item() == 1
    assert H.hbl_get_device_error() == 0                  # reading clears the word


def test_context_usable_after_timeout(H):
    from hadamard_bit_quant_b200 import layer
    H.hbl_selftest_wait_timeout(1000)
    assert H.hbl_get_device_error() == 5
    case = inputs.tiny_case()
    X, W = case.make_x(), case.make_w()
    Wpk, wsc = layer.pack_weights(W.cuda())
    Y = layer.forward(X.cuda(), Wpk, wsc, case.N, 4, 1)
    a, T = oracle.weight_quant(W.numpy())
    ref = oracle.forward(X.to(torch.float64).numpy(), T, a, 4, 1)
    codes, scales, _ = layer.quantize(X.cuda(), 4, 1)
    diff = parity.check_codes(codes.cpu().numpy(), ref["codes"], ref["tie"], scales.cpu().numpy(), ref["s"])
    parity.check_y(Y.float().cpu().numpy(), ref["Y"], ref["s"], a, diff.sum(1))
    assert H.hbl_get_device_error() == 0


def test_selftest_rejects_bad_limits(H):
    with pytest.raises(H.HblError):
        H.hbl_selftest_wait_timeout(0)
