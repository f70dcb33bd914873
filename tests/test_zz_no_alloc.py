"""The allocation-free forward (hbl_forward_noalloc) against the caller-workspace
forward (hbl_forward_ws), through the C ABI.

hbl_forward_noalloc serves callers that cannot allocate device memory (a
serving process whose pool already holds nearly all of HBM, code that cannot
afford the synchronisation of cudaMalloc/cudaFree, hosts that forbid plugin
allocations). Its workspace is a fixed device array shared by every call, so
the test runs each case twice in a row: the second call must not see stale
state from the first. This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

import parity
from hadamard_bit_quant_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def H():
    from hadamard_bit_quant_b200 import build, hbl
    build.build()
    assert torch.cuda.is_available()
    hbl.lib()
    return hbl


CASES = [
    # M, K, N, act_bits, use_hadamard
    (16, 4096, 4096, 4, 1),    # decode-shaped o_proj, W1.58A4
    (3, 1024, 256, 8, 0),      # plain BitLinear, INT8
    (100, 4096, 512, 4, 1),    # warp-level GEMM path: split-K partials accumulate in the workspace
]


@pytest.mark.parametrize("M,K,N,a,h", CASES)
def test_noalloc_matches_workspace_forward(H, M, K, N, a, h):
    from hadamard_bit_quant_b200 import layer
    X = inputs.student_t(M, K, 11 + M).cuda()
    Wpk, wsc = layer.pack_weights(inputs.gaussian_weights(N, K, 12 + N).cuda())
    ws = layer.workspace(M, K, N, "cuda")
    ref = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    H.hbl_forward_ws(X, M, K, N, Wpk, wsc, a, h, ref, ws, ws.numel())
    yref = ref.float().cpu().numpy()
    for call in range(2):
        Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        H.hbl_forward_noalloc(X, M, K, N, Wpk, wsc, a, h, Y)
        torch.cuda.synchronize()
        y = Y.float().cpu().numpy()
        assert np.all(np.isfinite(y)), f"call {call}: output not fully written"
        assert np.all(np.abs(y - yref) <= parity.Y_RTOL * np.abs(yref)), f"call {call}"
    assert H.hbl_get_device_error() == 0


def test_noalloc_rejects_sizes_beyond_its_workspace(H):
    from hadamard_bit_quant_b200 import layer
    M, K, N = 4096, 16384, 256          # int8 codes alone need 64 MiB > 8 MiB
    X = torch.zeros(M, K, dtype=torch.bfloat16, device="cuda")
    Wpk, wsc = layer.pack_weights(inputs.gaussian_weights(N, K, 1).cuda())
    Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(H.HblError) as e:
        H.hbl_forward_noalloc(X, M, K, N, Wpk, wsc, 4, 1, Y)
    assert e.value.status == 7
