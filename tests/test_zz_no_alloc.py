"""The allocation-free forward (hbl_forward_noalloc) against the caller-workspace
forward (hbl_forward_ws), through the C ABI.

hbl_forward_noalloc serves callers that cannot allocate device memory (a
serving process whose pool already holds nearly all of HBM, code that cannot
afford the synchronisation of cudaMalloc/cudaFree, hosts that forbid plugin
allocations). Its workspace is a fixed device array shared by every call, so
the test runs each case twice in a row: the second call must not see stale
state from the first. Both entry points run the same kernels on the same
inputs, so their outputs must be identical bit for bit. This file is
collected last on purpose.
"""
import pytest
import torch

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
    # M, K, N, act_bits, use_hadamard, GEMM path (0 = by size, 1 = warp-level split-K)
    (16, 4096, 4096, 4, 1, 0),     # decode-shaped o_proj, W1.58A4 (fused kernel: token rows exchanged through the workspace)
    (3, 1024, 256, 8, 0, 0),       # plain BitLinear, INT8
    (100, 4096, 512, 4, 1, 1),     # split-K: codes, scales and int32 partials all live in the workspace
    (200, 2048, 1024, 8, 1, 2),    # persistent tcgen05 GEMM reading codes from the workspace
]


def _kernels_of(H, fn):
    """Names of the library kernels one call launches (the library's own launch profile)."""
    H.hbl_profile_enable(1)
    fn()
    torch.cuda.synchronize()
    names = set(H.profile_table())
    H.hbl_profile_enable(0)
    return names


@pytest.mark.parametrize("M,K,N,a,h,path", CASES)
def test_noalloc_matches_workspace_forward(H, M, K, N, a, h, path):
    from hadamard_bit_quant_b200 import layer
    X = inputs.student_t(M, K, 11 + M).cuda()
    Wpk, wsc = layer.pack_weights(inputs.gaussian_weights(N, K, 12 + N).cuda())
    ws = layer.workspace(M, K, N, "cuda")
    ref = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    H.hbl_set_gemm_path(path)
    try:
        H.hbl_forward_ws(X, M, K, N, Wpk, wsc, a, h, ref, ws, ws.numel())
        # dirty the shared array with another size first, so stale contents would show
        Xo = inputs.student_t(37, 1024, 5).cuda()
        Wo, ao = layer.pack_weights(inputs.gaussian_weights(64, 1024, 6).cuda())
        H.hbl_forward_noalloc(Xo, 37, 1024, 64, Wo, ao, 4, 1,
                              torch.empty(37, 64, dtype=torch.bfloat16, device="cuda"))
        for call in range(2):
            Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
            names = _kernels_of(H, lambda: H.hbl_forward_noalloc(X, M, K, N, Wpk, wsc, a, h, Y))
            if path == 1:
                # the path that zeroes and accumulates into the shared array really ran
                assert {"memset_acc", "gemm_mma"} <= names, names
            assert torch.equal(Y, ref), f"call {call}: differs from hbl_forward_ws"
    finally:
        H.hbl_set_gemm_path(0)
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
