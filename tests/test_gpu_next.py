"""Parity of the next rows' CUDA paths with the oracle: the RMSNorm prologue of
Eq. 9, the rotated-weight variant (Table 5 ablation), the Hadamard backward
(Eq. 10) and the post-RoPE QKV quantiser."""
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
    assert torch.cuda.is_available()
    hbl.lib()
    return hbl


def _gain(K, seed):
    g = torch.Generator().manual_seed(seed)
    return (0.5 + torch.rand(K, generator=g)).float()


# ----------------------------------------------------------------------------- f1: LN prologue
@pytest.mark.parametrize("M,K,a,h,use_gain", [(8, 256, 4, 1, True), (16, 4096, 4, 1, True), (130, 4096, 8, 1, False),
                                              (3, 16384, 4, 1, True), (33, 768, 8, 0, True), (5, 4096, 4, 0, False)])
def test_quantize_ln(H, M, K, a, h, use_gain):
    X = inputs.gaussian_with_outliers(M, K, K + 5, inputs.outlier_channels(K, 0.01, 2).tolist(), 50.0)
    g = _gain(K, 1) if use_gain else None
    codes = torch.empty(M, K, dtype=torch.int8, device="cuda")
    scales = torch.empty(M, dtype=torch.float32, device="cuda")
    csum = torch.empty(M, dtype=torch.int32, device="cuda")
    H.hbl_quantize_ln(X.cuda(), M, K, g.cuda() if g is not None else None, a, h, codes, scales, csum)
    xn = oracle.rmsnorm(X.to(torch.float64).numpy(), None if g is None else g.numpy())
    xr = oracle.hadamard(xn) if h else xn
    c_ref, s_ref, tie = oracle.quantize_act(xr, a)
    c = codes.cpu().numpy()
    parity.check_codes(c, c_ref, tie, scales.cpu().numpy(), s_ref)
    assert np.array_equal(csum.cpu().numpy(), c.astype(np.int64).sum(1))


@pytest.mark.parametrize("M,K,N,a,h", [(16, 4096, 4096, 4, 1), (300, 2048, 256, 4, 1), (7, 1024, 144, 8, 0)])
def test_forward_ln(H, M, K, N, a, h):
    from hadamard_bit_quant_b200 import layer
    X = inputs.gaussian_with_outliers(M, K, 3, inputs.outlier_channels(K, 0.01, 3).tolist(), 50.0)
    W = inputs.gaussian_weights(N, K, 4)
    g = _gain(K, 2)
    Wpk, wsc = layer.pack_weights(W.cuda())
    ws = layer.workspace(M, K, N, "cuda")
    Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    H.hbl_forward_ln_ws(X.cuda(), M, K, N, g.cuda(), Wpk, wsc, a, h, Y, ws, ws.numel())
    codes = torch.empty(M, K, dtype=torch.int8, device="cuda")
    scales = torch.empty(M, dtype=torch.float32, device="cuda")
    H.hbl_quantize_ln(X.cuda(), M, K, g.cuda(), a, h, codes, scales, None)
    alpha, T = oracle.weight_quant(W.numpy())
    ref = oracle.forward_ln(X.to(torch.float64).numpy(), g.numpy(), T, alpha, a, h)
    diff = parity.check_codes(codes.cpu().numpy(), ref["codes"], ref["tie"], scales.cpu().numpy(), ref["s"])
    parity.check_y(Y.float().cpu().numpy(), ref["Y"], ref["s"], alpha, diff.sum(1))


@pytest.mark.parametrize("M,K,N,a,h", [(16, 4096, 4096, 4, 1), (5, 4096, 512, 8, 0), (2, 8192, 64, 4, 1),
                                       (11, 2048, 4096, 8, 1)])
def test_forward_ln_fused_matches_two_kernel(H, M, K, N, a, h):
    """With the RMSNorm prologue, the single-kernel decode forward gives the same
    bits as the quantiser kernel + decode GEMM."""
    from hadamard_bit_quant_b200 import layer
    X = inputs.gaussian_with_outliers(M, K, 8, inputs.outlier_channels(K, 0.01, 4).tolist(), 50.0)
    W = inputs.gaussian_weights(N, K, 9)
    g = _gain(K, 3)
    Wpk, wsc = layer.pack_weights(W.cuda())
    ws = layer.workspace(M, K, N, "cuda")
    out = {}
    try:
        for path in (6, 5):
            H.hbl_set_gemm_path(path)
            Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
            H.hbl_forward_ln_ws(X.cuda(), M, K, N, g.cuda(), Wpk, wsc, a, h, Y, ws, ws.numel())
            out[path] = Y
    finally:
        H.hbl_set_gemm_path(0)
    torch.cuda.synchronize()
    assert H.hbl_get_device_error() == 0
    assert torch.equal(out[6], out[5])


# ----------------------------------------------------------------------------- f2: rotated weights
@pytest.mark.parametrize("N,K", [(64, 256), (256, 4096), (16, 16384)])
def test_pack_weights_rotated(H, N, K):
    from hadamard_bit_quant_b200 import layer
    W = inputs.gaussian_weights(N, K, 7)
    Wpk = torch.empty(N * K // 4, dtype=torch.uint8, device="cuda")
    wsc = torch.empty(1, dtype=torch.float32, device="cuda")
    Wrot = torch.empty(N, K, dtype=torch.float32, device="cuda")
    H.hbl_pack_weights_rotated(W.cuda(), N, K, Wpk, wsc, Wrot)
    T = layer.unpack_weights(Wpk, N, K).cpu().numpy()
    torch.cuda.synchronize()
    # the rotation itself (Hadamard parity rule, per row)
    ref_rot64 = W.double().numpy() @ oracle.hadamard_matrix(K).T
    parity.check_hadamard(Wrot.cpu().numpy(), ref_rot64)
    # alpha and codes: the GPU rotates in fp32, so alpha may differ by an ulp and codes may flip
    # where |W H^T| / (alpha + eps) sits within fp32 rounding of 1/2
    a_ref, T_ref = oracle.rotated_weight_quant(W.numpy())
    assert abs(wsc.item() - float(a_ref)) <= 1e-6 * float(a_ref)
    q = np.abs(ref_rot64) / (float(a_ref) + oracle.EPS)
    near = np.abs(q - 0.5) < 1e-5
    diff = T != T_ref
    assert np.all(near[diff]), f"{int((diff & ~near).sum())} ternary codes differ away from a tie"
    # Q_w(W H^T) . Q(H x) tracks x . W^T (the rotation cancels in the exact product)
    from hadamard_bit_quant_b200 import layer as L
    M = 8
    X = inputs.gaussian_with_outliers(M, K, 5, [1, K // 2], 40.0)
    Y = L.forward(X.cuda(), Wpk, wsc, N, 8, 1).float().cpu().numpy()
    exact = X.double().numpy() @ W.double().numpy().T
    ref = oracle.forward(X.to(torch.float64).numpy(), T, wsc.item(), 8, 1)
    parity.check_y(Y, ref["Y"], ref["s"], wsc.item(), np.zeros(M))
    rel = np.linalg.norm(Y - exact) / np.linalg.norm(exact)
    assert rel < 0.7, rel      # ternary weights: coarse, but clearly the same product


# ----------------------------------------------------------------------------- f3: backward
@pytest.mark.parametrize("M,K", [(3, 256), (9, 4096), (100, 4096), (4, 16384), (2, 32768)])
def test_hadamard_backward(H, M, K):
    g = torch.Generator().manual_seed(M + K)
    G = torch.randn(M, K, generator=g, dtype=torch.float32) * 3.0
    dX = torch.empty(M, K, dtype=torch.float32, device="cuda")
    H.hbl_hadamard_backward_f32(G.cuda(), M, K, dX)
    got = dX.cpu().numpy()
    ref = oracle.hadamard_backward(G.double().numpy())
    parity.check_hadamard(got, ref)
    # adjoint identity on the GPU result: <H x, g> = <x, dX>
    x = torch.randn(M, K, generator=g, dtype=torch.float64).numpy()
    lhs = np.sum((x @ oracle.hadamard_matrix(K).T) * G.double().numpy(), axis=1)
    rhs = np.sum(x * got.astype(np.float64), axis=1)
    assert np.allclose(lhs, rhs, rtol=1e-5, atol=1e-5 * np.sqrt(K))


# ----------------------------------------------------------------------------- f4: QKV
@pytest.mark.parametrize("T,Hh,d,bits,bos", [(4, 8, 128, 4, 0), (33, 32, 128, 3, 0), (5, 4, 64, 4, -1),
                                             (2, 3, 256, 8, 1), (17, 8, 128, 2, 3)])
def test_quantize_qkv(H, T, Hh, d, bits, bos):
    g = torch.Generator().manual_seed(T * Hh + d)
    X = (torch.randn(T, Hh, d, generator=g) * torch.rand(T, Hh, 1, generator=g) * 8).to(torch.bfloat16)
    codes = torch.empty(T, Hh, d, dtype=torch.uint8, device="cuda")
    gamma = torch.empty(T, Hh, dtype=torch.float32, device="cuda")
    H.hbl_quantize_qkv(X.cuda(), T, Hh, d, bits, bos, codes, gamma)
    rows = X.reshape(T * Hh, d).double().numpy()
    bos_rows = list(range(bos * Hh, bos * Hh + Hh)) if bos >= 0 else []
    u_ref, g_ref, b_ref, tie = oracle.quantize_qkv(rows, bits, bos_rows)
    u = codes.reshape(T * Hh, d).cpu().numpy().astype(np.int64)
    assert np.array_equal(gamma.reshape(-1).cpu().numpy().astype(np.float64), g_ref)
    diff = u != u_ref.astype(np.int64)
    assert np.all(np.abs(u - u_ref.astype(np.int64))[diff] == 1)
    assert np.all(tie[diff])
    assert diff.sum() <= max(1, int(1e-4 * diff.size))
