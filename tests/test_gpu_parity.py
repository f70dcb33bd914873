"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Stage by stage -- packed weights and alpha, the Hadamard in fp32, codes and
scales, the integer GEMM, the bf16 output -- on the seeded workloads, at sizes
the oracle finishes in seconds (several tiles plus ragged tails) and at the
full benchmark sizes on sampled tokens.
"""
import numpy as np
import pytest
import torch

import oracle
import parity
from hadamard_bit_quant_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    from hadamard_bit_quant_b200 import build, layer
    build.build()
    assert torch.cuda.is_available()
    return layer


def dev(t):
    return t.to("cuda")


def _oracle_weights(W):
    return oracle.weight_quant(W.numpy())


# ----------------------------------------------------------------------------- weights
@pytest.mark.parametrize("N,K,seed", [(256, 256, 0), (48, 768, 5), (4096, 4096, 1), (1024, 16384, 2),
                                      (16, 32768, 9)])
def test_pack_bit_exact(L, N, K, seed):
    W = inputs.gaussian_weights(N, K, seed)
    a_ref, T_ref = _oracle_weights(W)
    Wpk, ws = L.pack_weights(dev(W))
    T = L.unpack_weights(Wpk, N, K)
    torch.cuda.synchronize()
    assert ws.item() == float(a_ref), (ws.item(), float(a_ref))
    assert np.array_equal(T.cpu().numpy(), T_ref)


def test_pack_special_weights(L):
    # all zero (alpha = 0: every code 0), a wide dynamic range, exact half-way points
    N, K = 16, 256
    for W in (torch.zeros(N, K), torch.randn(N, K, generator=torch.Generator().manual_seed(3))
              * torch.logspace(-30, 30, K)[None, :].float(),
              torch.full((N, K), 0.5) * torch.where(torch.arange(K) % 2 == 0, 1.0, -1.0)[None, :]):
        W = W.float().contiguous()
        a_ref, T_ref = _oracle_weights(W)
        Wpk, ws = L.pack_weights(dev(W))
        T = L.unpack_weights(Wpk, N, K)
        assert ws.item() == float(a_ref)
        assert np.array_equal(T.cpu().numpy(), T_ref)


# ----------------------------------------------------------------------------- Hadamard
@pytest.mark.parametrize("K", [256, 512, 1024, 2048, 4096, 8192, 16384, 32768])
def test_hadamard_f32(L, K):
    M = 3 if K >= 16384 else 9
    X = inputs.gaussian_with_outliers(M, K, 10 + K, [1, K // 3, K - 1], 40.0)
    Xr = L.hadamard_f32(dev(X)).cpu().numpy()
    ref = oracle.hadamard(X.to(torch.float64).numpy())
    parity.check_hadamard(Xr, ref)


# Batches above the few-token threshold (64 tokens) take the throughput
# configurations of the transform (more values per thread, several tokens per
# CTA for small K); each K is checked there too, with ragged CTA tails, on
# sampled tokens (tokens are independent, so a sampled row is exact).
@pytest.mark.parametrize("K,M", [(256, 65), (512, 70), (1024, 129), (2048, 100), (4096, 257), (8192, 97),
                                 (16384, 130), (32768, 66)])
def test_hadamard_f32_many_tokens(L, K, M):
    X = inputs.gaussian_with_outliers(M, K, 20 + K, inputs.outlier_channels(K, 0.01, 3).tolist(), 50.0)
    rng = np.random.default_rng(K)
    rows = np.unique(np.concatenate([[0, 1, M - 2, M - 1], rng.integers(0, M, 12)]))
    Xr = L.hadamard_f32(dev(X)).cpu().numpy()[rows]
    ref = oracle.hadamard(X[rows].to(torch.float64).numpy())
    parity.check_hadamard(Xr, ref)


def test_hadamard_f32_prefill_shape(L):
    """The prefill down_proj input (M=4096, K=16384, gated heavy-tailed values):
    the transform's fp32 output on 40 sampled tokens, first and last included."""
    case = inputs.prefill_down_case()
    X = case.make_x()
    rng = np.random.default_rng(2)
    rows = np.unique(np.concatenate([[0, 1, 4094, 4095], rng.integers(0, case.M, 36)]))
    Xr = L.hadamard_f32(dev(X)).cpu().numpy()[rows]
    ref = oracle.hadamard(X[rows].to(torch.float64).numpy())
    assert len(rows) >= 32
    parity.check_hadamard(Xr, ref)


def test_hadamard_special_rows(L):
    K = 4096
    X = torch.zeros(4, K)
    X[1, 17] = 3.0                      # spike: every output +-3/64
    X[2, :] = 1.0                       # constant: all energy in X_r[0]
    X[3] = torch.randn(K, generator=torch.Generator().manual_seed(1))
    X = X.to(torch.bfloat16)
    Xr = L.hadamard_f32(dev(X)).cpu().numpy()
    ref = oracle.hadamard(X.to(torch.float64).numpy())
    assert np.all(Xr[0] == 0)
    assert np.allclose(np.abs(Xr[1]), 3.0 / 64, rtol=0, atol=0)
    parity.check_hadamard(Xr[1:], ref[1:])


# ----------------------------------------------------------------------------- quantiser
def _check_quant(L, X, act_bits, use_h):
    codes, scales, csum = L.quantize(dev(X), act_bits, use_h)
    Xd = X.to(torch.float64).numpy()
    Xr = oracle.hadamard(Xd) if use_h else Xd
    c_ref, s_ref, tie = oracle.quantize_act(Xr, act_bits)
    c = codes.cpu().numpy()
    parity.check_codes(c, c_ref, tie, scales.cpu().numpy(), s_ref)
    assert np.array_equal(csum.cpu().numpy(), c.astype(np.int64).sum(1))
    return c


@pytest.mark.parametrize("act_bits", [4, 8])
@pytest.mark.parametrize("K,M", [(256, 8), (256, 37), (1024, 19), (4096, 16), (4096, 130), (8192, 5),
                                 (16384, 6), (32768, 3)])
def test_quantize_hadamard(L, act_bits, K, M):
    X = inputs.gaussian_with_outliers(M, K, K + M, inputs.outlier_channels(K, 0.01, 1).tolist(), 50.0)
    _check_quant(L, X, act_bits, 1)


@pytest.mark.parametrize("act_bits", [4, 8])
@pytest.mark.parametrize("K,M", [(256, 3), (768, 33), (4096, 17), (12288, 4), (16384, 2), (40960, 2)])
def test_quantize_plain(L, act_bits, K, M):
    X = inputs.student_t(M, K, K + 3)
    _check_quant(L, X, act_bits, 0)


@pytest.mark.parametrize("act_bits", [4, 8])
def test_quantize_degenerate_rows(L, act_bits):
    K = 1024
    X = torch.zeros(5, K)
    X[1, 100] = -7.0
    X[2, :] = 2.0
    X[3, :] = 1e-6
    X[4] = torch.randn(K, generator=torch.Generator().manual_seed(2)) * 1e4
    X = X.to(torch.bfloat16)
    c = _check_quant(L, X, act_bits, 1)
    assert np.all(c[0] == 0)
    _check_quant(L, X, act_bits, 0)


# ----------------------------------------------------------------------------- integer GEMM
@pytest.mark.parametrize("M,K,N", [(1, 256, 16), (5, 512, 48), (16, 4096, 4096), (37, 1024, 80),
                                   (130, 2048, 272), (64, 16384, 128), (300, 768, 64)])
def test_gemm_codes_bit_exact(L, M, K, N):
    g = torch.Generator().manual_seed(M * 7 + K)
    codes = torch.randint(-128, 128, (M, K), generator=g, dtype=torch.int8)
    W = inputs.gaussian_weights(N, K, M + N)
    _, T_ref = _oracle_weights(W)
    Wpk, _ = L.pack_weights(dev(W))
    acc = L.gemm_codes(dev(codes), Wpk, N).cpu().numpy()
    assert np.array_equal(acc, oracle.gemm_int(codes.numpy(), T_ref))


def test_gemm_codes_extremes(L):
    M, K, N = 4, 32768, 32
    codes = torch.full((M, K), -128, dtype=torch.int8)
    codes[1] = 127
    W = torch.where(torch.arange(K)[None, :] % 3 == 0, -1.0, 1.0).repeat(N, 1).float()
    W[N // 2:] *= -1
    _, T_ref = _oracle_weights(W)
    Wpk, _ = L.pack_weights(dev(W))
    acc = L.gemm_codes(dev(codes), Wpk, N).cpu().numpy()
    assert np.array_equal(acc, oracle.gemm_int(codes.numpy(), T_ref))


# ----------------------------------------------------------------------------- forward
def _forward_case(L, X, W, act_bits, use_h, rows=None, ws=False):
    a_ref, T_ref = _oracle_weights(W)
    M, K = X.shape
    N = W.shape[0]
    Wpk, wsc = L.pack_weights(dev(W))
    Xd = dev(X)
    wsb = L.workspace(M, K, N, "cuda") if ws else None
    Y = L.forward(Xd, Wpk, wsc, N, act_bits, use_h, ws=wsb)
    codes, scales, _ = L.quantize(Xd, act_bits, use_h)
    torch.cuda.synchronize()
    rows = np.arange(M) if rows is None else np.asarray(rows)
    ref = oracle.forward_rows(X.to(torch.float64).numpy(), T_ref, a_ref, act_bits, use_h, rows)
    c = codes.cpu().numpy()[rows]
    diff = parity.check_codes(c, ref["codes"], ref["tie"], scales.cpu().numpy()[rows], ref["s"])
    # given the GPU's own codes the oracle's integer GEMM is reproduced exactly by Y's construction
    parity.check_y(Y.float().cpu().numpy()[rows], ref["Y"], ref["s"], a_ref, diff.sum(1))
    return Y


def test_forward_tiny_config(L):
    case = inputs.tiny_case()
    _forward_case(L, case.make_x(), case.make_w(), case.act_bits, case.use_hadamard)


@pytest.mark.parametrize("case", inputs.decode_oproj_cases(), ids=lambda c: c.label)
def test_forward_decode_config(L, case):
    _forward_case(L, case.make_x(), case.make_w(), case.act_bits, case.use_hadamard)


def test_forward_prefill_config_sampled(L):
    case = inputs.prefill_down_case()
    rng = np.random.default_rng(0)
    rows = np.unique(np.concatenate([[0, 127, 128, case.M - 1], rng.integers(0, case.M, 28)]))
    _forward_case(L, case.make_x(), case.make_w(), case.act_bits, case.use_hadamard, rows, ws=True)


@pytest.mark.parametrize("M", [1, 64, 512, 4096])
def test_forward_block7b(L, M):
    rng = np.random.default_rng(M)
    for case in inputs.block7b_cases(M):
        rows = None if M <= 64 else np.unique(np.concatenate([[0, M - 1], rng.integers(0, M, 14)]))
        _forward_case(L, case.make_x(), case.make_w(), case.act_bits, case.use_hadamard, rows)


def test_forward_sweep_sample(L):
    rng = np.random.default_rng(4)
    pts = [(int(rng.choice(inputs.SWEEP_MS)), int(rng.choice(inputs.SWEEP_KN)), int(rng.choice(inputs.SWEEP_KN)),
            int(rng.choice([4, 8])), int(rng.integers(0, 2))) for _ in range(6)]
    pts.append((16384, 2048, 2048, 4, 1))
    pts.append((1, 16384, 16384, 8, 0))
    for (M, K, N, a, h) in pts:
        case = inputs.sweep_case(M, K, N, a, h)
        rows = np.unique(np.concatenate([[0, M - 1], rng.integers(0, M, 30)]))
        _forward_case(L, case.make_x(), case.make_w(), a, h, rows)


@pytest.mark.parametrize("M,K,N,a,h", [(1, 256, 16, 4, 1), (7, 512, 48, 8, 1), (65, 768, 80, 4, 0),
                                       (129, 1024, 144, 8, 0), (3, 32768, 64, 4, 1), (2, 65536, 32, 8, 0)])
def test_forward_ragged_and_extreme_shapes(L, M, K, N, a, h):
    X = inputs.student_t(M, K, M + K)
    W = inputs.gaussian_weights(N, K, N + K)
    _forward_case(L, X, W, a, h, ws=True)


def test_forward_empty_batch(L):
    W = inputs.gaussian_weights(64, 256, 0)
    Wpk, wsc = L.pack_weights(dev(W))
    Y = L.forward(torch.empty(0, 256, dtype=torch.bfloat16, device="cuda"), Wpk, wsc, 64, 4, 1)
    assert Y.shape == (0, 64)


def test_forward_rejects_bad_workspace(L):
    from hadamard_bit_quant_b200 import hbl
    W = inputs.gaussian_weights(64, 256, 0)
    Wpk, wsc = L.pack_weights(dev(W))
    X = dev(inputs.student_t(4, 256, 0))
    small = torch.empty(64, dtype=torch.uint8, device="cuda")
    with pytest.raises(hbl.HblError) as e:
        L.forward(X, Wpk, wsc, 64, 4, 1, ws=small)
    assert e.value.status == 7
    assert hbl.hbl_get_device_error() == 0


# ----------------------------------------------------------------------------- both GEMM kernels
@pytest.fixture
def gemm_path(L):
    from hadamard_bit_quant_b200 import hbl
    yield hbl.hbl_set_gemm_path
    hbl.hbl_set_gemm_path(0)


@pytest.mark.parametrize("path", [0, 1, 2, 3, 4, 5],
                         ids=["auto", "mma_sync", "tcgen05", "decode_1cta", "tcgen05_1tile", "stream"])
@pytest.mark.parametrize("M,K,N", [(256, 256, 128), (16, 4096, 512), (64, 32768, 32), (33, 1024, 144),
                                   (1, 2048, 16), (9, 16384, 4096), (16, 8192, 2416), (3, 4096, 16 * 1184), (1, 256, 16), (37, 512, 48), (300, 1024, 272),
                                   (512, 4096, 256), (257, 2048, 130 * 16), (1024, 16384, 128)])
def test_gemm_paths_bit_exact(L, gemm_path, path, M, K, N):
    gemm_path(path)
    g = torch.Generator().manual_seed(M + K + N)
    codes = torch.randint(-128, 128, (M, K), generator=g, dtype=torch.int8)
    W = inputs.gaussian_weights(N, K, M + 1)
    _, T_ref = _oracle_weights(W)
    Wpk, _ = L.pack_weights(dev(W))
    acc = L.gemm_codes(dev(codes), Wpk, N).cpu().numpy()
    from hadamard_bit_quant_b200 import hbl
    assert hbl.hbl_get_device_error() == 0
    assert np.array_equal(acc, oracle.gemm_int(codes.numpy(), T_ref))


@pytest.mark.parametrize("path", [1, 2, 4], ids=["mma_sync", "tcgen05", "tcgen05_1tile"])
def test_forward_paths(L, gemm_path, path):
    gemm_path(path)
    case = inputs.prefill_down_case(M=300)
    case.K, case.N = 4096, 512
    _forward_case(L, case.make_x(), case.make_w(), 4, 1, ws=True)
    _forward_case(L, inputs.student_t(129, 1024, 1), inputs.gaussian_weights(80, 1024, 2), 8, 0)


# ----------------------------------------------------------------------------- fused decode forward
FUSED_SHAPES = [(1, 2048, 16, 4, 1), (2, 4096, 4096, 8, 1), (3, 4096, 48, 4, 0), (5, 8192, 2416, 4, 1),
                (8, 8192, 256, 8, 0), (9, 2048, 4096, 4, 1), (16, 4096, 4096, 4, 1), (16, 4096, 4096, 8, 0),
                (12, 2048, 16 * 1184, 8, 1), (16, 4096, 16 * 1200, 4, 1), (7, 4096, 1024, 4, 1)]


@pytest.mark.parametrize("M,K,N,a,h", FUSED_SHAPES)
def test_fused_forward_matches_two_kernel_path(L, gemm_path, M, K, N, a, h):
    """The single-kernel decode forward (transform, quantiser, GEMM and dequant
    with the codes exchanged inside a cluster) gives the same bits as the
    quantiser kernel followed by each decode GEMM kernel; those are checked
    against the oracle by the other forward and GEMM tests."""
    from hadamard_bit_quant_b200 import hbl
    X = inputs.gaussian_with_outliers(M, K, M + K, inputs.outlier_channels(K, 0.01, 1).tolist(), 50.0)
    W = inputs.gaussian_weights(N, K, N + 1)
    Wpk, wsc = L.pack_weights(dev(W))
    Xd = dev(X)
    out = {}
    for path in (6, 5, 3):
        gemm_path(path)
        out[path] = L.forward(Xd, Wpk, wsc, N, a, h).clone()
    torch.cuda.synchronize()
    assert hbl.hbl_get_device_error() == 0
    assert torch.equal(out[6], out[5])
    assert torch.equal(out[6], out[3])


@pytest.mark.parametrize("path", [5, 3], ids=["stream", "decode_no_cluster"])
@pytest.mark.parametrize("case", inputs.decode_oproj_cases(), ids=lambda c: c.label)
def test_forward_decode_two_kernel_paths(L, gemm_path, path, case):
    gemm_path(path)
    _forward_case(L, case.make_x(), case.make_w(), case.act_bits, case.use_hadamard)


def test_chained_forwards_match_synchronised(L):
    """Back-to-back forwards on one stream, each consuming the previous output
    (programmatic dependent launches overlap their prologues), must give the
    same bits as the same chain with a device synchronisation after each step,
    and as the chain replayed from a CUDA graph."""
    K = N = 4096
    layers = [L.pack_weights(dev(inputs.gaussian_weights(N, K, 50 + i))) for i in range(6)]
    for M, a in ((16, 4), (3, 8), (200, 4)):
        X0 = dev(inputs.gaussian_with_outliers(M, K, 9, [5, 700], 30.0))
        ws = L.workspace(M, K, N, "cuda")

        def chain(sync):
            x = X0
            for Wpk, wsc in layers:
                x = L.forward(x, Wpk, wsc, N, a, 1, ws=ws)
                if sync:
                    torch.cuda.synchronize()
            return x

        ref = chain(True).clone()
        got = chain(False).clone()
        torch.cuda.synchronize()
        assert torch.equal(ref, got)
        outs = []
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            outs.append(chain(False))
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(ref, outs[0])
        from hadamard_bit_quant_b200 import hbl
        assert hbl.hbl_get_device_error() == 0
