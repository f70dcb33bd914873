"""Pins for the CPU oracle: it is checked against what the pages and the mathematics fix.

Nothing here re-types an oracle formula. Each check uses an independent fact:
hand-worked examples (``tests/golden``), a second construction (the
bit-pattern form of the Hadamard matrix, a butterfly FWHT), closed forms,
invariants, statistics derived from mean|X| = sigma*sqrt(2/pi), library
routines (``math.fsum``, ``fractions``, torch's bf16 cast, integer matmul) and
brute force on tiny inputs. ``test_oracle_mutations.py`` plants mistakes in
copies of the oracle functions and shows that these checks catch them.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from hadamard_bit_quant_b200 import inputs

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


# ----------------------------------------------------------------------------
# Independent constructions and checks, parameterised by the function under test
# so that the mutation tests can run them against planted mistakes.
# ----------------------------------------------------------------------------
def popcount_hadamard(n):
    """H[i, j] = (-1)^popcount(i & j) / sqrt(n): the sign of each entry is set by the
    bit patterns of its row and column index (section 3.4, 'Definition and Structure')."""
    i = np.arange(n)[:, None]
    j = np.arange(n)[None, :]
    bits = np.bitwise_count((i & j).astype(np.uint64)).astype(np.int64)
    return np.where(bits % 2 == 0, 1.0, -1.0) / math.sqrt(n)


def butterfly_fwht(x):
    """Fast Walsh-Hadamard transform by in-place butterflies, pure Python, natural order."""
    a = [float(v) for v in x]
    n = len(a)
    h = 1
    while h < n:
        for i in range(0, n, 2 * h):
            for j in range(i, i + h):
                u, v = a[j], a[j + h]
                a[j], a[j + h] = u + v, u - v
        h *= 2
    s = 1.0 / math.sqrt(n)
    return [v * s for v in a]


def check_hadamard(hadamard_matrix, hadamard):
    for n in (1, 2, 4, 8, 16, 32, 64, 128, 256, 1024):
        H = hadamard_matrix(n)
        P = popcount_hadamard(n)
        assert np.allclose(H, P, rtol=0, atol=1e-15), f"recursion != bit-pattern form at n={n}"
        assert np.allclose(H @ H.T, np.eye(n), atol=1e-12)          # orthogonal
        assert np.allclose(H, H.T, atol=0)                            # symmetric
        assert np.allclose(H @ H, np.eye(n), atol=1e-12)              # involution
    g = _gold("hadamard_small.json")
    for m in (1, 2, 3):
        H = hadamard_matrix(2 ** m)
        want = np.array(g[f"H{m}_signs"], dtype=np.float64) * g[f"H{m}_scale"]
        assert np.allclose(H, want, rtol=0, atol=1e-15)
    rng = np.random.default_rng(7)
    for n in (2, 4, 8, 16):
        for _ in range(5):
            x = rng.standard_normal((1, n))
            got = hadamard(x)[0]
            assert np.allclose(got, butterfly_fwht(x[0]), atol=1e-13)
    for n in (16, 256, 4096):
        e0 = np.zeros((1, n)); e0[0, 0] = 1.0
        one = np.ones((1, n))
        assert np.allclose(hadamard(e0)[0], np.full(n, 1 / math.sqrt(n)), atol=1e-14)
        want = np.zeros(n); want[0] = math.sqrt(n)
        assert np.allclose(hadamard(one)[0], want, atol=1e-9)
        x = rng.standard_normal((3, n))
        xr = hadamard(x)
        assert np.allclose(np.linalg.norm(xr, axis=1), np.linalg.norm(x, axis=1), rtol=1e-12)
        assert np.allclose(hadamard(xr), x, atol=1e-10)               # applied twice
        # A single spike at channel c is smeared evenly: every entry is +-A/sqrt(n)
        c = int(rng.integers(n)); A = 37.5
        sp = np.zeros((1, n)); sp[0, c] = A
        out = hadamard(sp)[0]
        assert np.allclose(np.abs(out), A / math.sqrt(n), rtol=1e-13)
        assert np.array_equal(np.sign(out), np.sign(popcount_hadamard(n)[:, c]))


def check_quantizers(quantize_int4, quantize_int8):
    g = _gold("quantizers_small.json")
    for case in g["int4"]:
        c, s, _ = quantize_int4(np.array([case["x"]], dtype=np.float64))
        assert c[0].tolist() == case["codes"], case
        assert math.isclose(float(s[0]), case["s"], rel_tol=1e-12, abs_tol=1e-300)
    for case in g["int8"]:
        c, s, _ = quantize_int8(np.array([case["x"]], dtype=np.float64))
        assert c[0].tolist() == case["codes"], case
        assert math.isclose(float(s[0]), case["s"], rel_tol=1e-12, abs_tol=1e-300)
    # Spike: after H, every |entry| is equal, so INT4 codes are all +-3
    # (v = +-sqrt(7)*beta/(beta+eps)) and INT8 codes all +-127.
    n = 1024
    sp = np.zeros((2, n)); sp[0, 5] = 80.0; sp[1, 900] = -3.0
    xr = oracle.hadamard(sp)
    c4, s4, _ = quantize_int4(xr)
    c8, s8, _ = quantize_int8(xr)
    assert np.array_equal(np.abs(c4), np.full((2, n), 3))
    assert np.array_equal(np.abs(c8), np.full((2, n), 127))
    assert np.array_equal(np.sign(c4), np.sign(xr))
    assert np.allclose(s4, np.array([80.0, 3.0]) / math.sqrt(n) / math.sqrt(7), rtol=1e-12)
    assert np.allclose(s8, np.array([80.0, 3.0]) / math.sqrt(n) / 127, rtol=1e-12)
    # Invariants on Gaussian-like rows
    rng = np.random.default_rng(11)
    x = rng.standard_normal((64, 4096)) * rng.uniform(0.1, 10, (64, 1))
    c4, s4, t4 = quantize_int4(x)
    c8, s8, t8 = quantize_int8(x)
    assert c4.min() >= -8 and c4.max() <= 7
    assert c8.min() >= -127 and c8.max() <= 127          # -128 is unreachable (|v| < 127.5)
    assert np.all(np.abs(c8).max(axis=1) == 127)          # absmax maps to +-127
    # Positive per-token scaling leaves the codes unchanged and scales s (eps aside)
    lam = rng.uniform(0.5, 2.0, (64, 1))
    c4b, s4b, t4b = quantize_int4(x * lam)
    keep = ~(t4 | t4b)
    assert np.array_equal(c4[keep], c4b[keep])
    assert np.allclose(s4b, s4 * lam[:, 0], rtol=1e-12)
    # Sign symmetry (ties to even are symmetric; only -8 <-> 7 clip breaks it)
    c4n, _, _ = quantize_int4(-x)
    m = (c4 > -8) & (c4 < 7)
    assert np.array_equal(c4n[m], -c4[m])
    assert np.all(c4n[c4 == -8] == 7)
    assert np.all((c4n[c4 == 7] == -7) | (c4n[c4 == 7] == -8))
    # Dequantised values stay within half a step of the input where not clipped
    # (plus the eps shift: |v| * eps / sqrt(7) <= 7.5 * 1e-5 / 2.64 < 3e-5)
    deq = c4 * s4[:, None]
    inside = (c4 > -8) & (c4 < 7)
    step = np.broadcast_to(s4[:, None], x.shape)
    assert np.all(np.abs(deq - x)[inside] <= 0.5 * step[inside] * (1 + 1e-12) + 3e-5)
    # Statistics for Gaussian input: beta = sigma*sqrt(2/pi) so v ~ sqrt(7*pi/2) z:
    # P(code = 7) = P(z >= 6.5/3.316) ~ 0.0250, P(code = -8) = P(z < -7.5/3.316) ~ 0.0119
    z = np.random.default_rng(3).standard_normal((64, 16384))
    c4, _, _ = quantize_int4(z)
    k = math.sqrt(7 * math.pi / 2)
    p7 = 0.5 * math.erfc((6.5 / k) / math.sqrt(2))
    p8 = 0.5 * math.erfc((7.5 / k) / math.sqrt(2))
    assert abs(np.mean(c4 == 7) - p7) < 0.05 * p7
    assert abs(np.mean(c4 == -8) - p8) < 0.07 * p8
    p0 = math.erf((0.5 / k) / math.sqrt(2))
    assert abs(np.mean(c4 == 0) - p0) < 0.02 * p0


def check_weight_quant(weight_scale, ternarize):
    g = _gold("hbitlinear_worked.json")
    W = np.array(g["W"], dtype=np.float32)
    a = weight_scale(W)
    assert abs(float(a) - g["alpha"]) < 1e-7
    assert ternarize(W, a).tolist() == g["T"]
    rng = np.random.default_rng(5)
    for shape, scale in [((7, 13), 1.0), ((64, 256), 0.02), ((3, 5), 1e-30), ((300, 301), 3e4)]:
        W = (rng.standard_normal(shape) * scale).astype(np.float32)
        exact = Fraction(0)
        for v in np.abs(W.astype(np.float64)).ravel():
            exact += Fraction(float(v))
        want = np.float32(float(exact) / W.size)             # exact sum -> fp64 -> /n -> fp32
        assert weight_scale(W) == want
        assert math.isclose(float(weight_scale(W)), float(np.mean(np.abs(W.astype(np.float64)))),
                            rel_tol=1e-6)
    # Ternary codes: values, monotonicity, odd symmetry, thresholds around alpha/2
    W = (rng.standard_normal((256, 1024)) * 0.02).astype(np.float32)
    a = weight_scale(W)
    T = ternarize(W, a)
    assert set(np.unique(T).tolist()) <= {-1, 0, 1}
    assert np.array_equal(ternarize(-W, a), -T)
    order = np.argsort(W.ravel(), kind="stable")
    assert np.all(np.diff(T.ravel()[order].astype(np.int64)) >= 0)
    aw = np.abs(W)
    assert np.all(T[aw < 0.499 * a] == 0)
    assert np.all(np.abs(T[aw > 0.501 * a]) == 1)
    # Zero fraction for Gaussian W: |w| < alpha/2 with alpha = sigma*sqrt(2/pi)
    Wb = np.random.default_rng(9).standard_normal((1024, 4096)).astype(np.float32)
    Tb = ternarize(Wb, weight_scale(Wb))
    p0 = math.erf(0.5 * math.sqrt(2 / math.pi) / math.sqrt(2))
    assert abs(np.mean(Tb == 0) - p0) < 0.005


def check_gemm(gemm_int):
    rng = np.random.default_rng(2)
    M, N, K = 3, 5, 7
    c = rng.integers(-128, 128, (M, K)).astype(np.int8)
    t = rng.integers(-1, 2, (N, K)).astype(np.int8)
    acc = gemm_int(c, t)
    for m in range(M):
        for n in range(N):
            assert acc[m, n] == sum(int(c[m, k]) * int(t[n, k]) for k in range(K))
    c = rng.integers(-128, 128, (17, 4096)).astype(np.int8)
    t = rng.integers(-1, 2, (33, 4096)).astype(np.int8)
    want = torch.from_numpy(c.astype(np.int64)) @ torch.from_numpy(t.astype(np.int64)).T
    assert np.array_equal(gemm_int(c, t), want.numpy())
    # extremes: all -128 against all -1 / +1
    c = np.full((2, 16384), -128, np.int8)
    t = np.stack([np.full(16384, -1, np.int8), np.full(16384, 1, np.int8)])
    assert gemm_int(c, t).tolist() == [[128 * 16384, -128 * 16384]] * 2


def check_bf16(to_bf16):
    rng = np.random.default_rng(4)
    x = (rng.standard_normal(100000) * np.exp(rng.uniform(-30, 30, 100000))).astype(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(to_bf16(x.astype(np.float64)), want)
    # exact ties go to even: 1 + 2^-8 is halfway between 1 and 1 + 2^-7
    ties = np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 2 ** -130 * 1.5])
    assert to_bf16(ties).tolist() == [1.0, 1 + 2 ** -6, -1.0, np.float32(2 ** -130 * 1.5)]


def check_forward(forward):
    g = _gold("hbitlinear_worked.json")
    X = np.array(g["X"], dtype=np.float64)
    T = np.array(g["T"], dtype=np.int8)
    alpha = oracle.weight_scale(np.array(g["W"], dtype=np.float32))
    for bits, key in ((4, "int4"), (8, "int8")):
        out = forward(X, T, alpha, bits, 1)
        assert np.allclose(out["Xr"], g["Xr"], atol=1e-14)
        assert out["codes"].tolist() == g[key]["codes"]
        assert np.allclose(out["s"], g[key]["s"], rtol=1e-12)
        assert out["acc"].tolist() == g[key]["acc"]
        assert out["Y"].tolist() == g[key]["Y"]
    # With the Hadamard on, the layer multiplies the rotated input X_r = H x by the
    # ternary weights. The quantised output must track X_r . (alpha T) within the
    # INT8 quantisation error, and must not track the unrotated x . (alpha T)
    # (catches a Hadamard that is skipped or applied along the wrong axis).
    case = inputs.tiny_case()
    Xt = case.make_x().to(torch.float64).numpy()
    W = case.make_w().numpy()
    a, Tt = oracle.weight_quant(W)
    out = forward(Xt, Tt, a, 8, 1)
    Wq = Tt.astype(np.float64) * float(a)
    rot = popcount_hadamard(Xt.shape[1])
    ref = (Xt @ rot.T) @ Wq.T
    plain = Xt @ Wq.T
    assert np.linalg.norm(out["Y"] - ref) / np.linalg.norm(ref) < 0.05
    assert np.linalg.norm(out["Y"] - plain) / np.linalg.norm(plain) > 0.5


# ----------------------------------------------------------------------------
def test_hadamard_pins():
    check_hadamard(oracle.hadamard_matrix, oracle.hadamard)


def test_hadamard_rejects_non_power_of_two():
    with pytest.raises(ValueError):
        oracle.hadamard_matrix(12)


def test_quantizer_pins():
    check_quantizers(oracle.quantize_int4, oracle.quantize_int8)


def test_weight_quant_pins():
    check_weight_quant(oracle.weight_scale, oracle.ternarize)


def test_gemm_pins():
    check_gemm(oracle.gemm_int)


def test_bf16_pins():
    check_bf16(oracle.to_bf16)


def test_forward_pins():
    check_forward(oracle.forward)


def test_round_clip_brute_force():
    vals = np.arange(-300, 301) / 4.0          # includes every half-integer in range
    for lo, hi in ((-1, 1), (-8, 7), (-128, 127)):
        got = oracle.round_clip(vals, lo, hi)
        for v, r in zip(vals, got):
            cands = list(range(lo, hi + 1))
            d = [abs(v - c) for c in cands]
            best = min(d)
            ties = [c for c, dd in zip(cands, d) if dd == best]
            want = ties[0] if len(ties) == 1 else [c for c in ties if c % 2 == 0][0]
            assert r == want, (v, r, want)


def test_exact_sum_matches_fsum():
    rng = np.random.default_rng(1)
    for scale in (1.0, 1e-3, 1e30, 1e-40):
        x = (np.abs(rng.standard_normal(20000)) * scale).astype(np.float32).astype(np.float64)
        assert oracle.exact_sum_rounded(x) == math.fsum(x)
    x = np.concatenate([np.float32([3e38, 1e-45, 1.0, 2 ** -24]).astype(np.float64),
                        np.abs(rng.standard_normal(1000)).astype(np.float32)])
    assert oracle.exact_sum_rounded(x) == math.fsum(x)


def test_near_tie_flags():
    # gamma = 127 fixes the INT8 multiplier at 127/(127+eps) = 1 - 7.9e-8, so
    # v = x to 1e-5: 10.5 and -3.5 sit at ties, 10.4, 0 and 127 do not.
    xr = np.array([[127.0, 10.5, 10.4, -3.5, 0.0]])
    _, _, tie8 = oracle.quantize_int8(xr)
    assert tie8[0].tolist() == [False, True, False, True, False]
    # INT4: beta = 2 (mean of |[7.5, -0.5, 0, 0]|... chosen so v lands on +-clip edges)
    x = np.array([[8.0, 0.0, 0.0, 0.0]])      # beta = 2, v = sqrt7/2 * 8 = 10.58 -> clipped, no tie
    _, _, tie4 = oracle.quantize_int4(x)
    assert not tie4.any()
