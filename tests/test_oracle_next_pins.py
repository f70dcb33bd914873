"""Pins for the oracle functions beyond the LN-free forward: the RMSNorm
prologue, the weight-and-activation rotation variant, the Hadamard backward
(Eq. 10) and the post-RoPE QKV quantiser. Each check uses a fact independent
of the oracle's own formula (hand-worked values, adjoint identities,
invariants, the bit-pattern Hadamard)."""
import json
import math
import os

import numpy as np
import pytest

import oracle
from test_oracle_pins import popcount_hadamard

GOLD = os.path.join(os.path.dirname(__file__), "golden", "next_rows_small.json")


def _g():
    with open(GOLD) as f:
        return json.load(f)


def check_rmsnorm(rmsnorm):
    g = _g()["rmsnorm"]
    assert np.allclose(rmsnorm(np.array(g["x"])), g["y"], rtol=1e-12)
    rng = np.random.default_rng(0)
    x = rng.standard_normal((8, 512)) * rng.uniform(0.5, 50, (8, 1))
    y = rmsnorm(x)
    assert np.allclose(np.sqrt(np.mean(y * y, axis=1)), 1.0, rtol=1e-5)       # unit RMS
    assert np.allclose(rmsnorm(3.7 * x), y, rtol=1e-6)                          # scale invariant
    gain = rng.uniform(0.5, 2.0, 512)
    assert np.allclose(rmsnorm(x, gain), y * gain[None, :], rtol=1e-12)
    assert np.all(rmsnorm(np.zeros((1, 16))) == 0)
    assert np.allclose(np.sign(y), np.sign(x))


def check_rotation(rotate_weights):
    rng = np.random.default_rng(1)
    W = (rng.standard_normal((16, 256)) * 0.02).astype(np.float32)
    R = rotate_weights(W)
    assert R.dtype == np.float32
    assert np.allclose(R.astype(np.float64), W.astype(np.float64) @ popcount_hadamard(256).T, atol=1e-7)
    assert np.allclose(np.linalg.norm(R, axis=1), np.linalg.norm(W, axis=1), rtol=1e-5)
    assert np.allclose(rotate_weights(R), W, atol=1e-7)                       # H is an involution
    x = rng.standard_normal((4, 256))
    # (W H^T)(H x) = W x: the rotation cancels in the un-quantised product
    assert np.allclose((x @ popcount_hadamard(256).T) @ R.T.astype(np.float64),
                       x @ W.T.astype(np.float64), atol=1e-5)


def check_backward(hadamard_backward):
    rng = np.random.default_rng(2)
    for n in (16, 256, 4096):
        x = rng.standard_normal((3, n))
        gr = rng.standard_normal((3, n))
        Hx = x @ popcount_hadamard(n).T
        # adjoint identity <H x, g> = <x, H^T g>: the definition of the backward map
        assert np.allclose(np.sum(Hx * gr, axis=1), np.sum(x * hadamard_backward(gr), axis=1), rtol=1e-9)
        assert np.allclose(hadamard_backward(Hx), x, atol=1e-10)


def check_qkv(quantize_qkv, dequantize_qkv):
    g = _g()["qkv"]
    x = np.array([g["x"]])
    for b in ("4", "3"):
        u, gamma, bb, _ = quantize_qkv(x, int(b))
        assert u[0].tolist() == g["codes"][b] and gamma[0] == 1.0 and bb[0] == int(b)
    u, _, bb, _ = quantize_qkv(x, 4, bos_rows=[0])
    assert u[0].tolist() == g["codes"]["8"] and bb[0] == 8
    rng = np.random.default_rng(3)
    X = rng.standard_normal((64, 128)) * rng.uniform(0.1, 10, (64, 1))
    for b in (3, 4, 8):
        u, gamma, bb, tie = quantize_qkv(X, b, bos_rows=[0, 5])
        top = 2 ** bb - 1
        assert np.all(u <= top[:, None])
        am = np.argmax(np.abs(X), axis=1)
        ext = u[np.arange(64), am]
        assert np.all((ext == 0) | (ext == top))                    # absmax maps to an end of the range
        step = 2.0 * gamma / top
        err = np.abs(dequantize_qkv(u, gamma, bb) - X)
        assert np.all(err <= 0.5 * step[:, None] * (1 + 1e-9) + 1e-4 * gamma[:, None])
        order = np.argsort(X[7])
        assert np.all(np.diff(u[7][order].astype(int)) >= 0)        # monotone


def test_rmsnorm_pins():
    check_rmsnorm(oracle.rmsnorm)


def test_forward_ln_is_quantiser_invariant():
    # quantisers are invariant to a positive per-token factor, so LN without a
    # gain leaves the codes unchanged (away from ties) and rescales s
    rng = np.random.default_rng(4)
    X = rng.standard_normal((6, 1024)) * rng.uniform(0.5, 20, (6, 1))
    a, T = oracle.weight_quant((rng.standard_normal((32, 1024)) * 0.02).astype(np.float32))
    for bits in (4, 8):
        f = oracle.forward(X, T, a, bits, 1)
        fl = oracle.forward_ln(X, None, T, a, bits, 1)
        keep = ~(f["tie"] | fl["tie"])
        assert np.array_equal(f["codes"][keep], fl["codes"][keep])
        r = 1.0 / np.sqrt(np.mean(X * X, axis=1) + oracle.RMS_EPS)
        assert np.allclose(fl["s"], f["s"] * r, rtol=1e-6)


def test_rotation_pins():
    check_rotation(oracle.rotate_weights)


def test_backward_pins():
    check_backward(oracle.hadamard_backward)


def test_qkv_pins():
    check_qkv(oracle.quantize_qkv, oracle.dequantize_qkv)


# planted mistakes must be caught
def _rms_mean(X, gain=None):
    X = np.asarray(X, np.float64)
    return X / (np.mean(np.abs(X), axis=1) + 1e-5)[:, None]


def _rms_no_sqrt(X, gain=None):
    X = np.asarray(X, np.float64)
    return X / (np.mean(X * X, axis=1) + 1e-5)[:, None]


@pytest.mark.parametrize("fn", [_rms_mean, _rms_no_sqrt])
def test_rmsnorm_mutants(fn):
    with pytest.raises(AssertionError):
        check_rmsnorm(fn)


def _rot_unscaled(W):
    W = np.asarray(W, np.float64)
    return (W @ (popcount_hadamard(W.shape[1]) * math.sqrt(W.shape[1])).T).astype(np.float32)


def _rot_cols(W):
    W = np.asarray(W, np.float64)
    return (popcount_hadamard(W.shape[0]) @ W).astype(np.float32)


@pytest.mark.parametrize("fn", [_rot_unscaled, _rot_cols])
def test_rotation_mutants(fn):
    with pytest.raises(AssertionError):
        check_rotation(fn)


def _bwd_twice(G):
    return oracle.hadamard_backward(oracle.hadamard_backward(G))


def _bwd_scaled(G):
    return oracle.hadamard_backward(G) * 2.0


@pytest.mark.parametrize("fn", [_bwd_twice, _bwd_scaled])
def test_backward_mutants(fn):
    with pytest.raises(AssertionError):
        check_backward(fn)


def _qkv_full_pow(Xh, bits, bos_rows=()):
    Xh = np.asarray(Xh, np.float64)
    b = np.full(Xh.shape[0], bits); b[list(bos_rows)] = 8
    top = (2.0 ** b)[:, None]
    gam = np.max(np.abs(Xh), 1)
    u = np.clip(np.rint(0.5 * top * (Xh / (gam + 1e-5)[:, None] + 1)), 0, top - 1)
    return u.astype(np.uint8), gam, b, np.zeros(Xh.shape, bool)


def _qkv_no_bos(Xh, bits, bos_rows=()):
    return oracle.quantize_qkv(Xh, bits, ())


@pytest.mark.parametrize("fn", [_qkv_full_pow, _qkv_no_bos])
def test_qkv_mutants(fn):
    with pytest.raises(AssertionError):
        check_qkv(fn, oracle.dequantize_qkv)
