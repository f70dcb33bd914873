"""Plant plausible mistakes in copies of the oracle functions (on the CPU) and show
that the pins of ``test_oracle_pins.py`` reject every one of them."""
import math

import numpy as np
import pytest

import oracle
from oracle import hbl_oracle as ho
import test_oracle_pins as pins


def _expect_fail(check, *fns):
    with pytest.raises((AssertionError, ValueError, FloatingPointError)):
        with np.errstate(all="ignore"):
            check(*fns)


def _had_from(build):
    def hadamard(X):
        X = np.asarray(X, dtype=np.float64)
        return X @ build(X.shape[1]).T
    return hadamard


def _rec(n, block, scale):
    m = int(n).bit_length() - 1
    S = np.ones((1, 1))
    for _ in range(m):
        S = block(S)
    return S * scale(n, m)


HAD_MUTANTS = {
    "sign in the wrong quadrant": lambda n: _rec(n, lambda S: np.block([[S, -S], [S, S]]),
                                                 lambda n, m: 2.0 ** (-m / 2)),
    "scale 1/n instead of 1/sqrt(n)": lambda n: _rec(n, lambda S: np.block([[S, S], [S, -S]]),
                                                     lambda n, m: 1.0 / n),
    "no normalisation": lambda n: _rec(n, lambda S: np.block([[S, S], [S, -S]]),
                                       lambda n, m: 1.0),
    "bit-reversed (sequency-like) order": lambda n: (
        ho.hadamard_matrix(n)[np.array([int(format(i, f"0{max(1, n.bit_length() - 1)}b")[::-1], 2)
                                        for i in range(n)])] if n > 1 else ho.hadamard_matrix(n)),
}


@pytest.mark.parametrize("name", list(HAD_MUTANTS))
def test_hadamard_mutants_caught(name):
    build = HAD_MUTANTS[name]
    _expect_fail(pins.check_hadamard, build, _had_from(build))


def _q4(anchor=math.sqrt(7), stat="mean", lo=-8, hi=7, eps=ho.EPS, rnd=np.rint):
    def q(Xr):
        Xr = np.asarray(Xr, dtype=np.float64)
        beta = np.mean(np.abs(Xr), 1) if stat == "mean" else np.max(np.abs(Xr), 1)
        v = (anchor / (beta + eps))[:, None] * Xr
        c = np.minimum(np.maximum(rnd(v), lo), hi).astype(np.int8)
        return c, beta / anchor, np.zeros(v.shape, bool)
    return q


def _q8(top=127.0, eps=ho.EPS, rnd=np.rint):
    def q(Xr):
        Xr = np.asarray(Xr, dtype=np.float64)
        g = np.max(np.abs(Xr), 1)
        v = (top / (g + eps))[:, None] * Xr
        c = np.minimum(np.maximum(rnd(v), -128), 127).astype(np.int8)
        return c, g / top, np.zeros(v.shape, bool)
    return q


Q_MUTANTS = {
    "INT4 anchor 7 instead of sqrt(7)": (_q4(anchor=7.0), ho.quantize_int8),
    "INT4 anchor 3.5": (_q4(anchor=3.5), ho.quantize_int8),
    "INT4 absmax instead of absmean": (_q4(stat="max"), ho.quantize_int8),
    "INT4 clip [-7, 7]": (_q4(lo=-7), ho.quantize_int8),
    "INT4 floor instead of round": (_q4(rnd=np.floor), ho.quantize_int8),
    "INT4 eps dropped": (_q4(eps=0.0), ho.quantize_int8),
    "INT8 128 instead of 127": (ho.quantize_int4, _q8(top=128.0)),
    "INT8 round half away from zero": (ho.quantize_int4, _q8(rnd=lambda v: np.trunc(v + np.copysign(0.5, v)))),
}


@pytest.mark.parametrize("name", list(Q_MUTANTS))
def test_quantizer_mutants_caught(name):
    _expect_fail(pins.check_quantizers, *Q_MUTANTS[name])


def _scale_max(W):
    return np.float32(np.max(np.abs(np.asarray(W, np.float64))))


def _scale_fp32_sum(W):
    w = np.abs(np.asarray(W, np.float32))
    return np.float32(np.sum(w, dtype=np.float32) / np.float32(w.size))


def _tern(rnd=np.rint, eps=ho.EPS, lo=-1):
    def t(W, alpha):
        w = np.asarray(W, np.float32)
        q = w / (np.float32(alpha) + np.float32(eps))
        return np.minimum(np.maximum(rnd(q), lo), 1).astype(np.int8)
    return t


W_MUTANTS = {
    "alpha = absmax": (_scale_max, ho.ternarize),
    "alpha summed in fp32": (_scale_fp32_sum, ho.ternarize),
    "ternary by floor": (ho.weight_scale, _tern(rnd=np.floor)),
    "binary {0,1} clip": (ho.weight_scale, _tern(lo=0)),
}


@pytest.mark.parametrize("name", list(W_MUTANTS))
def test_weight_mutants_caught(name):
    _expect_fail(pins.check_weight_quant, *W_MUTANTS[name])


def _gemm_transposed_t(c, t):
    c = np.asarray(c, np.float64); t = np.asarray(t, np.float64)
    return (c @ t[:, ::-1].T).astype(np.int64)


def _gemm_drop_last(c, t):
    c = np.asarray(c, np.float64)[:, :-1]; t = np.asarray(t, np.float64)[:, :-1]
    return (c @ t.T).astype(np.int64)


def _gemm_int16_wrap(c, t):
    return ho.gemm_int(c, t).astype(np.int16).astype(np.int64)


@pytest.mark.parametrize("fn", [_gemm_transposed_t, _gemm_drop_last, _gemm_int16_wrap])
def test_gemm_mutants_caught(fn):
    _expect_fail(pins.check_gemm, fn)


def _bf16_truncate(y):
    y = np.asarray(y, np.float64).astype(np.float32)
    b = y.view(np.uint32) & np.uint32(0xFFFF0000)
    return b.view(np.float32)


def _bf16_via_fp16(y):
    return np.asarray(y, np.float64).astype(np.float16).astype(np.float32)


@pytest.mark.parametrize("fn", [_bf16_truncate, _bf16_via_fp16])
def test_bf16_mutants_caught(fn):
    _expect_fail(pins.check_bf16, fn)


def _fwd_no_hadamard(X, T, alpha, act_bits, use_hadamard):
    return ho.forward(X, T, alpha, act_bits, 0)


def _fwd_alpha_twice(X, T, alpha, act_bits, use_hadamard):
    out = ho.forward(X, T, alpha, act_bits, use_hadamard)
    out["Y"] = ho.to_bf16(out["Y"].astype(np.float64) * float(alpha))
    return out


def _fwd_wrong_scale_rule(X, T, alpha, act_bits, use_hadamard):
    return ho.forward(X, T, alpha, 12 - act_bits, use_hadamard)


@pytest.mark.parametrize("fn", [_fwd_no_hadamard, _fwd_alpha_twice, _fwd_wrong_scale_rule])
def test_forward_mutants_caught(fn):
    _expect_fail(pins.check_forward, fn)
