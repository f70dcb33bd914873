"""Plain CPU oracle for the H-BitLinear forward of BitNet v2.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference leg of ``bench.py`` may import or call this
module. The product path (``hadamard_bit_quant_b200``) never imports it, and
it imports nothing from the product path: the two share no code. Inputs come
from ``hadamard_bit_quant_b200.inputs`` (random draws only) and are passed in
as arrays.

Source: "BitNet v2: Native 4-bit Activations with Hadamard Transformation for
1-bit LLMs", architecture walkthrough page, section 3.4 ("Detailed,
Sentence-Based Technical Breakdown"):
  * Weight quantiser, Eq. 1-2 (sub-section "Weight Quantization").
  * INT8 / INT4 activation quantisers, Eq. 7 / Eq. 8 (sub-section
    "Activation Quantization").
  * Hadamard matrix and transform, Eq. 3-6 (sub-section "The Hadamard
    Transformation", "Definition and Structure").
  * H-BitLinear composite, Eq. 9 (sub-section "H-BitLinear: The Composite
    Layer").

Everything here is the plain definition: an explicit K x K Hadamard matrix
built by the recursion of Eq. 6 (O(K^2) per token), scalar quantisers applied
element by element in fp64, and an exact integer GEMM. No fast transform, no
blocking, no fusion.

Readings where the pages leave a step open (each is a choice):
  * EPS = 1e-5, in the denominator only; the dequant factors are alpha,
    gamma/127 and beta/sqrt(7) exactly as printed.
  * round() in RoundClip is round-half-to-even.
  * The Hadamard normalisation is 2^(-m/2) overall (1/sqrt(2) per level of
    the recursion), Sylvester (natural) order.
  * alpha is the exact mean of |W| over the whole tensor: the exact sum
    rounded once to fp64, divided by the element count in fp64, rounded to
    fp32. The ternary decision W / (alpha + eps) is taken in fp32, the
    precision the kernel uses for it.
  * act_bits selects the scale rule (absmax/127 for INT8, absmean/sqrt(7) for
    INT4) whether or not the Hadamard transform is applied.
  * The LN inside Eq. 9 is not part of this forward (the layer input is
    taken as already normalised); see ``rmsnorm`` for the separate prologue.
"""
from __future__ import annotations

import math
from fractions import Fraction
from functools import lru_cache

import numpy as np

EPS = 1e-5
SQRT7 = math.sqrt(7.0)

INT8_RANGE = (-128, 127)   # Eq. 7 clip bounds
INT4_RANGE = (-8, 7)       # Eq. 8 clip bounds
TERN_RANGE = (-1, 1)       # Eq. 1 clip bounds

# Codes whose pre-rounding value lies this close to a half-integer are "near
# ties": a kernel that computes the same value in fp32 may round them the
# other way.
TIE_WINDOW = 1e-3


# ---------------------------------------------------------------------------
# Eq. 2: RoundClip
# ---------------------------------------------------------------------------
def round_clip(x, a, b):
    """RoundClip(x, a, b) = min(max(round(x), a), b)  [section 3.4, Eq. 2].

    round() is round-half-to-even (numpy ``rint``).
    """
    return np.minimum(np.maximum(np.rint(x), a), b)


# ---------------------------------------------------------------------------
# Eq. 1-2: ternary weight quantiser
# ---------------------------------------------------------------------------
def exact_sum_rounded(values) -> float:
    """Exact sum of an array of fp32-representable numbers, rounded once to fp64.

    Each value is split exactly into an integer significand (< 2^24) and a
    power of two; significands are summed per exponent (exact in fp64 while
    the count stays below 2^29) and the per-exponent totals are combined as
    exact rationals. Python's int/int division rounds correctly, so the
    result equals ``math.fsum`` of the same numbers.
    """
    a = np.asarray(values, dtype=np.float64).ravel()
    if a.size == 0:
        return 0.0
    assert a.size < (1 << 29), "per-exponent fp64 sums would stop being exact"
    m, e = np.frexp(a)
    mi = np.rint(m * 2.0 ** 24)
    assert np.array_equal(mi * 2.0 ** -24, m), "inputs must be fp32-representable"
    e = e.astype(np.int64) - 24
    emin = int(e.min())
    sums = np.bincount(e - emin, weights=mi)
    total = Fraction(0)
    for k, s in enumerate(sums):
        if s != 0.0:
            total += Fraction(int(s)) * Fraction(2) ** (k + emin)
    return float(total)


def weight_scale(W) -> np.float32:
    """alpha = mean(|W|) over the whole tensor  [section 3.4, Eq. 1].

    Exact sum rounded to fp64, divided by the element count in fp64, then
    rounded to fp32 (the scalar stored beside the packed weights).
    """
    w = np.asarray(W, dtype=np.float32)
    s = exact_sum_rounded(np.abs(w.astype(np.float64)))
    return np.float32(s / w.size)


def ternarize(W, alpha) -> np.ndarray:
    """Ternary codes RoundClip(W / (alpha + eps), -1, 1)  [section 3.4, Eq. 1].

    The division is the fp32 one (IEEE, correctly rounded), the same
    precision the kernel uses to take this decision. Returns int8 in {-1,0,1}.
    """
    w = np.asarray(W, dtype=np.float32)
    den = np.float32(alpha) + np.float32(EPS)          # fp32 add
    q = w / den                                        # fp32 divide
    return round_clip(q, *TERN_RANGE).astype(np.int8)


def weight_quant(W):
    """Q_w(W) as (alpha, codes): the dequantised weight is alpha * codes [Eq. 1]."""
    alpha = weight_scale(W)
    return alpha, ternarize(W, alpha)


# ---------------------------------------------------------------------------
# Eq. 3-6: Hadamard
# ---------------------------------------------------------------------------
def _log2_exact(n: int) -> int:
    m = int(n).bit_length() - 1
    if n < 1 or (1 << m) != n:
        raise ValueError(f"Hadamard size must be a power of two, got {n}")
    return m


@lru_cache(maxsize=2)
def hadamard_matrix(n: int) -> np.ndarray:
    """H_m for n = 2^m by the recursion of Eq. 6, in fp64.

    H_0 = (1); H_m = (1/sqrt 2) [[H_{m-1}, H_{m-1}], [H_{m-1}, -H_{m-1}]].
    The signs are built by the recursion without scaling and the m factors of
    1/sqrt(2) are applied once as 2^(-m/2).
    """
    m = _log2_exact(n)
    S = np.ones((1, 1), dtype=np.float64)
    for _ in range(m):
        S = np.block([[S, S], [S, -S]])
    S *= 2.0 ** (-m / 2.0)
    S.setflags(write=False)
    return S


def hadamard(X) -> np.ndarray:
    """Hadamard(x) = H_m x for every token (row) of X  [section 3.4, Eq. 3-5].

    Explicit O(K^2) matrix-vector products in fp64. X is M x K.
    """
    X = np.asarray(X, dtype=np.float64)
    H = hadamard_matrix(X.shape[1])
    return X @ H.T


# ---------------------------------------------------------------------------
# Eq. 7-8: per-token activation quantisers
# ---------------------------------------------------------------------------
def _near_ties(v, lo, hi):
    """Where |frac(v) - 1/2| < TIE_WINDOW and the two neighbours clip to different codes."""
    f = np.floor(v)
    near = np.abs((v - f) - 0.5) < TIE_WINDOW
    differ = np.clip(f, lo, hi) != np.clip(f + 1.0, lo, hi)
    return near & differ


def quantize_int8(Xr):
    """Q_INT8: gamma = max|x| per token; codes RoundClip(127/(gamma+eps) x, -128, 127)  [Eq. 7].

    Returns (codes int8 M x K, scale gamma/127 fp64 M, near-tie map M x K).
    """
    Xr = np.asarray(Xr, dtype=np.float64)
    gamma = np.max(np.abs(Xr), axis=1)
    v = (127.0 / (gamma + EPS))[:, None] * Xr
    codes = round_clip(v, *INT8_RANGE).astype(np.int8)
    return codes, gamma / 127.0, _near_ties(v, *INT8_RANGE)


def quantize_int4(Xr):
    """Q_INT4: beta = mean|x| per token; codes RoundClip(sqrt7/(beta+eps) x, -8, 7)  [Eq. 8].

    Returns (codes int8 M x K, scale beta/sqrt(7) fp64 M, near-tie map M x K).
    """
    Xr = np.asarray(Xr, dtype=np.float64)
    beta = np.mean(np.abs(Xr), axis=1)
    v = (SQRT7 / (beta + EPS))[:, None] * Xr
    codes = round_clip(v, *INT4_RANGE).astype(np.int8)
    return codes, beta / SQRT7, _near_ties(v, *INT4_RANGE)


def quantize_act(Xr, act_bits: int):
    """Per-token activation quantiser chosen by act_bits (8 -> Eq. 7, 4 -> Eq. 8)."""
    if act_bits == 8:
        return quantize_int8(Xr)
    if act_bits == 4:
        return quantize_int4(Xr)
    raise ValueError(f"act_bits must be 4 or 8, got {act_bits}")


# ---------------------------------------------------------------------------
# Eq. 9: the quantised product and its dequantisation
# ---------------------------------------------------------------------------
def gemm_int(codes, T) -> np.ndarray:
    """acc[m, n] = sum_k codes[m, k] * T[n, k], exactly, as int64.

    Computed with an fp64 matrix product, which is exact here: every product
    and every partial sum is an integer of magnitude <= 128 * K < 2^53.
    """
    c = np.asarray(codes, dtype=np.float64)
    t = np.asarray(T, dtype=np.float64)
    K = c.shape[1]
    assert t.shape[1] == K
    assert 128 * K < 2 ** 53
    assert np.all(np.abs(t) <= 1) and np.all(np.abs(c) <= 128)
    return (c @ t.T).astype(np.int64)


def to_bf16(y) -> np.ndarray:
    """Round fp64 values to the nearest bf16 (8 significant bits), ties to even.

    Returned as fp32 values (every bf16 is exactly representable in fp32).
    bf16 subnormals (below 2^-126) keep a fixed spacing of 2^-133.
    """
    y = np.asarray(y, dtype=np.float64)
    assert np.all(np.isfinite(y))
    _, e = np.frexp(y)
    e = np.maximum(e, -125)
    q = np.rint(np.ldexp(y, 8 - e))
    r = np.ldexp(q, e - 8)
    assert np.all(np.abs(r) <= 3.3895313892515355e38)
    return r.astype(np.float32)


def dequant(acc, s, alpha) -> np.ndarray:
    """Y = bf16(acc * s[m] * alpha): activation scale times weight scale  [Eq. 1, 7, 8, 9]."""
    y = np.asarray(acc, dtype=np.float64) * np.asarray(s, np.float64)[:, None] \
        * float(np.float32(alpha))
    return to_bf16(y)


def forward(X, T, alpha, act_bits: int, use_hadamard: int) -> dict:
    """H-BitLinear forward Y = Q_w(W) . Q_INT8/4(X_r), X_r = Hadamard(X)  [Eq. 9].

    X: M x K activations (values of the bf16 input, any float dtype).
    T, alpha: ternary codes (N x K) and weight scale from ``weight_quant``.
    Returns a dict with Xr (fp64), codes, s, tie, acc (int64) and Y (bf16
    values as fp32).
    """
    X = np.asarray(X, dtype=np.float64)
    Xr = hadamard(X) if use_hadamard else X.copy()
    codes, s, tie = quantize_act(Xr, act_bits)
    acc = gemm_int(codes, T)
    Y = dequant(acc, s, alpha)
    return dict(Xr=Xr, codes=codes, s=s, tie=tie, acc=acc, Y=Y)


def forward_rows(X, T, alpha, act_bits: int, use_hadamard: int, rows, cols=None) -> dict:
    """The same forward restricted to some tokens (rows) and output features (cols).

    Each token is independent, so sampled rows of a large problem are exact.
    """
    X = np.asarray(X, dtype=np.float64)[np.asarray(rows)]
    T = np.asarray(T)
    if cols is not None:
        T = T[np.asarray(cols)]
    return forward(X, T, alpha, act_bits, use_hadamard)


# ---------------------------------------------------------------------------
# Beyond the forward of Eq. 9 without LN: the LN prologue, the
# weight-and-activation rotation variant, the Hadamard backward and the
# post-RoPE QKV quantiser.
# ---------------------------------------------------------------------------
RMS_EPS = 1e-5   # reading: the pages give no epsilon for the RMSNorm; the quantisers' 1e-5 is reused


def rmsnorm(X, gain=None):
    """LN of Eq. 9, "RMS normalization in practice" (section 3.4, "H-BitLinear:
    The Composite Layer"): x / sqrt(mean(x^2) + eps), times an optional
    per-channel gain. fp64."""
    X = np.asarray(X, dtype=np.float64)
    r = 1.0 / np.sqrt(np.mean(X * X, axis=1) + RMS_EPS)
    Y = X * r[:, None]
    if gain is not None:
        Y = Y * np.asarray(gain, dtype=np.float64)[None, :]
    return Y


def forward_ln(X, gain, T, alpha, act_bits: int, use_hadamard: int) -> dict:
    """H-BitLinear with its LN: X_r = Hadamard(LN(X)), Y = Q_w(W) . Q(X_r)  [Eq. 9]."""
    return forward(rmsnorm(X, gain), T, alpha, act_bits, use_hadamard)


def rotate_weights(W) -> np.ndarray:
    """W H^T of the weight-and-activation rotation variant (section 3.4, ablation
    of Table 5): every weight row w becomes H w. Returned as fp32 (the precision
    the ternary decision is taken in)."""
    W = np.asarray(W, dtype=np.float64)
    H = hadamard_matrix(W.shape[1])
    return (W @ H.T).astype(np.float32)


def rotated_weight_quant(W):
    """Q_w(W H^T): alpha and ternary codes of the rotated weights  [Eq. 1 on W H^T]."""
    return weight_quant(rotate_weights(W))


def hadamard_backward(G) -> np.ndarray:
    """dL/dX = H^T dL/dX_r for every token (row) of G  [section 3.4, Eq. 10].

    Written with the transpose, as in the chain rule; H is symmetric, so this
    equals another forward transform. fp64.
    """
    G = np.asarray(G, dtype=np.float64)
    H = hadamard_matrix(G.shape[1])
    return G @ H           # row form of H^T g


def quantize_qkv(Xh, bits: int, bos_rows=()):
    """Post-RoPE QKV quantiser (section 3.4, "QKV Attention Quantization"):
    unsigned integers from the absmax of each head vector.

    Reading: gamma = max|x| over one head of one token; the interval
    [-gamma, gamma] maps onto [0, 2^b - 1]:
        u = RoundClip((2^b - 1)/2 * (x / (gamma + eps) + 1), 0, 2^b - 1),
    dequantised as (2u / (2^b - 1) - 1) * gamma. Rows listed in bos_rows (the
    BOS token's heads) use 8 bits whatever `bits` is.
    Xh: (rows, d) head vectors. Returns (codes uint8, gamma fp64, bits per row,
    near-tie map).
    """
    Xh = np.asarray(Xh, dtype=np.float64)
    b = np.full(Xh.shape[0], int(bits))
    b[list(bos_rows)] = 8
    top = (2.0 ** b - 1.0)[:, None]
    gamma = np.max(np.abs(Xh), axis=1)
    v = 0.5 * top * (Xh / (gamma + EPS)[:, None] + 1.0)
    u = np.minimum(np.maximum(np.rint(v), 0.0), top)
    f = np.floor(v)
    near = np.abs((v - f) - 0.5) < TIE_WINDOW
    differ = np.minimum(np.maximum(f, 0.0), top) != np.minimum(np.maximum(f + 1.0, 0.0), top)
    return u.astype(np.uint8), gamma, b, near & differ


def dequantize_qkv(u, gamma, b):
    top = (2.0 ** np.asarray(b, dtype=np.float64) - 1.0)[:, None]
    return (2.0 * np.asarray(u, dtype=np.float64) / top - 1.0) * np.asarray(gamma, np.float64)[:, None]
