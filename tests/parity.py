"""Comparison rules between the CUDA path and the oracle (numeric criteria of the
H-BitLinear forward).

* Hadamard: per token, max |X_r,gpu - X_r,ref| <= 1e-5 * max |X_r,ref| (fp32).
* Codes: identical except +-1 where the oracle flags a near tie, and at most
  1e-4 of all codes may differ (at least one flip allowed in cases with fewer
  than 1e4 codes, where a rate of 1e-4 cannot be resolved). Scales agree to 1e-5 relative.
* Integer accumulators: bit-exact given the same codes.
* Y (bf16): |Y_gpu - Y_ref| <= 1e-2 |Y_ref| + s[m] * alpha * (differing codes
  in row m) -- the second term bounds what a tie-flipped code can change.
"""
import numpy as np

HAD_RTOL = 1e-5
SCALE_RTOL = 1e-5
CODE_DIFF_FRAC = 1e-4
Y_RTOL = 1e-2


def check_hadamard(xr_gpu, xr_ref):
    xr_gpu = np.asarray(xr_gpu, np.float64)
    err = np.max(np.abs(xr_gpu - xr_ref), axis=1)
    ref = np.max(np.abs(xr_ref), axis=1)
    bad = err > HAD_RTOL * ref + 1e-30
    assert not bad.any(), f"Hadamard mismatch in {bad.sum()} tokens, worst rel {np.max(err / np.maximum(ref, 1e-30)):.3e}"


def check_codes(codes_gpu, codes_ref, tie_ref, scales_gpu, scales_ref):
    cg = np.asarray(codes_gpu, np.int64)
    cr = np.asarray(codes_ref, np.int64)
    diff = cg != cr
    assert np.all(np.abs(cg - cr)[diff] == 1), "a code differs by more than 1"
    assert np.all(tie_ref[diff]), f"{int((diff & ~tie_ref).sum())} codes differ away from a near tie"
    # a rate of 1e-4 cannot be resolved below 1e4 codes: small cases may flip one tie
    allowed = max(1, int(CODE_DIFF_FRAC * diff.size))
    assert diff.sum() <= allowed, f"too many tie flips: {int(diff.sum())} of {diff.size}"
    sg = np.asarray(scales_gpu, np.float64)
    assert np.all(np.abs(sg - scales_ref) <= SCALE_RTOL * np.abs(scales_ref) + 1e-30), "scales differ"
    return diff


def check_y(y_gpu, y_ref, s_ref, alpha, ndiff_rows):
    yg = np.asarray(y_gpu, np.float64)
    yr = np.asarray(y_ref, np.float64)
    bound = Y_RTOL * np.abs(yr) + (np.asarray(s_ref, np.float64) * float(alpha) * ndiff_rows * 1.01)[:, None]
    err = np.abs(yg - yr)
    bad = err > bound + 1e-30
    assert not bad.any(), f"Y mismatch at {int(bad.sum())} of {bad.size}, worst excess {np.max(err - bound):.3e}"
