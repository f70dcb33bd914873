"""ctypes binding of libhbl.so (C ABI declared in include/hbl.h).

Argument marshalling only: every step of the forward runs in the library's
CUDA kernels. Pointer arguments accept a torch tensor (its data_ptr) or an
integer address; ``stream`` defaults to torch's current CUDA stream. Each call
raises ``HblError`` when the library returns a status other than HBL_OK.
"""
from __future__ import annotations

import ctypes
import os

_SO = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libhbl.so")
_LIB = None

STATUS = {0: "HBL_OK", 1: "HBL_ERR_INVALID_ARG", 2: "HBL_ERR_SHAPE", 3: "HBL_ERR_CUDA",
          4: "HBL_ERR_ALLOC", 5: "HBL_ERR_TIMEOUT", 6: "HBL_ERR_UNSUPPORTED", 7: "HBL_ERR_WORKSPACE"}

# (name, restype, argtypes) for every entry point of include/hbl.h
_P, _I, _Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
SIGNATURES = [
    ("hbl_status_string", ctypes.c_char_p, [_I]),
    ("hbl_version", _I, []),
    ("hbl_packed_bytes", _Z, [_I, _I]),
    ("hbl_pack_weights", _I, [_P, _I, _I, _P, _P, _P]),
    ("hbl_unpack_weights", _I, [_P, _I, _I, _P, _P]),
    ("hbl_workspace_bytes", _Z, [_I, _I, _I]),
    ("hbl_forward_ws", _I, [_P, _I, _I, _I, _P, _P, _I, _I, _P, _P, _Z, _P]),
    ("hbl_forward", _I, [_P, _I, _I, _I, _P, _P, _I, _I, _P, _P]),
    ("hbl_forward_noalloc", _I, [_P, _I, _I, _I, _P, _P, _I, _I, _P, _P]),
    ("hbl_hadamard_f32", _I, [_P, _I, _I, _P, _P]),
    ("hbl_quantize", _I, [_P, _I, _I, _I, _I, _P, _P, _P, _P]),
    ("hbl_gemm_codes", _I, [_P, _I, _I, _I, _P, _P, _P]),
    ("hbl_forward_ln_ws", _I, [_P, _I, _I, _I, _P, _P, _P, _I, _I, _P, _P, _Z, _P]),
    ("hbl_quantize_ln", _I, [_P, _I, _I, _P, _I, _I, _P, _P, _P, _P]),
    ("hbl_pack_weights_rotated", _I, [_P, _I, _I, _P, _P, _P, _P]),
    ("hbl_hadamard_backward_f32", _I, [_P, _I, _I, _P, _P]),
    ("hbl_quantize_qkv", _I, [_P, _I, _I, _I, _I, _I, _P, _P, _P]),
    ("hbl_selftest_wait_timeout", _I, [_I, _P, _P]),
    ("hbl_get_device_error", _I, [_P]),
    ("hbl_set_gemm_path", _I, [_I]),
    ("hbl_profile_enable", _I, [_I]),
    ("hbl_profile_count", _I, []),
    ("hbl_profile_get", _I, [_I, ctypes.c_char_p, _I, ctypes.POINTER(_I), ctypes.POINTER(ctypes.c_double)]),
]


class HblError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


def lib():
    """Load libhbl.so (built in-tree); fails loudly when it is missing."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(_SO):
            raise ImportError(f"{_SO} is missing: build it with `python -m hadamard_bit_quant_b200.build`")
        L = ctypes.CDLL(_SO)
        for name, res, args in SIGNATURES:
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _LIB = L
    return _LIB


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(st: int, where: str) -> int:
    if st != 0:
        raise HblError(st, where)
    return st


def hbl_status_string(status: int) -> str:
    return lib().hbl_status_string(status).decode()


def hbl_version() -> int:
    return lib().hbl_version()


def hbl_packed_bytes(N: int, K: int) -> int:
    return lib().hbl_packed_bytes(N, K)


def hbl_workspace_bytes(M: int, K: int, N: int) -> int:
    return lib().hbl_workspace_bytes(M, K, N)


def hbl_pack_weights(W, N, K, Wpk, wscale, stream=None):
    return _check(lib().hbl_pack_weights(_ptr(W), N, K, _ptr(Wpk), _ptr(wscale), _stream(stream)),
                  "hbl_pack_weights")


def hbl_unpack_weights(Wpk, N, K, T, stream=None):
    return _check(lib().hbl_unpack_weights(_ptr(Wpk), N, K, _ptr(T), _stream(stream)), "hbl_unpack_weights")


def hbl_forward_ws(X, M, K, N, Wpk, wscale, act_bits, use_hadamard, Y, ws, ws_bytes, stream=None):
    return _check(lib().hbl_forward_ws(_ptr(X), M, K, N, _ptr(Wpk), _ptr(wscale), act_bits, use_hadamard,
                                       _ptr(Y), _ptr(ws), ws_bytes, _stream(stream)), "hbl_forward_ws")


def hbl_forward(X, M, K, N, Wpk, wscale, act_bits, use_hadamard, Y, stream=None):
    return _check(lib().hbl_forward(_ptr(X), M, K, N, _ptr(Wpk), _ptr(wscale), act_bits, use_hadamard,
                                    _ptr(Y), _stream(stream)), "hbl_forward")


def hbl_forward_noalloc(X, M, K, N, Wpk, wscale, act_bits, use_hadamard, Y, stream=None):
    """Forward with the library's fixed 8 MiB device workspace: no allocation (see include/hbl.h)."""
    return _check(lib().hbl_forward_noalloc(_ptr(X), M, K, N, _ptr(Wpk), _ptr(wscale), act_bits, use_hadamard,
                                            _ptr(Y), _stream(stream)), "hbl_forward_noalloc")


def hbl_hadamard_f32(X, M, K, Xr, stream=None):
    return _check(lib().hbl_hadamard_f32(_ptr(X), M, K, _ptr(Xr), _stream(stream)), "hbl_hadamard_f32")


def hbl_quantize(X, M, K, act_bits, use_hadamard, codes, scales, csum=None, stream=None):
    return _check(lib().hbl_quantize(_ptr(X), M, K, act_bits, use_hadamard, _ptr(codes), _ptr(scales),
                                     _ptr(csum), _stream(stream)), "hbl_quantize")


def hbl_gemm_codes(codes, M, K, N, Wpk, acc, stream=None):
    return _check(lib().hbl_gemm_codes(_ptr(codes), M, K, N, _ptr(Wpk), _ptr(acc), _stream(stream)),
                  "hbl_gemm_codes")


def hbl_forward_ln_ws(X, M, K, N, gain, Wpk, wscale, act_bits, use_hadamard, Y, ws, ws_bytes, stream=None):
    return _check(lib().hbl_forward_ln_ws(_ptr(X), M, K, N, _ptr(gain), _ptr(Wpk), _ptr(wscale), act_bits,
                                          use_hadamard, _ptr(Y), _ptr(ws), ws_bytes, _stream(stream)),
                  "hbl_forward_ln_ws")


def hbl_quantize_ln(X, M, K, gain, act_bits, use_hadamard, codes, scales, csum=None, stream=None):
    return _check(lib().hbl_quantize_ln(_ptr(X), M, K, _ptr(gain), act_bits, use_hadamard, _ptr(codes),
                                        _ptr(scales), _ptr(csum), _stream(stream)), "hbl_quantize_ln")


def hbl_pack_weights_rotated(W, N, K, Wpk, wscale, Wrot, stream=None):
    return _check(lib().hbl_pack_weights_rotated(_ptr(W), N, K, _ptr(Wpk), _ptr(wscale), _ptr(Wrot),
                                                 _stream(stream)), "hbl_pack_weights_rotated")


def hbl_hadamard_backward_f32(dXr, M, K, dX, stream=None):
    return _check(lib().hbl_hadamard_backward_f32(_ptr(dXr), M, K, _ptr(dX), _stream(stream)),
                  "hbl_hadamard_backward_f32")


def hbl_quantize_qkv(X, T, H, d, bits, bos_token, codes, gamma, stream=None):
    return _check(lib().hbl_quantize_qkv(_ptr(X), T, H, d, bits, bos_token, _ptr(codes), _ptr(gamma),
                                         _stream(stream)), "hbl_quantize_qkv")


def hbl_selftest_wait_timeout(timeout_us, gave_up=None, stream=None):
    return _check(lib().hbl_selftest_wait_timeout(int(timeout_us), _ptr(gave_up), _stream(stream)),
                  "hbl_selftest_wait_timeout")


def hbl_get_device_error(stream=None):
    return lib().hbl_get_device_error(_stream(stream))


def hbl_set_gemm_path(path: int) -> int:
    return _check(lib().hbl_set_gemm_path(int(path)), "hbl_set_gemm_path")


def hbl_profile_enable(enable: int) -> int:
    return _check(lib().hbl_profile_enable(int(enable)), "hbl_profile_enable")


def hbl_profile_count() -> int:
    return lib().hbl_profile_count()


def hbl_profile_get(i: int):
    """Returns (kernel name, launches, total device ms) of profile entry i."""
    name = ctypes.create_string_buffer(64)
    n = _I(0)
    ms = ctypes.c_double(0.0)
    _check(lib().hbl_profile_get(i, name, 64, ctypes.byref(n), ctypes.byref(ms)), "hbl_profile_get")
    return name.value.decode(), n.value, ms.value


def profile_table() -> dict:
    """All profile entries as {name: (launches, total_ms)}."""
    return {nm: (n, ms) for nm, n, ms in (hbl_profile_get(i) for i in range(hbl_profile_count()))}
