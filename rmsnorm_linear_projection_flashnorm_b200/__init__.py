"""Python binding of libflashnorm: the fused RMSNorm + linear projection in the
FlashNorm form for B200 (sm_100a).

Argument marshalling only.  Every step of the computation runs in the CUDA
kernels behind the C ABI declared in ``include/flashnorm.h``; the functions
here take torch tensors (or raw integer device addresses), pass their device
pointers and the stream handle through ctypes, and return the ``fn_status``
code.  There is no fallback: if ``libflashnorm.so`` has not been built, the
first call raises ``ImportError``.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

from .build import LIB_PATH, build  # noqa: F401

FN_OK = 0
FN_ERR_INVALID_ARG = 1
FN_ERR_UNSUPPORTED_SHAPE = 2
FN_ERR_ALIGNMENT = 3
FN_ERR_ALIAS = 4
FN_ERR_WORKSPACE = 5
FN_ERR_CUDA = 6
FN_ERR_TIMEOUT = 7
FN_ERR_UNSUPPORTED_DEVICE = 8

FN_W_BF16 = 0
FN_W_FP8_E4M3_B128 = 1
FN_W_MXFP8_E4M3 = 2

FN_DEBUG_WAIT_BUDGET_NS = 1
FN_DEBUG_WITHHOLD_ARRIVE = 2
FN_DEBUG_FORCE_PATH = 3
FN_DEBUG_PREFETCH = 4
FN_DEBUG_CLUSTER = 5
FN_DEBUG_DECODE_GROUPS = 6
FN_DEBUG_PAIR_TILE = 7

_vp, _i64, _f32, _sz, _int = ctypes.c_void_p, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t, ctypes.c_int

_SIGNATURES = {
    "fn_fold_weights": (_int, [_vp, _vp, _vp, _i64, _i64, _int, _vp, _vp, _vp]),
    "fn_workspace_size": (_sz, [_i64, _i64, _i64, _int, _int]),
    "fn_norm_proj": (_int, [_vp, _i64, _i64, _vp, _vp, _int, _i64, _f32, _vp, _vp, _sz, _vp]),
    "fn_norm_proj_swiglu": (_int, [_vp, _i64, _i64, _vp, _vp, _int, _i64, _f32, _vp, _vp, _sz, _vp]),
    "fn_norm_proj_swiglu_nvfp4": (_int, [_vp, _i64, _i64, _vp, _vp, _int, _i64, _f32, _vp, _vp, _vp, _vp, _sz,
                                         _vp]),
    "fn_norm_proj_swiglu_nvfp4_swizzled": (_int, [_vp, _i64, _i64, _vp, _vp, _int, _i64, _f32, _vp, _vp, _vp, _vp,
                                                  _sz, _vp]),
    "fn_norm_proj_partial": (_int, [_vp, _i64, _i64, _vp, _vp, _int, _i64, _vp, _vp, _sz, _vp]),
    "fn_post_scale": (_int, [_vp, _i64, _i64, _int, _i64, _f32, _vp, _vp]),
    "fn_norm_proj_static": (_int, [_vp, _i64, _i64, _vp, _vp, _int, _i64, _f32, _vp, _vp]),
    "fn_adaln_shift_bias": (_int, [_vp, _i64, _vp, _vp, _i64, _i64, _vp, _vp]),
    "fn_norm_proj_adaln": (_int, [_vp, _i64, _i64, _vp, _vp, _int, _i64, _int, _f32, _vp, _vp, _vp, _i64, _vp, _vp,
                                  _sz, _vp]),
    "fn_workspace_size_adaln": (_sz, [_i64, _i64, _int, _int]),
    "fn_query_device_status": (_int, [_vp, ctypes.POINTER(ctypes.c_uint), _vp]),
    "fn_query_static_status": (_int, [ctypes.POINTER(ctypes.c_uint), _vp]),
    "fn_rmsnorm": (_int, [_vp, _i64, _i64, _vp, _f32, _vp, _vp]),
    "fn_dequant_fp8": (_int, [_vp, _vp, _i64, _i64, _vp, _vp]),
    "fn_dequant_mxfp8": (_int, [_vp, _vp, _i64, _i64, _vp, _vp]),
    "fn_status_string": (ctypes.c_char_p, [_int]),
    "fn_version": (_int, []),
    "fn_kernel_launches": (ctypes.c_uint64, []),
    "fn_set_debug": (_int, [_int, _i64]),
}

_lib: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    """The loaded library; raises ImportError when it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m rmsnorm_linear_projection_flashnorm_b200.build` (nvcc, sm_100a)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(s) -> Optional[int]:
    if s is None:
        import torch
        if torch.cuda.is_available() and torch.cuda.is_initialized():
            return torch.cuda.current_stream().cuda_stream or None
        return None
    if isinstance(s, int):
        return s or None
    return s.cuda_stream or None


class FnError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {status_string(status)}")


def check(status: int, what: str = "flashnorm") -> None:
    if status != FN_OK:
        raise FnError(status, what)


def status_string(status: int) -> str:
    return lib().fn_status_string(status).decode()


def fn_version() -> int:
    return lib().fn_version()


def fn_kernel_launches() -> int:
    return lib().fn_kernel_launches()


def fn_set_debug(key: int, value: int) -> int:
    return lib().fn_set_debug(key, value)


def fn_fold_weights(W0, W1, g, d: int, N: int, out_type: int, Wp, scales=None, stream=None) -> int:
    return lib().fn_fold_weights(_ptr(W0), _ptr(W1), _ptr(g), d, N, out_type, _ptr(Wp), _ptr(scales),
                                 _stream(stream))


def fn_workspace_size(M: int, d: int, N: int, wt: int = FN_W_BF16, swiglu: int = 0) -> int:
    return lib().fn_workspace_size(M, d, N, wt, int(swiglu))


def fn_norm_proj(x, M: int, d: int, Wp, scales, wt: int, N: int, eps: float, y, workspace, ws_bytes: int,
                 stream=None) -> int:
    return lib().fn_norm_proj(_ptr(x), M, d, _ptr(Wp), _ptr(scales), wt, N, eps, _ptr(y), _ptr(workspace),
                              ws_bytes, _stream(stream))


def fn_norm_proj_swiglu(x, M: int, d: int, Wp, scales, wt: int, N: int, eps: float, out, workspace,
                        ws_bytes: int, stream=None) -> int:
    return lib().fn_norm_proj_swiglu(_ptr(x), M, d, _ptr(Wp), _ptr(scales), wt, N, eps, _ptr(out),
                                     _ptr(workspace), ws_bytes, _stream(stream))


def fn_norm_proj_swiglu_nvfp4(x, M: int, d: int, Wp, scales, wt: int, N: int, eps: float, global_scale, out_q,
                              out_sf, workspace, ws_bytes: int, stream=None) -> int:
    return lib().fn_norm_proj_swiglu_nvfp4(_ptr(x), M, d, _ptr(Wp), _ptr(scales), wt, N, eps, _ptr(global_scale),
                                           _ptr(out_q), _ptr(out_sf), _ptr(workspace), ws_bytes, _stream(stream))


def fn_norm_proj_partial(x, M: int, d: int, Wp, scales, wt: int, ncols: int, partial, workspace, ws_bytes: int,
                         stream=None) -> int:
    return lib().fn_norm_proj_partial(_ptr(x), M, d, _ptr(Wp), _ptr(scales), wt, ncols, _ptr(partial),
                                      _ptr(workspace), ws_bytes, _stream(stream))


def fn_post_scale(partial, M: int, N: int, swiglu: int, d_total: int, eps: float, y, stream=None) -> int:
    return lib().fn_post_scale(_ptr(partial), M, N, swiglu, d_total, eps, _ptr(y), _stream(stream))


def fn_norm_proj_static(x, M: int, d: int, Wp, scales, wt: int, N: int, eps: float, y, stream=None) -> int:
    return lib().fn_norm_proj_static(_ptr(x), M, d, _ptr(Wp), _ptr(scales), wt, N, eps, _ptr(y), _stream(stream))


def fn_query_device_status(workspace, stream=None):
    """Returns (status, raw status word)."""
    word = ctypes.c_uint(0)
    st = lib().fn_query_device_status(_ptr(workspace), ctypes.byref(word), _stream(stream))
    return st, word.value


def fn_query_static_status(stream=None):
    """Status of fn_norm_proj_static's scratch on the current device:
    (status, raw status word); the word is cleared."""
    word = ctypes.c_uint(0)
    st = lib().fn_query_static_status(ctypes.byref(word), _stream(stream))
    return st, word.value


def fn_rmsnorm(x, M: int, d: int, g, eps: float, h, stream=None) -> int:
    return lib().fn_rmsnorm(_ptr(x), M, d, _ptr(g), eps, _ptr(h), _stream(stream))


def fn_dequant_fp8(q, scales, d: int, ncols: int, W, stream=None) -> int:
    return lib().fn_dequant_fp8(_ptr(q), _ptr(scales), d, ncols, _ptr(W), _stream(stream))


def fn_dequant_mxfp8(q, scales, d: int, ncols: int, W, stream=None) -> int:
    return lib().fn_dequant_mxfp8(_ptr(q), _ptr(scales), d, ncols, _ptr(W), _stream(stream))


def fn_adaln_shift_bias(shift, n_cond: int, W0, W1, d: int, N: int, B, stream=None) -> int:
    return lib().fn_adaln_shift_bias(_ptr(shift), n_cond, _ptr(W0), _ptr(W1), d, N, _ptr(B), _stream(stream))


def fn_norm_proj_adaln(x, M: int, d: int, Wp, scales, wt: int, N: int, swiglu: int, eps: float, adaln_scale,
                       shift_bias, adaln_index, n_cond: int, y, workspace, ws_bytes: int, stream=None) -> int:
    return lib().fn_norm_proj_adaln(_ptr(x), M, d, _ptr(Wp), _ptr(scales), wt, N, int(swiglu), eps,
                                    _ptr(adaln_scale), _ptr(shift_bias), _ptr(adaln_index), n_cond, _ptr(y),
                                    _ptr(workspace), ws_bytes, _stream(stream))


def fn_workspace_size_adaln(d: int, N: int, wt: int = FN_W_BF16, swiglu: int = 0) -> int:
    return lib().fn_workspace_size_adaln(d, N, wt, int(swiglu))


def fn_norm_proj_swiglu_nvfp4_swizzled(x, M: int, d: int, Wp, scales, wt: int, N: int, eps: float, global_scale,
                                       out_q, out_sf, workspace, ws_bytes: int, stream=None) -> int:
    return lib().fn_norm_proj_swiglu_nvfp4_swizzled(_ptr(x), M, d, _ptr(Wp), _ptr(scales), wt, N, eps,
                                                    _ptr(global_scale), _ptr(out_q), _ptr(out_sf), _ptr(workspace),
                                                    ws_bytes, _stream(stream))
