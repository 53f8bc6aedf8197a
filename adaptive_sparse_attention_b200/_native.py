"""ctypes declarations of libentmax_attn.so (the C ABI of include/entmax_attn.h).

The shared library is built in-tree by ``adaptive_sparse_attention_b200.build``.  There is no
fallback: if it is missing or does not load, every entry point raises.
"""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libentmax_attn.so")

OK, EINVAL, EALIGN, ECUDA, ETIMEOUT, ENOMEM = 0, 1, 2, 3, 4, 5
FP32, BF16 = 0, 1
FLAG_CUDA_CORES = 1
FLAG_ALL_FALLBACK = 2
FLAG_NO_BLOCK_MASK = 8  # ENTMAX_ATTN_FLAG_NO_BLOCK_MASK
FLAG_TEST_STALL = 4  # test hook of the bounded device waits (ENTMAX_ATTN_FLAG_TEST_STALL)
FLAG_SUPPORT = 16  # output from the supports the tau pass records (ENTMAX_ATTN_FLAG_SUPPORT)
FLAG_OUT_FP32 = 32  # fp32 out for bf16 inputs (ENTMAX_ATTN_FLAG_OUT_FP32)
NOALLOC_SCRATCH_BYTES = 16 << 20  # ENTMAX_ATTN_NOALLOC_SCRATCH_BYTES

_c_int, _c_float, _c_size_t, _vp = ctypes.c_int, ctypes.c_float, ctypes.c_size_t, ctypes.c_void_p
_c_uint = ctypes.c_uint

# name -> (restype, argtypes); kept in the order of include/entmax_attn.h
SIGNATURES = {
    "entmax_attn_fwd": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int,
                                 _c_int, _c_float, _c_int, _c_int, _vp, _c_int, _vp]),
    "entmax_attn_fwd_no_block_mask": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int,
                                               _c_int, _c_int, _c_float, _c_int, _c_int, _vp,
                                               _c_int, _vp]),
    "entmax_attn_mask_words": (_c_size_t, [_c_int, _c_int, _c_int, _c_int]),
    "entmax_attn_mask_layout": (_c_int, [_c_int, _c_int, _c_int, _c_int,
                                         ctypes.POINTER(_c_int), ctypes.POINTER(_c_int)]),
    "entmax_attn_workspace_bytes": (_c_size_t, [_c_int, _c_int, _c_int, _c_int]),
    "entmax_attn_workspace_min_bytes": (_c_size_t, [_c_int, _c_int, _c_int, _c_int]),
    "entmax_attn_tau_pass": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_size_t, _c_int, _c_int, _c_int,
                                      _c_int, _c_int, _c_float, _c_int, _c_int, _vp, _c_int,
                                      _c_uint, _vp]),
    "entmax_attn_screen_bytes": (_c_size_t, [_c_int, _c_int, _c_int, _c_int, _c_int]),
    "entmax_attn_tau_pass_screened": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_size_t, _vp, _c_size_t,
                                               _c_int, _c_int, _c_int, _c_int, _c_int, _c_float,
                                               _c_int, _c_int, _vp, _c_int, _c_uint, _vp]),
    "entmax_attn_out_pass": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_size_t, _vp, _c_int, _c_int,
                                      _c_int, _c_int, _c_int, _c_float, _c_int, _vp, _c_int,
                                      _c_uint, _vp]),
    "entmax_attn_bwd": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _c_size_t, _vp, _vp, _vp, _vp,
                                 _c_int, _c_int, _c_int, _c_int, _c_int, _c_float, _c_int, _vp,
                                 _c_int, _c_uint, _vp]),
    "entmax_attn_fallback_tiles": (_c_int, [_vp, _vp]),
    "entmax_attn_rows": (_c_int, [_vp, ctypes.c_longlong, _vp, ctypes.c_longlong, _vp, _c_int,
                                  _c_int, _c_float, _c_int, _c_int, _vp]),
    "entmax_attn_route_chunks": (_c_int, [_vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int,
                                          _c_int, _c_int, _c_float, _c_int, _c_int, _c_int,
                                          _c_float, _c_int, _vp]),
    "entmax_attn_status": (_c_int, [_vp]),
    "entmax_attn_release_workspaces": (None, []),
    "entmax_attn_fwd_noalloc": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int,
                                         _c_int, _c_int, _c_float, _c_int, _c_int, _vp, _c_int,
                                         _vp]),
    "entmax_attn_fwd_host": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int,
                                      _c_int, _c_int, _c_float, _c_int, _c_int, _vp, _c_int,
                                      _vp]),
    "entmax_attn_strerror": (ctypes.c_char_p, [_c_int]),
    "entmax_attn_last_cuda_error": (ctypes.c_char_p, []),
}

_lib = None


class NativeLibraryError(RuntimeError):
    pass


def lib():
    """The loaded library (loaded once).  Raises NativeLibraryError if it is not built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise NativeLibraryError(
            f"{LIB_PATH} is missing; build it with `python -m adaptive_sparse_attention_b200.build`")
    try:
        h = ctypes.CDLL(LIB_PATH)
    except OSError as e:
        raise NativeLibraryError(f"cannot load {LIB_PATH}: {e}") from e
    for name, (res, args) in SIGNATURES.items():
        f = getattr(h, name)
        f.restype = res
        f.argtypes = args
    _lib = h
    return h


class EntmaxAttnError(RuntimeError):
    def __init__(self, code: int, where: str):
        msg = lib().entmax_attn_strerror(code).decode()
        if code == ECUDA:
            msg += ": " + lib().entmax_attn_last_cuda_error().decode()
        super().__init__(f"{where} failed with code {code} ({msg})")
        self.code = code


def check(code: int, where: str) -> None:
    if code != OK:
        raise EntmaxAttnError(code, where)
