"""ctypes declarations of the C ABI in include/dory.h (marshalling only).

Loading fails loudly: there is no fallback implementation of any entry
point.
"""
import ctypes
import os
from ctypes import (POINTER, Structure, c_char_p, c_double, c_int, c_int64,
                    c_uint8, c_void_p)

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)),
                        "libdory.so")

DORY_OK = 0
ERRORS = {-1: "DORY_ERR_ARG", -2: "DORY_ERR_UNSUPPORTED", -3: "DORY_ERR_CACHE",
          -4: "DORY_ERR_CUDA", -5: "DORY_ERR_TIMEOUT", -6: "DORY_ERR_WORKSPACE",
          -7: "DORY_ERR_DEVICE"}
KV_MODES = {"per_loop": 0, "last_loop": 1}


class DoryConfig(Structure):
    _fields_ = [("d", c_int), ("n_q_heads", c_int), ("n_kv_heads", c_int),
                ("head_dim", c_int), ("ffn", c_int), ("vocab", c_int),
                ("n_in_blocks", c_int), ("n_rec_blocks", c_int),
                ("n_out_blocks", c_int), ("layer_types", POINTER(c_uint8)),
                ("swa_window", c_int), ("rope_theta_swa", c_double),
                ("rope_theta_full", c_double), ("wfmt", c_int)]


class DoryTensor(Structure):
    _fields_ = [("name", c_char_p), ("d_ptr", c_void_p), ("bytes", c_int64)]


class DoryKernelStat(Structure):
    _fields_ = [("name", ctypes.c_char * 32), ("launches", c_int64),
                ("total_ms", c_double), ("bytes", c_double),
                ("flops", c_double)]


_P = c_void_p
_I64P = POINTER(c_int64)
SIGNATURES = {
    "dory_init_weights": (c_int, [POINTER(DoryConfig), POINTER(DoryTensor),
                                  c_int, POINTER(c_void_p)]),
    "dory_kv_cache_bytes": (c_int, [_P, c_int, c_int, c_int, c_int, c_int,
                                    _I64P]),
    "dory_kv_cache_bind": (c_int, [_P, _P, c_int64, c_int, c_int, c_int, c_int,
                                   c_int, _P, POINTER(c_void_p)]),
    "dory_cache_length": (c_int, [_P, POINTER(c_int)]),
    "dory_cache_reset": (c_int, [_P, _P]),
    "dory_cache_fill_synthetic": (c_int, [_P, _P, c_int, ctypes.c_uint64, _P]),
    "dory_cache_copy_prefix": (c_int, [_P, _P, _P, c_int, c_int, _P]),
    "dory_workspace_bytes": (c_int, [_P, c_int, c_int, _I64P]),
    "dory_prefill": (c_int, [_P, _P, _P, c_int, c_int, c_int, c_int, c_int,
                             _P, _P, _P, c_int64, _P]),
    "dory_decode_step": (c_int, [_P, _P, _P, c_int, c_int, c_int, _P, _P, _P,
                                 c_int64, _P]),
    "dory_decode_step_static": (c_int, [_P, _P, _P, c_int, c_int, c_int, _P,
                                        _P, _P]),
    "dory_prefill_mixed": (c_int, [_P, _P, _P, c_int, c_int, _P, c_int, c_int,
                                   c_int, _P, _P, _P, c_int64, _P]),
    "dory_decode_step_mixed": (c_int, [_P, _P, _P, c_int, _P, c_int, c_int,
                                       _P, _P, _P, c_int64, _P]),
    "dory_debug_gemm_bf16": (c_int, [_P, c_int, _P, _P, c_int, c_int, c_int,
                                     _P]),
    "dory_debug_gemm_bf16_split": (c_int, [_P, c_int, _P, _P, c_int, c_int,
                                           c_int, c_int, POINTER(c_int), _P]),
    "dory_debug_dequant": (c_int, [_P, c_char_p, c_int, c_int, _P, _P]),
    "dory_debug_bounded_wait": (c_int, [_P, c_int, _P]),
    "dory_debug_gemv": (c_int, [_P, c_char_p, _P, c_int, _P, c_int,
                                POINTER(c_int), _P]),
    "dory_copy_state": (c_int, [_P, _P, c_int, c_int, c_int, _P, _P]),
    "dory_spec_workspace_bytes": (c_int, [_P, c_int, c_int, _I64P]),
    "dory_spec_decode_step": (c_int, [_P, _P, _P, c_int, c_int, c_int, c_int,
                                      ctypes.c_float, _P, _P, POINTER(c_int),
                                      _P, c_int64, _P]),
    "dory_debug_spec_accept": (c_int, [_P, _P, _P, _P, c_int, c_int, c_int,
                                       ctypes.c_float, _P, _P, _P]),
    "dory_sync_status": (c_int, [_P, _P]),
    "dory_profile_enable": (c_int, [_P, c_int]),
    "dory_profile_read": (c_int, [_P, POINTER(DoryKernelStat), c_int,
                                  POINTER(c_int), _P]),
    "dory_strerror": (c_char_p, [c_int]),
    "dory_cache_free": (None, [_P]),
    "dory_free": (None, [_P]),
}

_lib = None


def load():
    """Load libdory.so (built by looped_ngpt_b200.build) and declare it."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m looped_ngpt_b200.build` (needs nvcc)")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


class DoryError(RuntimeError):
    def __init__(self, fn, code):
        super().__init__(f"{fn} -> {code} ({ERRORS.get(code, '?')})")
        self.code = code


def check(fn, code):
    if code != DORY_OK:
        raise DoryError(fn, code)
    return code
