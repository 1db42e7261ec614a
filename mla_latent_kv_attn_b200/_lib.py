"""ctypes loader for libmla_b200.so (the C ABI declared in include/mla.h).

Loading never falls back to anything: if the library is missing or lacks a symbol the import
of the op raises, naming the build command.
"""
from __future__ import annotations

import ctypes
import os
import threading
from ctypes import c_float, c_int32, c_size_t, c_void_p, POINTER

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmla_b200.so")
# the same library built with MLA_DEBUG (device-side contract checks; see include/mla.h)
DEBUG_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmla_b200_debug.so")

# mla_status codes (include/mla.h)
MLA_OK = 0
MLA_ERR_INVALID_ARG = 1
MLA_ERR_UNSUPPORTED = 2
MLA_ERR_ALIGNMENT = 3
MLA_ERR_CUDA = 4
MLA_ERR_DEVICE_TIMEOUT = 5
MLA_ERR_WORKSPACE = 6
MLA_ERR_DEVICE_CHECK = 7

MLA_BF16 = 0
MLA_FP32 = 1
MLA_PATH_AUTO = 0
MLA_PATH_SIMT = 1
MLA_PATH_TC_SINGLE = 2
MLA_PATH_TC_PAIR = 3

MLA_PROJECT = 1
MLA_APPEND = 2
MLA_PROJECT_AND_APPEND = 3


class MLAConfigC(ctypes.Structure):
    """Mirror of struct mla_config."""

    _fields_ = [
        ("d_model", c_int32), ("n_heads", c_int32), ("d_head", c_int32), ("d_c", c_int32),
        ("d_rope", c_int32), ("d_cq", c_int32), ("rope_pairs_t", c_int32),
        ("rope_pairs_h", c_int32), ("rope_pairs_w", c_int32), ("rope_base", c_float),
        ("softmax_scale", c_float), ("frame_h", c_int32), ("frame_w", c_int32),
        ("chunk_frames", c_int32), ("window_frames", c_int32), ("batch", c_int32),
        ("dtype", c_int32), ("kernel_path", c_int32),
    ]


_P = c_void_p
_I32P = POINTER(c_int32)
_CFG = POINTER(MLAConfigC)

# name -> (restype, argtypes)
SIGNATURES = {
    "mla_status_string": (ctypes.c_char_p, [c_int32]),
    "mla_last_error": (ctypes.c_char_p, []),
    "mla_abi_version": (c_int32, []),
    "mla_config_check": (c_int32, [_CFG]),
    "mla_cache_append": (c_int32, [_CFG, _P, _P, _P, _P, _P, c_int32, c_int32, _P]),
    "mla_rope3d": (c_int32, [_CFG, _P, c_int32, c_int32, c_int32, c_int32, c_int32, c_int32, _P,
                             c_int32, c_int32, _P]),
    "mla_key_positions": (c_int32, [_CFG, _P, c_int32, c_int32, _P, _P]),
    "mla_compose_query_weights": (c_int32, [_CFG, _P, _P, _P, _P, _P]),
    "mla_query_proj": (c_int32, [_CFG, _P, _P, _P, _P, _P, c_int32, _P]),
    "mla_project_chunk": (c_int32, [_CFG, _P, _P, _P, _P, _P, _P, c_int32, _P]),
    "mla_project_latents": (c_int32, [_CFG, _P, _P, _P, _P, _P]),
    "mla_project_latents_rotated": (c_int32, [_CFG, _P, _P, _P, _P, _P, _P, c_int32, c_int32,
                                              c_int32, _P, c_size_t, _P, _P]),
    "mla_attention_fwd_from_cq_prerotated": (c_int32, [_CFG, _P, _P, _P, _P, _P, c_int32,
                                                       c_int32, _P, _P, _P, _P, c_size_t, _P,
                                                       _P]),
    "mla_attention_fwd_from_cq": (c_int32, [_CFG, _P, _P, _P, _P, _P, c_int32, c_int32, _P, _P,
                                            _P, _P, c_size_t, _P, _P]),
    "mla_attention_fwd_from_cq_cached_ring": (c_int32, [_CFG, _P, _P, _P, _P, _P, c_int32, c_int32,
                                                        _P, _P, _P, _P, c_size_t, _P, _P]),
    "mla_attention_workspace_bytes": (c_size_t, [_CFG, c_int32]),
    "mla_attention_uses_tensor_cores": (c_int32, [_CFG, c_int32]),
    "mla_attention_bwd_workspace_bytes": (c_size_t, [_CFG, c_int32]),
    "mla_attention_bwd": (c_int32, [_CFG, _P, _P, _P, _P, c_int32, c_int32, _P, _P, _P, _P, _P, _P,
                                    _P, c_size_t, _P, _P]),
    "mla_attention_fwd": (c_int32, [_CFG, _P, _P, _P, _P, c_int32, c_int32, _P, _P, _P, _P,
                                    c_size_t, _P, _P]),
    "mla_out_proj": (c_int32, [_CFG, _P, _P, _P, _P, _P, _P]),
    "mla_rotate_ring_keys": (c_int32, [_CFG, _P, _P, c_int32, _P, c_size_t, _P]),
    "mla_attention_fwd_cached_ring": (c_int32, [_CFG, _P, _P, _P, _P, c_int32, c_int32, _P, _P,
                                                _P, _P, c_size_t, _P, _P]),
    "mla_attention_fwd_static_scratch": (c_int32, [_CFG, _P, _P, _P, _P, c_int32, c_int32, _P,
                                                   _P, _P, _P, _P]),
    "mla_selftest_wait_timeout": (c_int32, [_P, c_int32, _P]),
    "mla_selftest_exp2": (c_int32, [_P, _P, _P, _P, c_int32, _P]),
    "mla_selftest_sincos": (c_int32, [_P, _P, _P, c_int32, _P]),
    "mla_selftest_rope_angles": (c_int32, [_CFG, _P, c_int32, _P, _P, _P, _P]),
    "mla_probe_sm_clock": (c_int32, [_P, c_int32, c_int32, _P]),
}

_lib = None
_lock = threading.Lock()


class MLAError(RuntimeError):
    """A non-zero mla_status from the library."""

    def __init__(self, fn: str, status: int, message: str):
        self.status = status
        super().__init__(f"{fn} -> {status_string(status)}: {message}")


def lib() -> ctypes.CDLL:
    """The loaded library (loaded once)."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{LIB_PATH} is missing: build it with "
                    "`python -m mla_latent_kv_attn_b200.build` (nvcc, sm_100a)")
            handle = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(handle, name)   # AttributeError if a symbol is missing
                fn.restype = res
                fn.argtypes = args
            _lib = handle
    return _lib


def status_string(status: int) -> str:
    return lib().mla_status_string(status).decode()


def last_error() -> str:
    return lib().mla_last_error().decode()


def check(fn: str, status: int) -> None:
    if status != MLA_OK:
        raise MLAError(fn, status, last_error())
