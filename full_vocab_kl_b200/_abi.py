"""ctypes declarations of the C ABI in ``include/nb_kl.h`` (argument marshalling only).

The shared library is loaded from this package directory. There is no fallback: if
``libnbkl.so`` is missing, :func:`lib` raises, and every call of the Python API fails
loudly instead of computing anything another way.
"""

from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_char_p, c_float, c_int, c_int32, c_int64, c_size_t, c_uint64, c_void_p

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libnbkl.so")

NB_OK = 0
NB_ERR_INVALID_ARG = -1
NB_ERR_UNSUPPORTED = -2
NB_ERR_WORKSPACE = -3
NB_ERR_CUDA = -4
NB_ERR_TIMEOUT = -5
NB_BF16 = 0
NB_F32 = 1
NOALLOC_SCRATCH_BYTES = 64 * 1024 * 1024
VP_FIELDS = 7   # NB_KL_VP_FIELDS: floats per token of a vocabulary shard's state
SMALL_WORKSPACE_BYTES = 256   # NB_KL_SMALL_WORKSPACE_BYTES

# every function the header declares, with (restype, argtypes)
SIGNATURES = {
    "nb_kl_workspace_size": (c_size_t, [c_void_p, c_float]),
    "nb_kl_chunk_columns": (c_int64, [c_void_p]),
    "nb_kl_forward": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_float, c_float,
                              c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_size_t,
                              c_void_p]),
    "nb_kl_forward_side": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_float, c_float,
                                   c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                   c_void_p, c_size_t, c_void_p]),
    "nb_kl_vp_state": (c_int, [c_void_p, c_int64, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_float,
                               c_float, c_void_p, c_void_p, c_size_t, c_void_p]),
    "nb_kl_vp_combine": (c_int, [c_int64, c_int, c_void_p, c_void_p, c_int64, c_float, c_void_p, c_void_p,
                                 c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p]),
    "nb_kl_vp_jsd_partial": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_float,
                                     c_float, c_void_p, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "nb_kl_vp_jsd_combine": (c_int, [c_int64, c_int, c_void_p, c_void_p, c_int64, c_void_p, c_void_p, c_void_p,
                                     c_void_p, c_void_p]),
    "nb_kl_gram": (c_int, [c_void_p, c_int64, c_int64, c_void_p, c_void_p, c_void_p]),
    "nb_kl_project": (c_int, [c_void_p, c_int64, c_int64, c_void_p, c_int64, c_void_p, c_void_p, c_void_p]),
    "nb_kl_spectral_select": (c_int, [c_void_p, c_void_p, c_int64, c_int64, c_void_p, c_void_p, c_void_p,
                                      c_void_p]),
    "nb_kl_handoff_rows": (c_int, [c_void_p, c_void_p, c_int64, c_int64, c_void_p, c_int64, c_void_p]),
    "nb_kl_enable_peer_access": (c_int, [c_int]),
    "nb_kl_backward": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_float, c_float,
                               c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_void_p,
                               c_size_t, c_void_p]),
    "nb_kl_forward_noalloc": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_float,
                                      c_float, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                      c_void_p]),
    "nb_kl_noalloc_device_status": (c_int, [c_void_p]),
    "nb_kl_status_string": (c_char_p, [c_int]),
    "nb_kl_device_status": (c_int, [c_void_p, c_void_p]),
    "nb_kl_debug_gemm": (c_int, [c_void_p, c_int, c_void_p, c_int, c_int64, c_int64, c_int64, c_void_p, c_void_p,
                                 c_void_p]),
    "nb_kl_debug_wait_timeout": (c_int, [c_void_p, c_uint64, c_int, c_void_p]),
    "nb_kl_last_launch_count": (c_int, []),
    "nb_kl_timing_enable": (None, [c_int]),
    "nb_kl_timing_read": (c_int, [c_void_p, c_void_p, c_int]),
}

KERNEL_CATEGORIES = ("sweep_fwd", "sweep_jsd", "sweep_grad", "gemm_bwd", "rowops", "gemm_proj", "handoff")


class Shape(ctypes.Structure):
    """Mirror of ``nb_kl_shape``."""

    _fields_ = [
        ("n_tokens", c_int64),
        ("vocab", c_int64),
        ("d_s", c_int64),
        ("d_t", c_int64),
        ("h_dtype", c_int32),
        ("reserved", c_int32),
        ("ignore_index", c_int64),
        ("chunk_v", c_int64),
    ]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m full_vocab_kl_b200.build` "
                "(there is no CPU fallback)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().nb_kl_status_string(code).decode()


class NbKlError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        super().__init__(f"{fn} failed: {status_string(code)} ({code})")


def check(fn: str, code: int) -> None:
    if code != NB_OK:
        raise NbKlError(fn, code)


def shape_ptr(s: Shape):
    return ctypes.cast(ctypes.pointer(s), c_void_p)
