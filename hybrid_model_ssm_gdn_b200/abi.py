"""ctypes declarations of the C ABI in include/rssm.h (argument marshalling only).

The shared library is ``lib/librssm.so`` next to this file, built by
``hybrid_model_ssm_gdn_b200.build``.  Loading fails loudly if it is missing:
there is no fallback implementation.
"""

from __future__ import annotations

import ctypes as C
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "lib", "librssm.so")

# enums (values as in include/rssm.h)
MAMBA2, GDN = 0, 1
F32, BF16 = 0, 1
HP_F32, HP_F16_SR, HP_F8_SR = 0, 1, 2
READ_SAME, READ_NVFP4, READ_SHARED_NVFP4, READ_NVFP4D = 0, 1, 2, 3
STATUS = {0: "RSSM_OK", 1: "RSSM_ERR_ARG", 2: "RSSM_ERR_SHAPE", 3: "RSSM_ERR_UNSUPPORTED",
          4: "RSSM_ERR_ARENA_TOO_SMALL", 5: "RSSM_ERR_CUDA", 6: "RSSM_ERR_DEVICE"}
DEV_OK, DEV_PENDING, DEV_NO_VERIFY, DEV_ACCEPTED, DEV_TIMEOUT = 0, 1, 2, 3, 4


class Config(C.Structure):
    _fields_ = [("kind", C.c_int), ("batch", C.c_int), ("nheads", C.c_int), ("headdim", C.c_int),
                ("dstate", C.c_int), ("ngroups", C.c_int), ("window", C.c_int), ("max_draft", C.c_int),
                ("in_dtype", C.c_int), ("hp", C.c_int), ("read", C.c_int), ("seed", C.c_ulonglong),
                ("q_scale", C.c_float), ("A", C.c_void_p), ("D", C.c_void_p), ("skip_tau", C.c_float)]


class Tokens(C.Structure):
    _fields_ = [("x", C.c_void_p), ("B", C.c_void_p), ("C", C.c_void_p), ("dt", C.c_void_p),
                ("q", C.c_void_p), ("k", C.c_void_p), ("v", C.c_void_p), ("alpha", C.c_void_p),
                ("beta", C.c_void_p)]


class RSSMError(RuntimeError):
    def __init__(self, status: int, what: str, detail: str = ""):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)}{(' (' + detail + ')') if detail else ''}")


_P = C.c_void_p
_SIGS = {
    "rssm_arena_bytes": [C.POINTER(Config), C.POINTER(C.c_size_t)],
    "rssm_ring_bytes": [C.POINTER(Config), C.POINTER(C.c_size_t)],
    "rssm_create": [C.POINTER(Config), _P, C.c_size_t, C.POINTER(_P)],
    "rssm_destroy": [_P],
    "rssm_load_checkpoint": [_P, _P, _P],
    "rssm_mamba2_step": [_P, _P, _P, _P, _P, _P, _P],
    "rssm_gdn_step": [_P, _P, _P, _P, _P, _P, _P, _P],
    "rssm_verify": [_P, C.c_int, C.POINTER(Tokens), _P, _P],
    "rssm_commit": [_P, _P, _P],
    "rssm_flush": [_P, _P, _P],
    "rssm_export": [_P, _P, _P, _P, _P],
    "rssm_export_read_copy": [_P, _P, _P, _P, _P],
    "rssm_export_skip": [_P, _P, _P],
    "rssm_export_column_scales": [_P, _P, _P],
    "rssm_get_error": [_P, C.POINTER(C.c_int), C.POINTER(C.c_int), _P],
    "rssm_conv_mamba2_step": [C.POINTER(Config), _P, _P, _P, _P, _P, _P, _P],
    "rssm_conv_gdn_step": [C.POINTER(Config), _P, _P, _P, _P, _P, _P, _P, _P],
    "rssm_snap_verify": [C.POINTER(Config), _P, _P, C.c_int, C.POINTER(Tokens), _P, _P],
    "rssm_snap_commit": [C.POINTER(Config), _P, _P, _P],
    "rssm_sched_probe": [C.c_int, C.c_int, _P, _P, _P],
}

_lib = None


def load() -> C.CDLL:
    """Load lib/librssm.so once and declare every entry point; raises if it is absent."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m hybrid_model_ssm_gdn_b200.build`")
        lib = C.CDLL(LIB_PATH)
        for name, args in _SIGS.items():
            f = getattr(lib, name)
            f.argtypes = args
            f.restype = C.c_int
        lib.rssm_last_cuda_error.argtypes = []
        lib.rssm_last_cuda_error.restype = C.c_char_p
        _lib = lib
    return _lib


def check(status: int, what: str) -> None:
    if status != 0:
        detail = load().rssm_last_cuda_error().decode() if status == 5 else ""
        raise RSSMError(status, what, detail)
