"""ctypes loader of libnvfp4ws.so (the C ABI declared in include/nvfp4ws.h).

There is no fallback. If the library is missing or does not load, importing the
binding raises. Build it with ``python -m nvfp4_weight_streaming_gemm_b200.build``.
"""

from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libnvfp4ws.so")

c_i64, c_i32, c_p, c_sz = ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p, ctypes.c_size_t


class GemmProblem(ctypes.Structure):
    """nvfp4_gemm_problem: one GEMM of a weight pass. ``struct_size`` is filled in by the
    constructor (the library refuses any other value)."""
    _fields_ = [("struct_size", ctypes.c_uint32), ("X", c_p), ("q", c_p), ("sf", c_p), ("tensor_scale", c_p),
                ("N", c_i64), ("K", c_i64), ("Y", c_p), ("y_dtype", c_i32)]

    def __init__(self, *args, **kw):
        super().__init__(ctypes.sizeof(GemmProblem), *args, **kw)


class VerifySpec(ctypes.Structure):
    """nvfp4_verify_spec: the verify buffers of a pass whose last problem is the lm_head.
    ``struct_size`` is filled in by the constructor."""
    _fields_ = [("struct_size", ctypes.c_uint32), ("drafts", c_p), ("B", c_i32), ("D", c_i32), ("argmax", c_p),
                ("accept_len", c_p), ("max_logit", c_p), ("parents", c_p), ("accept_node", c_p)]

    def __init__(self, *args, **kw):
        super().__init__(ctypes.sizeof(VerifySpec), *args, **kw)


class Fp8Problem(ctypes.Structure):
    """fp8_gemm_problem: one GEMM of an FP8 weight pass. ``struct_size`` is filled in by the constructor."""
    _fields_ = [("struct_size", ctypes.c_uint32), ("X", c_p), ("q", c_p), ("scales", c_p), ("N", c_i64),
                ("K", c_i64), ("Y", c_p), ("y_dtype", c_i32)]

    def __init__(self, *args, **kw):
        super().__init__(ctypes.sizeof(Fp8Problem), *args, **kw)


class PassState(ctypes.Structure):
    """nvfp4_pass: caller-owned host state of an initialised pass."""
    _fields_ = [("opaque", ctypes.c_uint64 * 32)]


# name -> (restype, argtypes)
SIGNATURES = {
    "nvfp4ws_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "nvfp4ws_last_error": (ctypes.c_char_p, []),
    "nvfp4ws_version": (ctypes.c_int, []),
    "nvfp4ws_sm_count": (ctypes.c_int, []),
    "nvfp4_pack": (ctypes.c_int, [c_p, c_i64, c_i64, c_p, c_p, c_p, c_p, c_p]),
    "nvfp4_gemm_workspace_bytes": (c_sz, [c_i64, c_i64, c_i64]),
    "nvfp4_gemm_skinny": (ctypes.c_int, [c_p, c_p, c_p, c_p, c_i64, c_i64, c_i64, c_p, ctypes.c_int, c_p, c_sz, c_p]),
    "nvfp4_gemm_skinny_path": (ctypes.c_int, [c_p, c_p, c_p, c_p, c_i64, c_i64, c_i64, c_p, ctypes.c_int, c_p, c_sz,
                                              ctypes.c_int, c_p]),
    "lmhead_verify_workspace_bytes": (c_sz, [c_i64, c_i64, c_i64]),
    "lmhead_verify_argmax_accept": (ctypes.c_int, [c_p, c_p, c_p, c_p, c_i64, c_i64, c_i64, c_p, c_i32, c_i32, c_p,
                                                   c_p, c_p, c_p, c_sz, c_p]),
    "lmhead_verify_argmax_accept_path": (ctypes.c_int, [c_p, c_p, c_p, c_p, c_i64, c_i64, c_i64, c_p, c_i32, c_i32,
                                                        c_p, c_p, c_p, c_p, c_sz, ctypes.c_int, c_p]),
    "lmhead_verify_tree": (ctypes.c_int, [c_p, c_p, c_p, c_p, c_i64, c_i64, c_i64, c_p, c_p, c_i32, c_i32, c_p, c_p,
                                          c_p, c_p, c_p, c_sz, c_p]),
    "nvfp4_gemm_w4a4_workspace_bytes": (c_sz, [c_i64, c_i64, c_i64]),
    "nvfp4_gemm_w4a4": (ctypes.c_int, [c_p, c_p, c_p, c_p, c_i64, c_i64, c_i64, c_p, ctypes.c_int, c_p, c_sz, c_p]),
    "nvfp4ws_check": (ctypes.c_int, [c_p]),
    "nvfp4_gemm_skinny_noalloc": (ctypes.c_int, [c_p, c_p, c_p, c_p, c_i64, c_i64, c_i64, c_p, ctypes.c_int, c_p]),
    "nvfp4ws_kernel_launches": (ctypes.c_ulonglong, []),
    "nvfp4_pass_workspace_bytes": (c_sz, [ctypes.POINTER(GemmProblem), c_i32, c_i64, c_i32]),
    "nvfp4_pass_init": (ctypes.c_int, [ctypes.POINTER(PassState), ctypes.POINTER(GemmProblem), c_i32, c_i64,
                                       ctypes.POINTER(VerifySpec), c_p, c_sz]),
    "nvfp4_pass_run": (ctypes.c_int, [ctypes.POINTER(PassState), c_p]),
    "nvfp4_pass_workspace_bytes_ex": (c_sz, [ctypes.POINTER(GemmProblem), c_i32, c_i64, c_i32, ctypes.c_uint32]),
    "nvfp4_pass_init_ex": (ctypes.c_int, [ctypes.POINTER(PassState), ctypes.POINTER(GemmProblem), c_i32, c_i64,
                                          ctypes.POINTER(VerifySpec), ctypes.c_uint32, c_p, c_sz]),
    "fp8_pack": (ctypes.c_int, [c_p, c_i64, c_i64, c_p, c_p, c_p]),
    "fp8_gemm_workspace_bytes": (c_sz, [c_i64, c_i64, c_i64]),
    "fp8_gemm_skinny": (ctypes.c_int, [c_p, c_p, c_p, c_i64, c_i64, c_i64, c_p, ctypes.c_int, c_p, c_sz, c_p]),
    "fp8_gemm_skinny_path": (ctypes.c_int, [c_p, c_p, c_p, c_i64, c_i64, c_i64, c_p, ctypes.c_int, c_p, c_sz,
                                            ctypes.c_int, c_p]),
    "fp8_lmhead_verify_path": (ctypes.c_int, [c_p, c_p, c_p, c_i64, c_i64, c_i64, ctypes.POINTER(VerifySpec), c_p,
                                              c_sz, ctypes.c_int, c_p]),
    "fp8_lmhead_verify_workspace_bytes": (c_sz, [c_i64, c_i64, c_i64]),
    "fp8_lmhead_verify": (ctypes.c_int, [c_p, c_p, c_p, c_i64, c_i64, c_i64, ctypes.POINTER(VerifySpec), c_p, c_sz,
                                         c_p]),
    "fp8_pass_workspace_bytes": (c_sz, [ctypes.POINTER(Fp8Problem), c_i32, c_i64, c_i32]),
    "fp8_pass_workspace_bytes_path": (c_sz, [ctypes.POINTER(Fp8Problem), c_i32, c_i64, c_i32, ctypes.c_int]),
    "fp8_pass_init_path": (ctypes.c_int, [ctypes.POINTER(PassState), ctypes.POINTER(Fp8Problem), c_i32, c_i64,
                                          ctypes.POINTER(VerifySpec), ctypes.c_int, c_p, c_sz]),
    "fp8_pass_init": (ctypes.c_int, [ctypes.POINTER(PassState), ctypes.POINTER(Fp8Problem), c_i32, c_i64,
                                     ctypes.POINTER(VerifySpec), c_p, c_sz]),
    "fp8_pass_run": (ctypes.c_int, [ctypes.POINTER(PassState), c_p]),
}

_lib = None


def load() -> ctypes.CDLL:
    """Load the library once and declare every signature. Raises OSError if it is absent."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise OSError(f"{LIB_PATH} is missing: build it with `python -m nvfp4_weight_streaming_gemm_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib
