"""CPU checks of the C ABI: the library loads, exports every function that
include/nvfp4ws.h declares, and rejects bad arguments on the host before
touching the GPU. No compute call is made here."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "nvfp4ws.h")


@pytest.fixture(scope="module")
def lib():
    from nvfp4_weight_streaming_gemm_b200 import build, _lib
    build.build()
    return _lib.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = "\n".join(l for l in text.splitlines() if not l.lstrip().startswith("#"))
    names = []
    for decl in text.split(";"):
        if "(" not in decl or "typedef" in decl or "{" in decl.split("(")[0]:
            continue
        m = re.search(r"([A-Za-z_][A-Za-z0-9_]*)\s*\($", decl.split("(")[0] + "(")
        if m:
            names.append(m.group(1))
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("nvfp4_pack", "nvfp4_gemm_skinny", "lmhead_verify_argmax_accept",
                     "nvfp4_gemm_workspace_bytes", "lmhead_verify_workspace_bytes", "nvfp4ws_status_string",
                     "nvfp4ws_last_error", "nvfp4ws_check"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert missing == []


def test_binding_covers_header(lib):
    from nvfp4_weight_streaming_gemm_b200 import _lib
    assert sorted(_lib.SIGNATURES) == declared_functions()


def test_status_strings(lib):
    assert lib.nvfp4ws_status_string(0) == b"NVFP4WS_OK"
    assert lib.nvfp4ws_status_string(6) == b"NVFP4WS_ERR_DEVICE_TIMEOUT"
    assert lib.nvfp4ws_status_string(99) == b"NVFP4WS_UNKNOWN_STATUS"
    assert lib.nvfp4ws_version() >= 100


FAKE = 0x1000000        # 16-byte aligned, never dereferenced: validation fails first


def test_gemm_rejects_null_and_bad_shapes(lib):
    f = lib.nvfp4_gemm_skinny
    assert f(None, FAKE, FAKE, FAKE, 1, 16, 64, FAKE, 0, None, 0, None) == 1
    assert f(FAKE, FAKE, FAKE, FAKE, 0, 16, 64, FAKE, 0, None, 0, None) == 1
    assert f(FAKE, FAKE, FAKE, FAKE, 1, 16, 48, FAKE, 0, None, 0, None) == 2      # K % 32
    assert f(FAKE, FAKE, FAKE, FAKE, 257, 16, 64, FAKE, 0, None, 0, None) == 2    # M > 256
    assert f(FAKE + 8, FAKE, FAKE, FAKE, 1, 16, 64, FAKE, 0, None, 0, None) == 3  # misaligned X
    assert f(FAKE, FAKE, FAKE, FAKE, 1, 16, 64, FAKE + 4, 0, None, 0, None) == 3  # misaligned Y
    assert f(FAKE, FAKE, FAKE, FAKE, 1, 16, 64, FAKE, 7, None, 0, None) == 1      # bad y dtype
    assert b"K=48" in lib.nvfp4ws_last_error() or lib.nvfp4ws_last_error() != b""


def test_gemm_rejects_bad_path(lib):
    assert lib.nvfp4_gemm_skinny_path(FAKE, FAKE, FAKE, FAKE, 1, 16, 64, FAKE, 0, None, 0, 9, None) == 1


def test_pack_rejects(lib):
    f = lib.nvfp4_pack
    assert f(None, 4, 32, FAKE, FAKE, FAKE, None, None) == 1
    assert f(FAKE, 4, 24, FAKE, FAKE, FAKE, None, None) == 1                      # K % 16
    assert f(FAKE + 4, 4, 32, FAKE, FAKE, FAKE, None, None) == 3


def test_verify_rejects(lib):
    f = lib.lmhead_verify_argmax_accept
    # M != B*(D+1)
    assert f(FAKE, FAKE, FAKE, FAKE, 17, 100, 64, FAKE, 2, 16, FAKE, FAKE, None, FAKE, 1 << 20, None) == 1
    # drafts missing with D > 0
    assert f(FAKE, FAKE, FAKE, FAKE, 17, 100, 64, None, 1, 16, FAKE, FAKE, None, FAKE, 1 << 20, None) == 1
    # null outputs
    assert f(FAKE, FAKE, FAKE, FAKE, 17, 100, 64, FAKE, 1, 16, None, FAKE, None, FAKE, 1 << 20, None) == 1
    assert f(FAKE, FAKE, FAKE, FAKE, 1, 100, 64, None, 0, 0, FAKE, FAKE, None, FAKE, 1 << 20, None) == 1  # B < 1


def test_w4a4_rejects_on_the_host(lib):
    f = lib.nvfp4_gemm_w4a4
    assert f(None, FAKE, FAKE, FAKE, 1, 16, 256, FAKE, 0, None, 0, None) == 1          # null X
    assert f(FAKE, FAKE, FAKE, FAKE, 257, 16, 256, FAKE, 0, None, 0, None) == 2        # M > 256
    assert f(FAKE, FAKE, FAKE, FAKE, 4, 16, 256, FAKE, 3, None, 0, None) == 1          # bad y dtype
    assert f(FAKE, FAKE, FAKE, FAKE, 4, 16, 96, FAKE, 0, None, 0, None) == 2           # K % 256
    assert f(FAKE, FAKE, FAKE, FAKE, 4, 16, 256, FAKE + 4, 0, None, 0, None) == 3      # misaligned Y
    assert lib.nvfp4_gemm_w4a4_workspace_bytes(0, 16, 256) == 0
    assert lib.nvfp4_gemm_w4a4_workspace_bytes(257, 16, 256) == 0


def test_tree_verify_needs_parents(lib):
    f = lib.lmhead_verify_tree
    # D = 3 drafts but no parent array: refused before anything is launched
    assert f(FAKE, FAKE, FAKE, FAKE, 4, 100, 256, FAKE, None, 1, 3, FAKE, FAKE, None, None, None, 0, None) == 1
    assert b"parents" in lib.nvfp4ws_last_error()


def test_pass_flags_are_checked_first(lib):
    from nvfp4_weight_streaming_gemm_b200 import _lib as L
    arr = (L.GemmProblem * 1)()
    arr[0] = L.GemmProblem(FAKE, FAKE, FAKE, FAKE, 128, 256, FAKE, 0)
    assert lib.nvfp4_pass_workspace_bytes_ex(arr, 1, 17, 0, 8) == 0        # unknown flag
    assert lib.nvfp4_pass_workspace_bytes_ex(arr, 1, 17, 1, 2) == 0        # W4A4 with a verify problem
    assert lib.nvfp4_pass_workspace_bytes_ex(arr, 1, 17, 0, 6) == 0        # W4A4 with four terms
    assert lib.nvfp4_pass_workspace_bytes_ex(arr, 1, 71, 0, 0) == 0        # 5 terms: M <= 70
    assert lib.nvfp4_pass_workspace_bytes_ex(arr, 1, 89, 0, 4) == 0        # 4 terms: M <= 88
    assert lib.nvfp4_pass_workspace_bytes_ex(arr, 1, 71, 1, 4) == 0        # the verify keeps 5 terms
    st = L.PassState()
    assert lib.nvfp4_pass_init_ex(ctypes.byref(st), arr, 1, 17, None, 8, FAKE, 1 << 20) == 1
    assert b"flags" in lib.nvfp4ws_last_error()
    assert lib.nvfp4_pass_init_ex(ctypes.byref(st), arr, 1, 17, None, 6, FAKE, 1 << 20) == 1
    assert b"flags" in lib.nvfp4ws_last_error()


def test_fp8_rejects_on_the_host(lib):
    from nvfp4_weight_streaming_gemm_b200 import _lib as L
    p = lib.fp8_pack
    assert p(None, 4, 128, FAKE, FAKE, None) == 1
    assert p(FAKE, 4, 24, FAKE, FAKE, None) == 1                                     # K % 16
    assert p(FAKE + 4, 4, 128, FAKE, FAKE, None) == 3                                # misaligned W
    assert p(FAKE, 4, 128, FAKE, FAKE + 2, None) == 3                                # misaligned scales
    g = lib.fp8_gemm_skinny
    assert g(None, FAKE, FAKE, 1, 16, 128, FAKE, 0, FAKE, 1 << 30, None) == 1
    assert g(FAKE, FAKE, FAKE, 129, 16, 128, FAKE, 0, FAKE, 1 << 30, None) == 2      # M > 128
    assert g(FAKE, FAKE, FAKE, 4, 16, 192, FAKE, 0, FAKE, 1 << 30, None) == 2        # K % 128
    assert g(FAKE, FAKE, FAKE, 4, 16, 128, FAKE, 2, FAKE, 1 << 30, None) == 1        # bad y dtype
    assert g(FAKE, FAKE, FAKE, 4, 16, 128, FAKE + 4, 0, FAKE, 1 << 30, None) == 3    # misaligned Y
    assert g(FAKE, FAKE, FAKE, 4, 16, 128, FAKE, 0, None, 0, None) == 4              # no workspace
    assert lib.fp8_gemm_workspace_bytes(129, 16, 128) == 0
    assert lib.fp8_gemm_workspace_bytes(4, 16, 128) > 0
    v = lib.fp8_lmhead_verify
    spec = L.VerifySpec(FAKE, 2, 16, FAKE, FAKE, None, None, None)
    assert v(FAKE, FAKE, FAKE, 17, 100, 128, ctypes.byref(spec), FAKE, 1 << 30, None) == 1   # M != B*(D+1)
    assert v(FAKE, FAKE, FAKE, 17, 100, 128, None, FAKE, 1 << 30, None) == 1                 # no rule
    spec = L.VerifySpec(None, 1, 16, FAKE, FAKE, None, None, None)
    assert v(FAKE, FAKE, FAKE, 17, 100, 128, ctypes.byref(spec), FAKE, 1 << 30, None) == 1   # drafts missing


class _OldGemmProblem(ctypes.Structure):
    """nvfp4_gemm_problem as it was before struct_size (ABI versions up to 102)."""
    _fields_ = [("X", ctypes.c_void_p), ("q", ctypes.c_void_p), ("sf", ctypes.c_void_p),
                ("tensor_scale", ctypes.c_void_p), ("N", ctypes.c_int64), ("K", ctypes.c_int64),
                ("Y", ctypes.c_void_p), ("y_dtype", ctypes.c_int32)]


class _OldVerifySpec(ctypes.Structure):
    """nvfp4_verify_spec of ABI version 100: no struct_size, no parents, no accept_node."""
    _fields_ = [("drafts", ctypes.c_void_p), ("B", ctypes.c_int32), ("D", ctypes.c_int32),
                ("argmax", ctypes.c_void_p), ("accept_len", ctypes.c_void_p), ("max_logit", ctypes.c_void_p)]


def test_structs_carry_their_size(lib):
    from nvfp4_weight_streaming_gemm_b200 import _lib as L
    assert lib.nvfp4ws_version() >= 200
    assert L.GemmProblem(FAKE, FAKE, FAKE, FAKE, 128, 256, FAKE, 0).struct_size == ctypes.sizeof(L.GemmProblem)
    assert L.VerifySpec(FAKE, 1, 16).struct_size == ctypes.sizeof(L.VerifySpec)


def test_pass_refuses_a_struct_of_another_size(lib):
    """A caller built against another header version is refused on the host with
    INVALID_ARG, before any member past struct_size is read."""
    from nvfp4_weight_streaming_gemm_b200 import _lib as L
    arr = (L.GemmProblem * 2)()
    for i in range(2):
        arr[i] = L.GemmProblem(FAKE, FAKE, FAKE, FAKE, 128, 256, FAKE, 0)
    arr[1].struct_size = ctypes.sizeof(L.GemmProblem) - 8
    st = L.PassState()
    assert lib.nvfp4_pass_workspace_bytes(arr, 2, 17, 0) == 0
    assert lib.nvfp4_pass_init(ctypes.byref(st), arr, 2, 17, None, FAKE, 1 << 30) == 1
    assert b"problem 1: struct_size" in lib.nvfp4ws_last_error()
    # an array of the old layout: its first member is a pointer, never the struct size
    old = (_OldGemmProblem * 1)()
    old[0] = _OldGemmProblem(FAKE, FAKE, FAKE, FAKE, 128, 256, FAKE, 0)
    old_ptr = ctypes.cast(old, ctypes.POINTER(L.GemmProblem))
    assert lib.nvfp4_pass_init(ctypes.byref(st), old_ptr, 1, 17, None, FAKE, 1 << 30) == 1
    assert b"struct_size" in lib.nvfp4ws_last_error()
    # a short verify struct (the one that once had its missing members read as pointers)
    arr1 = (L.GemmProblem * 1)()
    arr1[0] = L.GemmProblem(FAKE, FAKE, FAKE, FAKE, 128, 256, None, 0)
    short = _OldVerifySpec(FAKE, 1, 16, FAKE, FAKE, None)
    vs_ptr = ctypes.cast(ctypes.pointer(short), ctypes.POINTER(L.VerifySpec))
    assert lib.nvfp4_pass_init(ctypes.byref(st), arr1, 1, 17, vs_ptr, FAKE, 1 << 30) == 1
    assert b"verify struct_size" in lib.nvfp4ws_last_error()
    assert lib.fp8_lmhead_verify(FAKE, FAKE, FAKE, 17, 100, 128, vs_ptr, FAKE, 1 << 30, None) == 1
    assert b"struct_size" in lib.nvfp4ws_last_error()


def test_fp8_pass_rejects_on_the_host(lib):
    from nvfp4_weight_streaming_gemm_b200 import _lib as L
    arr = (L.Fp8Problem * 2)()
    arr[0] = L.Fp8Problem(FAKE, FAKE, FAKE, 128, 256, FAKE, 0)
    arr[1] = L.Fp8Problem(FAKE, FAKE, FAKE, 128, 192, FAKE, 0)              # K % 128
    assert lib.fp8_pass_workspace_bytes(arr, 2, 17, 0) == 0
    assert lib.fp8_pass_workspace_bytes(arr, 1, 17, 0) > 0
    assert lib.fp8_pass_workspace_bytes(arr, 1, 129, 0) == 0                  # M > 128
    st = L.PassState()
    assert lib.fp8_pass_init(ctypes.byref(st), arr, 2, 17, None, FAKE, 1 << 30) == 2
    arr[1] = L.Fp8Problem(FAKE, FAKE, FAKE, 128, 256, None, 0)              # Y missing, not a verify problem
    assert lib.fp8_pass_init(ctypes.byref(st), arr, 2, 17, None, FAKE, 1 << 30) == 1
    spec = L.VerifySpec(FAKE, 2, 16, FAKE, FAKE, None, None, None)          # M != B*(D+1)
    assert lib.fp8_pass_init(ctypes.byref(st), arr, 2, 17, ctypes.byref(spec), FAKE, 1 << 30) == 1
    arr[0].struct_size = 8                                                   # another header's struct
    assert lib.fp8_pass_workspace_bytes(arr, 1, 17, 0) == 0
    assert lib.fp8_pass_init(ctypes.byref(st), arr, 1, 17, None, FAKE, 1 << 30) == 1
    assert b"struct_size" in lib.nvfp4ws_last_error()
    assert lib.fp8_pass_run(None, None) == 1
    assert lib.fp8_pass_run(ctypes.byref(L.PassState()), None) == 1       # never initialised
