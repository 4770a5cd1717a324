"""NVFP4 weight-streaming skinny GEMM and fused greedy verify for B200 (sm_100a).

A thin binding over the C ABI of ``libnvfp4ws.so`` (declared in
``include/nvfp4ws.h``). Every step of the computation runs in the library's CUDA
kernels. This module only checks tensor properties, allocates outputs with
torch, and passes raw device pointers and the current CUDA stream.

    q, sf, ts = pack(W)                        # fp32 [N, K] -> NVFP4
    Y = gemm(X, q, sf, ts)                     # bf16 [M, K] -> fp32 [M, N]
    t, L, vmax = verify(X, q, sf, ts, drafts)  # fused lm_head argmax + accept length
    t, L, node, vmax = verify_tree(X, q, sf, ts, drafts, parents)   # the same over a draft tree
    p = WeightPass([(X_i, q_i, sf_i, ts_i, Y_i), ...], M, verify=...)   # a whole list, one launch
    p.run()
    q8, s8 = fp8_pack(W)                       # fp32 [N, K] -> E4M3 + fp32 per 128 x 128 block
    Y = fp8_gemm(X, q8, s8)                    # and its verify: fp8_verify(X, q8, s8, drafts[, parents])
"""

from __future__ import annotations

import ctypes

import torch

from . import _lib

PATHS = {"auto": 0, "gemv": 1, "mma": 2, "gemv_regs": 3, "mma_f16": 4}
PASS_BATCH_INVARIANT = 1
PASS_W4A4 = 2
PASS_FOUR_TERMS = 4
FP8_PATHS = {"f16": 0, "terms": 1}
STATUS_OK = 0


class NVFP4WSError(RuntimeError):
    def __init__(self, status: int, where: str):
        lib = _lib.load()
        name = lib.nvfp4ws_status_string(status).decode()
        detail = lib.nvfp4ws_last_error().decode()
        super().__init__(f"{where}: {name}: {detail}")
        self.status = status


def lib() -> ctypes.CDLL:
    return _lib.load()


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _check(status: int, where: str):
    if status != STATUS_OK:
        raise NVFP4WSError(status, where)


def _need_cuda(t, name, dtype=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def pack(W: torch.Tensor, tensor_scale_in: torch.Tensor | None = None, stream=None, out=None):
    """Quantise fp32 W [N, K] to NVFP4. Returns ``(q uint8 [N, K/2], sf uint8 [N, K/16], ts fp32 [1])``."""
    _need_cuda(W, "W", torch.float32)
    N, K = W.shape
    if out is None:
        q = torch.empty((N, K // 2), dtype=torch.uint8, device=W.device)
        sf = torch.empty((N, K // 16), dtype=torch.uint8, device=W.device)
        ts = torch.empty(1, dtype=torch.float32, device=W.device)
    else:
        q, sf, ts = out
    if tensor_scale_in is not None:
        _need_cuda(tensor_scale_in, "tensor_scale_in", torch.float32)
    _check(lib().nvfp4_pack(_ptr(W), N, K, _ptr(q), _ptr(sf), _ptr(ts), _ptr(tensor_scale_in), _stream(stream)),
           "nvfp4_pack")
    return q, sf, ts


def gemm_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(lib().nvfp4_gemm_workspace_bytes(M, N, K))


def verify_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(lib().lmhead_verify_workspace_bytes(M, N, K))


def _workspace(nbytes: int, device, workspace):
    if nbytes == 0:
        return None
    if workspace is not None and workspace.numel() * workspace.element_size() >= nbytes:
        return workspace
    return torch.zeros(nbytes, dtype=torch.uint8, device=device)   # the library needs it zeroed once


def gemm(X: torch.Tensor, q: torch.Tensor, sf: torch.Tensor, ts: torch.Tensor, out: torch.Tensor | None = None,
         y_dtype: torch.dtype = torch.float32, workspace: torch.Tensor | None = None, path: str = "auto",
         stream=None) -> torch.Tensor:
    """Y[M, N] = X[M, K] . dequant(W)^T with X bf16; Y fp32 (default) or bf16."""
    _need_cuda(X, "X", torch.bfloat16)
    _need_cuda(q, "q", torch.uint8)
    _need_cuda(sf, "sf", torch.uint8)
    M, K = X.shape
    N = q.shape[0]
    if q.shape[1] * 2 != K or sf.shape != (N, K // 16):
        raise ValueError("q / sf shapes do not match X")
    if out is None:
        out = torch.empty((M, N), dtype=y_dtype, device=X.device)
    yd = {torch.float32: 0, torch.bfloat16: 1}[out.dtype]
    ws = _workspace(gemm_workspace_bytes(M, N, K), X.device, workspace)
    nbytes = 0 if ws is None else ws.numel()
    _check(lib().nvfp4_gemm_skinny_path(_ptr(X), _ptr(q), _ptr(sf), _ptr(ts), M, N, K, _ptr(out), yd, _ptr(ws),
                                        nbytes, PATHS[path], _stream(stream)), "nvfp4_gemm_skinny")
    return out


def verify(X: torch.Tensor, q: torch.Tensor, sf: torch.Tensor, ts: torch.Tensor, drafts: torch.Tensor,
           workspace: torch.Tensor | None = None, with_max_logit: bool = True, path: str = "auto", stream=None,
           out=None):
    """Fused lm_head greedy verify. ``drafts`` int32 [B, D]; X has M = B*(D+1) rows.

    Returns ``(argmax int32 [M], accept_len int32 [B], max_logit fp32 [M] or None)``.
    """
    _need_cuda(X, "X", torch.bfloat16)
    _need_cuda(drafts, "drafts", torch.int32)
    M, K = X.shape
    N = q.shape[0]
    B, D = drafts.shape
    if out is None:
        amax = torch.empty(M, dtype=torch.int32, device=X.device)
        acc = torch.empty(B, dtype=torch.int32, device=X.device)
        vmax = torch.empty(M, dtype=torch.float32, device=X.device) if with_max_logit else None
    else:
        amax, acc, vmax = out
    ws = _workspace(verify_workspace_bytes(M, N, K), X.device, workspace)
    nbytes = 0 if ws is None else ws.numel()
    dptr = _ptr(drafts) if drafts.numel() else None
    _check(lib().lmhead_verify_argmax_accept_path(_ptr(X), _ptr(q), _ptr(sf), _ptr(ts), M, N, K, dptr, B, D,
                                                  _ptr(amax), _ptr(acc), _ptr(vmax), _ptr(ws), nbytes, PATHS[path],
                                                  _stream(stream)), "lmhead_verify_argmax_accept")
    return amax, acc, vmax


def verify_tree(X: torch.Tensor, q: torch.Tensor, sf: torch.Tensor, ts: torch.Tensor, drafts: torch.Tensor,
                parents: torch.Tensor, workspace: torch.Tensor | None = None, with_max_logit: bool = True,
                stream=None, out=None):
    """Fused lm_head greedy verify of draft trees (``lmhead_verify_tree``). ``drafts`` and
    ``parents`` int32 [B, D]: node k >= 1 holds ``drafts[b, k-1]`` under node ``parents[b, k-1]``.

    Returns ``(argmax int32 [M], accept_len int32 [B], accept_node int32 [B], max_logit fp32 [M] or None)``.
    """
    _need_cuda(X, "X", torch.bfloat16)
    _need_cuda(drafts, "drafts", torch.int32)
    _need_cuda(parents, "parents", torch.int32)
    M, K = X.shape
    N = q.shape[0]
    B, D = drafts.shape
    if parents.shape != (B, D):
        raise ValueError("parents must have the shape of drafts")
    if out is None:
        amax = torch.empty(M, dtype=torch.int32, device=X.device)
        acc = torch.empty(B, dtype=torch.int32, device=X.device)
        node = torch.empty(B, dtype=torch.int32, device=X.device)
        vmax = torch.empty(M, dtype=torch.float32, device=X.device) if with_max_logit else None
    else:
        amax, acc, node, vmax = out
    ws = _workspace(verify_workspace_bytes(M, N, K), X.device, workspace)
    nbytes = 0 if ws is None else ws.numel()
    dptr = _ptr(drafts) if drafts.numel() else None
    pptr = _ptr(parents) if parents.numel() else None
    _check(lib().lmhead_verify_tree(_ptr(X), _ptr(q), _ptr(sf), _ptr(ts), M, N, K, dptr, pptr, B, D, _ptr(amax),
                                    _ptr(acc), _ptr(node), _ptr(vmax), _ptr(ws), nbytes, _stream(stream)),
           "lmhead_verify_tree")
    return amax, acc, node, vmax


def gemm_w4a4(X: torch.Tensor, q: torch.Tensor, sf: torch.Tensor, ts: torch.Tensor, out: torch.Tensor | None = None,
              y_dtype=torch.float32, workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """W4A4 product (``nvfp4_gemm_w4a4``): X bf16 [M, K] is quantised to NVFP4 per row, then
    multiplied by the packed weight on the block-scaled tensor cores. Returns Y [M, N]."""
    _need_cuda(X, "X", torch.bfloat16)
    M, K = X.shape
    N = q.shape[0]
    Y = out if out is not None else torch.empty((M, N), dtype=y_dtype, device=X.device)
    yd = {torch.float32: 0, torch.bfloat16: 1}[Y.dtype]
    ws = _workspace(int(lib().nvfp4_gemm_w4a4_workspace_bytes(M, N, K)), X.device, workspace)
    nbytes = 0 if ws is None else ws.numel()
    _check(lib().nvfp4_gemm_w4a4(_ptr(X), _ptr(q), _ptr(sf), _ptr(ts), M, N, K, _ptr(Y), yd, _ptr(ws), nbytes,
                                 _stream(stream)), "nvfp4_gemm_w4a4")
    return Y


def fp8_pack(W: torch.Tensor, stream=None, out=None):
    """Quantise fp32 W [N, K] to FP8 E4M3 with one fp32 scale per 128 x 128 block (``fp8_pack``).

    Returns ``(q uint8 [N, K], scales fp32 [ceil(N/128), ceil(K/128)])``.
    """
    _need_cuda(W, "W", torch.float32)
    N, K = W.shape
    if out is None:
        q = torch.empty((N, K), dtype=torch.uint8, device=W.device)
        scales = torch.empty(((N + 127) // 128, (K + 127) // 128), dtype=torch.float32, device=W.device)
    else:
        q, scales = out
    _check(lib().fp8_pack(_ptr(W), N, K, _ptr(q), _ptr(scales), _stream(stream)), "fp8_pack")
    return q, scales


def fp8_gemm(X: torch.Tensor, q: torch.Tensor, scales: torch.Tensor, out: torch.Tensor | None = None,
             y_dtype: torch.dtype = torch.float32, workspace: torch.Tensor | None = None, path: str = "f16",
             stream=None) -> torch.Tensor:
    """Y[M, N] = X[M, K] . dequant(W)^T for FP8 block-scaled W (``fp8_gemm_skinny_path``); X bf16.
    ``path``: "f16" (codes dequantised exactly to f16) or "terms" (codes straight into the FP8
    tensor cores, X as two residual E4M3 terms)."""
    _need_cuda(X, "X", torch.bfloat16)
    _need_cuda(q, "q", torch.uint8)
    _need_cuda(scales, "scales", torch.float32)
    M, K = X.shape
    N = q.shape[0]
    if q.shape[1] != K or scales.shape != ((N + 127) // 128, (K + 127) // 128):
        raise ValueError("q / scales shapes do not match X")
    Y = out if out is not None else torch.empty((M, N), dtype=y_dtype, device=X.device)
    yd = {torch.float32: 0, torch.bfloat16: 1}[Y.dtype]
    ws = _workspace(int(lib().fp8_gemm_workspace_bytes(M, N, K)), X.device, workspace)
    nbytes = 0 if ws is None else ws.numel()
    _check(lib().fp8_gemm_skinny_path(_ptr(X), _ptr(q), _ptr(scales), M, N, K, _ptr(Y), yd, _ptr(ws), nbytes,
                                      FP8_PATHS[path], _stream(stream)), "fp8_gemm_skinny")
    return Y


def fp8_verify(X: torch.Tensor, q: torch.Tensor, scales: torch.Tensor, drafts: torch.Tensor,
               parents: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
               with_max_logit: bool = True, path: str = "f16", stream=None):
    """Fused greedy verify over an FP8 lm_head (``fp8_lmhead_verify``): the chain rule, or the
    tree rule when ``parents`` is given.

    Returns ``(argmax int32 [M], accept_len int32 [B], accept_node int32 [B], max_logit fp32 [M] or None)``.
    """
    _need_cuda(X, "X", torch.bfloat16)
    _need_cuda(drafts, "drafts", torch.int32)
    M, K = X.shape
    N = q.shape[0]
    B, D = drafts.shape
    if parents is not None:
        _need_cuda(parents, "parents", torch.int32)
        if parents.shape != (B, D):
            raise ValueError("parents must have the shape of drafts")
    amax = torch.empty(M, dtype=torch.int32, device=X.device)
    acc = torch.empty(B, dtype=torch.int32, device=X.device)
    node = torch.empty(B, dtype=torch.int32, device=X.device)
    vmax = torch.empty(M, dtype=torch.float32, device=X.device) if with_max_logit else None
    spec = _lib.VerifySpec(_ptr(drafts) if drafts.numel() else None, B, D, _ptr(amax), _ptr(acc), _ptr(vmax),
                           _ptr(parents) if parents is not None and parents.numel() else None, _ptr(node))
    ws = _workspace(int(lib().fp8_lmhead_verify_workspace_bytes(M, N, K)), X.device, workspace)
    nbytes = 0 if ws is None else ws.numel()
    _check(lib().fp8_lmhead_verify_path(_ptr(X), _ptr(q), _ptr(scales), M, N, K, ctypes.byref(spec), _ptr(ws),
                                        nbytes, FP8_PATHS[path], _stream(stream)), "fp8_lmhead_verify")
    return amax, acc, node, vmax


def check(stream=None):
    """Synchronise and report a device-side bounded-wait failure, if any."""
    _check(lib().nvfp4ws_check(_stream(stream)), "nvfp4ws_check")


class WeightPass:
    """A list of independent GEMMs sharing M, run by one persistent launch (``nvfp4_pass_*``).

    ``problems`` is a list of ``(X, q, sf, ts, Y)``: X bf16 [M, K], the packed weight,
    and Y fp32 or bf16 [M, N]. With ``verify=(drafts, argmax, accept_len, max_logit)``
    the last problem is the lm_head: its Y may be None, and each run ends with the
    argmax over its rows and the accept lengths. ``verify`` may add ``(parents,
    accept_node)`` for a tree verify (``accept_node`` may be None). With
    ``batch_invariant`` every row gets the same bits for any M; with ``w4a4`` every
    problem is the W4A4 product of :func:`gemm_w4a4` (no verify; ``nvfp4_pass_init_ex``);
    with ``four_terms`` the GEMMs take 4 residual activation terms instead of 5 (~1e-4 of
    max|y| instead of ~1e-5; the verify keeps 5 and runs as a second launch).
    Every tensor is referenced by address: keep them alive and refill X in place
    between runs.
    """

    def __init__(self, problems, M: int, verify=None, workspace: torch.Tensor | None = None,
                 batch_invariant: bool = False, w4a4: bool = False, four_terms: bool = False):
        L = _lib
        n = len(problems)
        self._keep = []
        arr = (L.GemmProblem * n)()
        for i, (X, q, sf, ts, Y) in enumerate(problems):
            _need_cuda(X, "X", torch.bfloat16)
            _need_cuda(q, "q", torch.uint8)
            _need_cuda(sf, "sf", torch.uint8)
            if X.shape[0] != M:
                raise ValueError(f"problem {i}: X has {X.shape[0]} rows, expected M={M}")
            K = X.shape[1]
            N = q.shape[0]
            if q.shape[1] * 2 != K or sf.shape != (N, K // 16):
                raise ValueError(f"problem {i}: q / sf shapes do not match X")
            yd = 0
            if Y is not None:
                _need_cuda(Y, "Y")
                if Y.shape != (M, N):
                    raise ValueError(f"problem {i}: Y must be [{M}, {N}]")
                yd = {torch.float32: 0, torch.bfloat16: 1}[Y.dtype]
            arr[i] = L.GemmProblem(_ptr(X), _ptr(q), _ptr(sf), _ptr(ts), N, K, _ptr(Y), yd)
            self._keep.extend([X, q, sf, ts, Y])
        vs = None
        if verify is not None:
            drafts, amax, acc, vmax = verify[:4]
            parents, node = (tuple(verify[4:]) + (None, None))[:2]
            _need_cuda(drafts, "drafts", torch.int32)
            B, D = drafts.shape
            if parents is not None:
                _need_cuda(parents, "parents", torch.int32)
                if parents.shape != (B, D):
                    raise ValueError("parents must have the shape of drafts")
            vs = L.VerifySpec(_ptr(drafts) if drafts.numel() else None, B, D, _ptr(amax), _ptr(acc), _ptr(vmax),
                              _ptr(parents) if parents is not None and parents.numel() else None, _ptr(node))
            self._keep.extend([drafts, amax, acc, vmax, parents, node])
        flags = ((PASS_BATCH_INVARIANT if batch_invariant else 0) | (PASS_W4A4 if w4a4 else 0)
                 | (PASS_FOUR_TERMS if four_terms else 0))
        nbytes = int(lib().nvfp4_pass_workspace_bytes_ex(arr, n, M, 1 if verify is not None else 0, flags))
        if nbytes == 0:
            raise NVFP4WSError(1, "nvfp4_pass_workspace_bytes")
        dev = problems[0][0].device
        self.workspace = _workspace(nbytes, dev, workspace)
        self.workspace_bytes = nbytes
        self.state = L.PassState()
        _check(lib().nvfp4_pass_init_ex(ctypes.byref(self.state), arr, n, M,
                                        ctypes.byref(vs) if vs is not None else None, flags,
                                        _ptr(self.workspace), nbytes), "nvfp4_pass_init")
        self.M = M
        self.count = n

    def run(self, stream=None):
        _check(lib().nvfp4_pass_run(ctypes.byref(self.state), _stream(stream)), "nvfp4_pass_run")


class Fp8Pass:
    """A list of independent FP8 GEMMs sharing M, run by one persistent launch (``fp8_pass_*``).

    ``problems`` is a list of ``(X, q, scales, Y)``: X bf16 [M, K], the weight from
    :func:`fp8_pack`, and Y fp32 or bf16 [M, N]. ``verify`` is as for :class:`WeightPass`:
    ``(drafts, argmax, accept_len, max_logit[, parents, accept_node])``, and makes the last
    problem the lm_head (its Y may be None). ``path`` picks the FP8 kernel: "f16" (codes
    dequantised exactly to f16) or "terms" (codes straight into the FP8 tensor cores, X as two
    residual E4M3 terms; ``fp8_pass_init_path``). Every tensor is referenced by address: keep
    them alive and refill X in place between runs.
    """

    def __init__(self, problems, M: int, verify=None, workspace: torch.Tensor | None = None, path: str = "f16"):
        L = _lib
        n = len(problems)
        self._keep = []
        arr = (L.Fp8Problem * n)()
        for i, (X, q, scales, Y) in enumerate(problems):
            _need_cuda(X, "X", torch.bfloat16)
            _need_cuda(q, "q", torch.uint8)
            _need_cuda(scales, "scales", torch.float32)
            if X.shape[0] != M:
                raise ValueError(f"problem {i}: X has {X.shape[0]} rows, expected M={M}")
            K = X.shape[1]
            N = q.shape[0]
            if q.shape[1] != K or scales.shape != ((N + 127) // 128, (K + 127) // 128):
                raise ValueError(f"problem {i}: q / scales shapes do not match X")
            yd = 0
            if Y is not None:
                _need_cuda(Y, "Y")
                if Y.shape != (M, N):
                    raise ValueError(f"problem {i}: Y must be [{M}, {N}]")
                yd = {torch.float32: 0, torch.bfloat16: 1}[Y.dtype]
            arr[i] = L.Fp8Problem(_ptr(X), _ptr(q), _ptr(scales), N, K, _ptr(Y), yd)
            self._keep.extend([X, q, scales, Y])
        vs = None
        if verify is not None:
            drafts, amax, acc, vmax = verify[:4]
            parents, node = (tuple(verify[4:]) + (None, None))[:2]
            _need_cuda(drafts, "drafts", torch.int32)
            B, D = drafts.shape
            if parents is not None:
                _need_cuda(parents, "parents", torch.int32)
                if parents.shape != (B, D):
                    raise ValueError("parents must have the shape of drafts")
            vs = L.VerifySpec(_ptr(drafts) if drafts.numel() else None, B, D, _ptr(amax), _ptr(acc), _ptr(vmax),
                              _ptr(parents) if parents is not None and parents.numel() else None, _ptr(node))
            self._keep.extend([drafts, amax, acc, vmax, parents, node])
        kp = FP8_PATHS[path]
        nbytes = int(lib().fp8_pass_workspace_bytes_path(arr, n, M, 1 if verify is not None else 0, kp))
        if nbytes == 0:
            raise NVFP4WSError(1, "fp8_pass_workspace_bytes")
        dev = problems[0][0].device
        self.workspace = _workspace(nbytes, dev, workspace)
        self.workspace_bytes = nbytes
        self.state = L.PassState()
        _check(lib().fp8_pass_init_path(ctypes.byref(self.state), arr, n, M,
                                        ctypes.byref(vs) if vs is not None else None, kp, _ptr(self.workspace),
                                        nbytes), "fp8_pass_init")
        self.M = M
        self.count = n

    def run(self, stream=None):
        _check(lib().fp8_pass_run(ctypes.byref(self.state), _stream(stream)), "fp8_pass_run")
