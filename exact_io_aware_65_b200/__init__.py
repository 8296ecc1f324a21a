"""Exact IO-aware attention (FlashAttention forward and backward) for B200.

A thin ctypes binding over ``libfa.so``: it only checks tensor properties and
marshals pointers, sizes and the CUDA stream into the C ABI declared in
``include/fa.h``.  Every step of the computation runs in the library's CUDA
kernels; there is no fallback path.  PyTorch supplies device memory and
streams.

    O, LSE = fa.fwd(Q, K, V, mask="causal", scale=d ** -0.5)
    dQ, dK, dV = fa.bwd(Q, K, V, O, dO, LSE, mask="causal", scale=d ** -0.5)

Tensors are bf16 [B, H, N, d] contiguous CUDA tensors, LSE is fp32 [B, H, N].
``block_mask`` (mask="block") is a uint8 [ceil(N/128), ceil(N/128)] CUDA
tensor shared by every batch and head.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# FA_LIBRARY selects another build of the same library, e.g. the
# index-checking debug build libfa_debug.so.
LIB_PATH = os.environ.get("FA_LIBRARY") or os.path.join(_HERE, "libfa.so")

MASKS = {"none": 0, "causal": 1, "block": 2}
STATUS = {0: "FA_OK", 1: "FA_ERR_INVALID_ARG", 2: "FA_ERR_UNSUPPORTED", 3: "FA_ERR_CUDA",
          4: "FA_ERR_WORKSPACE", 5: "FA_ERR_TIMEOUT", 6: "FA_ERR_BOUNDS"}

# Every symbol include/fa.h declares, with its ctypes signature.
_vp, _i, _f, _sz, _u64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t, ctypes.c_uint64
SIGNATURES = {
    "fa_fwd": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _f, _vp, _vp, _vp]),
    "fa_bwd_workspace_size": (_sz, [_i, _i, _i, _i]),
    "fa_bwd": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _f, _vp, _vp, _vp, _vp, _sz, _vp]),
    "fa_bwd_stage": (_i, [_i, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _f, _vp, _vp, _vp, _vp,
                          _sz, _vp]),
    "fa_fwd_qk": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _f, _vp, _vp, _vp]),
    "fa_bwd_workspace_size_qk": (_sz, [_i, _i, _i, _i, _i]),
    "fa_bwd_qk": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _f, _vp, _vp, _vp, _vp, _sz,
                       _vp]),
    "fa_bwd_qk_deterministic": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _f, _vp, _vp,
                                     _vp, _vp, _sz, _vp]),
    "fa_fwd_varlen": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _f, _vp, _vp, _vp, _vp, _vp]),
    "fa_bwd_varlen": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _f, _vp, _vp, _i, _vp, _vp,
                           _vp, _vp, _sz, _vp]),
    "fa_decode_workspace_size": (_sz, [_i, _i, _i, _i, _i]),
    "fa_decode": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _vp, _vp, _vp, _sz, _vp]),
    "fa_standard_fwd_workspace_size": (_sz, [_i, _i, _i, _i]),
    "fa_standard_fwd": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _f, _vp, _vp, _vp, _sz, _vp]),
    "fa_bwd_static_workspace": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _f, _vp, _vp,
                                     _vp, _vp]),
    "fa_device_status": (_i, [_vp]),
    "fa_set_wait_timeout_ns": (None, [_u64]),
    "fa_status_string": (ctypes.c_char_p, [_i]),
    "fa_selftest_bounded_wait": (_i, [_u64, _vp]),
    "fa_selftest_mma_tile": (_i, [_vp, _vp, _vp, _i, _i, _i, _vp]),
}


class FAError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {STATUS.get(code, code)}")
        self.code = code


_lib = None


def lib() -> ctypes.CDLL:
    """Load libfa.so (build it first with ``python -m exact_io_aware_65_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise FAError(3, f"CUDA library missing at {LIB_PATH}; build it with "
                             "`python -m exact_io_aware_65_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _check(code: int, what: str):
    if code != 0:
        raise FAError(code, what)


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _mask(mask, block_mask, nbq=None, nbk=None, device=None):
    """Mask kind and block-mask pointer.  The kernels read a row-major
    [nbq, nbk] uint8 grid, so a block mask must hold exactly that many
    entries, contiguous, on the inputs' device."""
    kind = MASKS[mask] if isinstance(mask, str) else int(mask)
    ptr = None
    if kind == MASKS["block"]:
        if block_mask is None or not block_mask.is_cuda or block_mask.dtype != torch.uint8:
            raise FAError(1, "block mask must be a uint8 CUDA tensor")
        if not block_mask.is_contiguous():
            raise FAError(1, "block mask must be contiguous")
        if nbq is not None and block_mask.numel() != nbq * nbk:
            raise FAError(1, f"block mask must hold {nbq} x {nbk} entries (128-row query tiles by "
                             f"128-key tiles), got {tuple(block_mask.shape)}")
        if device is not None and block_mask.device != device:
            raise FAError(1, f"block mask must be on {device}")
        ptr = block_mask.data_ptr()
    return kind, ptr


def _tiles(n):
    return (n + 127) // 128


def _check_buf(t, name, shape, dtype, device):
    """A caller-supplied tensor the kernels read or write through a raw
    pointer: it must have exactly the size the call implies, be contiguous
    and sit on the inputs' device."""
    if not isinstance(t, torch.Tensor):
        raise FAError(1, f"{name} must be a tensor")
    if t.device != device or t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous():
        raise FAError(1, f"{name} must be a contiguous {dtype} tensor of shape {tuple(shape)} on {device}, got "
                         f"{t.dtype} {tuple(t.shape)} on {t.device}" + ("" if t.is_contiguous() else
                                                                       " (not contiguous)"))
    return t


def _workspace(ws, need, device):
    """Device pointer and size in bytes of a caller-supplied workspace."""
    if not isinstance(ws, torch.Tensor) or ws.device != device or not ws.is_contiguous():
        raise FAError(4, f"workspace must be a contiguous tensor on {device}")
    nbytes = ws.numel() * ws.element_size()
    if nbytes < need:
        raise FAError(4, f"workspace holds {nbytes} bytes, the call needs {need}")
    return ws.data_ptr(), nbytes


def _check_qkv(*ts):
    for t in ts:
        if not (isinstance(t, torch.Tensor) and t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous()
                and t.dim() == 4):
            raise FAError(1, "tensors must be contiguous bf16 CUDA tensors [B, H, N, d]")
    if any(t.device != ts[0].device for t in ts):
        raise FAError(1, "all tensors must be on one device")


def _nk(Q, K, V):
    """Key count of K, V [B,H,Nk,d] (heads and head dimension as Q's)."""
    if K.shape != V.shape or K.shape[:2] != Q.shape[:2] or K.shape[3] != Q.shape[3]:
        raise FAError(1, "K and V must be [B, H, Nk, d] with Q's B, H and d")
    return K.shape[2]


def _lens(t, B, device):
    """Device pointer of an optional per-batch-element length vector."""
    if t is None:
        return None
    if not (isinstance(t, torch.Tensor) and t.device == device and t.dtype == torch.int32 and t.is_contiguous()
            and t.numel() == B):
        raise FAError(1, f"sequence lengths must be a contiguous int32 tensor [B] on {device}")
    return t.data_ptr()


def _outputs(Q, N, O, LSE):
    """O [B,H,N,d] bf16 and LSE [B,H,N] fp32: the caller's, checked, or new."""
    B, H, _, d = Q.shape
    O = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=Q.device) if O is None else \
        _check_buf(O, "O", (B, H, N, d), torch.bfloat16, Q.device)
    LSE = torch.empty((B, H, N), dtype=torch.float32, device=Q.device) if LSE is None else \
        _check_buf(LSE, "LSE", (B, H, N), torch.float32, Q.device)
    return O, LSE


def fwd(Q, K, V, mask="none", block_mask=None, scale=None, O=None, LSE=None, stream=None, seqlens_q=None,
        seqlens_k=None):
    """O [B,H,Nq,d] bf16 and LSE [B,H,Nq] fp32 (natural log); K, V are
    [B,H,Nk,d] (Nk may differ from Nq: fa_fwd_qk)."""
    _check_qkv(Q, K, V)
    B, H, N, d = Q.shape
    Nk = _nk(Q, K, V)
    scale = d ** -0.5 if scale is None else float(scale)
    kind, mptr = _mask(mask, block_mask, _tiles(N), _tiles(Nk), Q.device)
    O, LSE = _outputs(Q, N, O, LSE)
    if seqlens_q is not None or seqlens_k is not None:
        _check(lib().fa_fwd_varlen(Q.data_ptr(), K.data_ptr(), V.data_ptr(), B, H, N, Nk, d, kind, mptr, scale,
                                   _lens(seqlens_q, B, Q.device), _lens(seqlens_k, B, Q.device), O.data_ptr(),
                                   LSE.data_ptr(), _stream(stream)), "fa_fwd_varlen")
    elif Nk == N:
        _check(lib().fa_fwd(Q.data_ptr(), K.data_ptr(), V.data_ptr(), B, H, N, d, kind, mptr, scale,
                            O.data_ptr(), LSE.data_ptr(), _stream(stream)), "fa_fwd")
    else:
        _check(lib().fa_fwd_qk(Q.data_ptr(), K.data_ptr(), V.data_ptr(), B, H, N, Nk, d, kind, mptr, scale,
                               O.data_ptr(), LSE.data_ptr(), _stream(stream)), "fa_fwd_qk")
    return O, LSE


def bwd_workspace_size(B, H, N, d, Nk=None) -> int:
    if Nk is None:
        return int(lib().fa_bwd_workspace_size(B, H, N, d))
    return int(lib().fa_bwd_workspace_size_qk(B, H, N, Nk, d))


def _bwd_buffers(Q, K, V, O, dO, LSE, dQ, dK, dV):
    """Checks the backward's inputs beyond Q, K, V and returns its outputs."""
    _check_qkv(Q, K, V, O, dO)
    B, H, N, d = Q.shape
    Nk = _nk(Q, K, V)
    _check_buf(O, "O", Q.shape, torch.bfloat16, Q.device)
    _check_buf(dO, "dO", Q.shape, torch.bfloat16, Q.device)
    _check_buf(LSE, "LSE", (B, H, N), torch.float32, Q.device)
    dQ = torch.empty_like(Q) if dQ is None else _check_buf(dQ, "dQ", Q.shape, torch.bfloat16, Q.device)
    dK = torch.empty_like(K) if dK is None else _check_buf(dK, "dK", K.shape, torch.bfloat16, Q.device)
    dV = torch.empty_like(V) if dV is None else _check_buf(dV, "dV", V.shape, torch.bfloat16, Q.device)
    return Nk, dQ, dK, dV


def bwd(Q, K, V, O, dO, LSE, mask="none", block_mask=None, scale=None, dQ=None, dK=None, dV=None,
        workspace=None, stream=None, deterministic=False, seqlens_q=None, seqlens_k=None):
    """dQ [B,H,Nq,d], dK, dV [B,H,Nk,d] bf16 (Nk may differ from Nq: fa_bwd_qk)."""
    Nk, dQ, dK, dV = _bwd_buffers(Q, K, V, O, dO, LSE, dQ, dK, dV)
    B, H, N, d = Q.shape
    scale = d ** -0.5 if scale is None else float(scale)
    kind, mptr = _mask(mask, block_mask, _tiles(N), _tiles(Nk), Q.device)
    need = bwd_workspace_size(B, H, N, d, Nk)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=Q.device)
    wptr, wbytes = _workspace(workspace, need, Q.device)
    if seqlens_q is not None or seqlens_k is not None:
        _check(lib().fa_bwd_varlen(Q.data_ptr(), K.data_ptr(), V.data_ptr(), O.data_ptr(), dO.data_ptr(),
                                   LSE.data_ptr(), B, H, N, Nk, d, kind, mptr, scale,
                                   _lens(seqlens_q, B, Q.device), _lens(seqlens_k, B, Q.device),
                                   1 if deterministic else 0, dQ.data_ptr(), dK.data_ptr(), dV.data_ptr(), wptr,
                                   wbytes, _stream(stream)), "fa_bwd_varlen")
    elif deterministic:
        _check(lib().fa_bwd_qk_deterministic(Q.data_ptr(), K.data_ptr(), V.data_ptr(), O.data_ptr(), dO.data_ptr(),
                                             LSE.data_ptr(), B, H, N, Nk, d, kind, mptr, scale, dQ.data_ptr(),
                                             dK.data_ptr(), dV.data_ptr(), wptr, wbytes, _stream(stream)),
               "fa_bwd_qk_deterministic")
    elif Nk == N:
        _check(lib().fa_bwd(Q.data_ptr(), K.data_ptr(), V.data_ptr(), O.data_ptr(), dO.data_ptr(),
                            LSE.data_ptr(), B, H, N, d, kind, mptr, scale, dQ.data_ptr(), dK.data_ptr(),
                            dV.data_ptr(), wptr, wbytes, _stream(stream)), "fa_bwd")
    else:
        _check(lib().fa_bwd_qk(Q.data_ptr(), K.data_ptr(), V.data_ptr(), O.data_ptr(), dO.data_ptr(),
                               LSE.data_ptr(), B, H, N, Nk, d, kind, mptr, scale, dQ.data_ptr(), dK.data_ptr(),
                               dV.data_ptr(), wptr, wbytes, _stream(stream)), "fa_bwd_qk")
    return dQ, dK, dV


def bwd_stage(stage, Q, K, V, O, dO, LSE, dQ, dK, dV, workspace, mask="none", block_mask=None,
              scale=None, stream=None):
    """One of the three launches of ``bwd`` (0: prep, 1: main, 2: dQ
    convert); running 0, 1, 2 in order on one workspace equals ``bwd``.
    Self-attention only (K, V with Q's sequence length)."""
    Nk, dQ, dK, dV = _bwd_buffers(Q, K, V, O, dO, LSE, dQ, dK, dV)
    B, H, N, d = Q.shape
    if Nk != N:
        raise FAError(1, "bwd_stage takes K and V with Q's sequence length")
    scale = d ** -0.5 if scale is None else float(scale)
    kind, mptr = _mask(mask, block_mask, _tiles(N), _tiles(N), Q.device)
    wptr, wbytes = _workspace(workspace, bwd_workspace_size(B, H, N, d), Q.device)
    _check(lib().fa_bwd_stage(int(stage), Q.data_ptr(), K.data_ptr(), V.data_ptr(), O.data_ptr(),
                              dO.data_ptr(), LSE.data_ptr(), B, H, N, d, kind, mptr, scale, dQ.data_ptr(),
                              dK.data_ptr(), dV.data_ptr(), wptr, wbytes, _stream(stream)), f"fa_bwd_stage({stage})")


def bwd_static_workspace(Q, K, V, O, dO, LSE, mask="none", block_mask=None, scale=None, dQ=None, dK=None,
                         dV=None, stream=None):
    """``bwd`` with the library's own fixed device scratch instead of a
    workspace (fa_bwd_static_workspace): allocates no workspace; calls whose
    kernels overlap on one device must not use it concurrently."""
    Nk, dQ, dK, dV = _bwd_buffers(Q, K, V, O, dO, LSE, dQ, dK, dV)
    B, H, N, d = Q.shape
    if Nk != N:
        raise FAError(1, "bwd_static_workspace takes K and V with Q's sequence length")
    scale = d ** -0.5 if scale is None else float(scale)
    kind, mptr = _mask(mask, block_mask, _tiles(N), _tiles(N), Q.device)
    _check(lib().fa_bwd_static_workspace(Q.data_ptr(), K.data_ptr(), V.data_ptr(), O.data_ptr(), dO.data_ptr(),
                                         LSE.data_ptr(), B, H, N, d, kind, mptr, scale, dQ.data_ptr(),
                                         dK.data_ptr(), dV.data_ptr(), _stream(stream)), "fa_bwd_static_workspace")
    return dQ, dK, dV


def decode(Q, K, V, mask="none", scale=None, O=None, LSE=None, workspace=None, stream=None):
    """Decode against a KV cache: Q [B,H,Nq,d] (Nq <= 16) against K, V
    [B,H,Nk,d]; returns O [B,H,Nq,d] bf16 and LSE [B,H,Nq] fp32."""
    _check_qkv(Q, K, V)
    B, H, N, d = Q.shape
    Nk = _nk(Q, K, V)
    scale = d ** -0.5 if scale is None else float(scale)
    kind = MASKS[mask] if isinstance(mask, str) else int(mask)
    if kind == MASKS["block"]:
        raise FAError(2, "decode takes no block mask")
    O, LSE = _outputs(Q, N, O, LSE)
    need = decode_workspace_size(B, H, N, Nk, d)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=Q.device)
    wptr, wbytes = _workspace(workspace, need, Q.device)
    _check(lib().fa_decode(Q.data_ptr(), K.data_ptr(), V.data_ptr(), B, H, N, Nk, d, kind, scale, O.data_ptr(),
                           LSE.data_ptr(), wptr, wbytes, _stream(stream)), "fa_decode")
    return O, LSE


def standard_fwd(Q, K, V, mask="none", block_mask=None, scale=None, O=None, LSE=None, workspace=None,
                 stream=None):
    """Standard (materialising) attention, the baseline: O [B,H,N,d] bf16 and
    LSE [B,H,N] fp32, through an N x N score grid in HBM."""
    _check_qkv(Q, K, V)
    B, H, N, d = Q.shape
    if _nk(Q, K, V) != N:
        raise FAError(1, "standard_fwd takes K and V with Q's sequence length")
    scale = d ** -0.5 if scale is None else float(scale)
    kind, mptr = _mask(mask, block_mask, _tiles(N), _tiles(N), Q.device)
    O, LSE = _outputs(Q, N, O, LSE)
    need = standard_fwd_workspace_size(B, H, N, d)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=Q.device)
    wptr, wbytes = _workspace(workspace, need, Q.device)
    _check(lib().fa_standard_fwd(Q.data_ptr(), K.data_ptr(), V.data_ptr(), B, H, N, d, kind, mptr, scale,
                                 O.data_ptr(), LSE.data_ptr(), wptr, wbytes, _stream(stream)), "fa_standard_fwd")
    return O, LSE


def standard_fwd_workspace_size(B, H, N, d) -> int:
    return int(lib().fa_standard_fwd_workspace_size(B, H, N, d))


def decode_workspace_size(B, H, Nq, Nk, d) -> int:
    return int(lib().fa_decode_workspace_size(B, H, Nq, Nk, d))


def device_status(stream=None) -> int:
    """Synchronise and read/clear the device status word (0 = ok, 5 = timeout)."""
    return int(lib().fa_device_status(_stream(stream)))


def set_wait_timeout_ns(ns: int):
    lib().fa_set_wait_timeout_ns(int(ns))


def selftest_bounded_wait(timeout_ns: int, stream=None):
    _check(lib().fa_selftest_bounded_wait(int(timeout_ns), _stream(stream)), "fa_selftest_bounded_wait")


def selftest_mma_tile(A, B, n, k, mode, stream=None):
    """C [128, n] fp32 = A [128, k] times Bt^T with Bt [n, k] (mode 0), or
    times B [k, n] (mode 1), on one tensor-core tile."""
    if not (isinstance(A, torch.Tensor) and A.is_cuda):
        raise FAError(1, "A must be a CUDA tensor")
    _check_buf(A, "A", (128, k), torch.bfloat16, A.device)
    _check_buf(B, "B", (n, k) if mode == 0 else (k, n), torch.bfloat16, A.device)
    C = torch.empty((128, n), dtype=torch.float32, device=A.device)
    _check(lib().fa_selftest_mma_tile(A.data_ptr(), B.data_ptr(), C.data_ptr(), n, k, mode, _stream(stream)),
           "fa_selftest_mma_tile")
    return C
