"""B200 (sm_100a) fused exact attention (forward and backward) — Python binding.

A thin ctypes layer over the C ABI in ``include/attn.h`` (the in-tree library
``libattn_b200.so``). It only marshals arguments: it checks dtypes, devices and
contiguity, allocates outputs with torch, and passes raw pointers and the
current CUDA stream. Every step of the computation runs in the library's CUDA
kernels; there is no other implementation to fall back to — if the library is
missing or cannot run, the call raises.

    o, lse = attn_fwd(q, k, v, causal=True)          # bf16 [B,H,N,d] on cuda
    dq, dk, dv = attn_bwd(q, k, v, o, lse, do, causal=True)
    o = attention(q, k, v, causal=True); o.backward(do)  # torch autograd
"""
from __future__ import annotations

import ctypes
import math
import os
import threading

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libattn_b200.so")

STATUS_NAMES = {
    0: "ATTN_OK",
    1: "ATTN_ERR_INVALID_ARG",
    2: "ATTN_ERR_UNSUPPORTED",
    3: "ATTN_ERR_ALIGNMENT",
    4: "ATTN_ERR_CUDA",
    5: "ATTN_ERR_TIMEOUT",
    6: "ATTN_ERR_WORKSPACE",
}


class AttnError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)}")


_lib = None
_lock = threading.Lock()

_c_int, _c_float, _vp, _sz = ctypes.c_int, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t
_SIGNATURES = {
    "attn_fwd": (_c_int, [_vp, _vp, _vp, _vp, _vp] + [_c_int] * 7 + [_c_float, _vp]),
    "attn_fwd_varlen": (_c_int, [_vp] * 7 + [_c_int] * 8 + [_c_float, _vp]),
    "attn_fwd_partial": (_c_int, [_vp] * 5 + [_c_int] * 7 + [_c_float, _c_int, _vp]),
    "attn_merge_partials": (_c_int, [_vp, _vp] + [_c_int] * 5 + [_vp, _vp, _vp]),
    "attn_partial_packed_floats": (ctypes.c_longlong, [_c_int] * 4),
    "attn_merge_partials_packed": (_c_int, [_vp] + [_c_int] * 5 + [_vp, _vp, _vp]),
    "attn_fwd_splitkv_num_splits": (_c_int, [_c_int] * 7),
    "attn_fwd_splitkv_workspace_size": (_sz, [_c_int] * 7),
    "attn_fwd_splitkv": (_c_int, [_vp] * 5 + [_c_int] * 7 + [_c_float, _c_int, _vp, _sz, _vp]),
    "attn_fwd_partial_splitkv": (_c_int, [_vp] * 5 + [_c_int] * 7 + [_c_float, _c_int, _c_int, _vp, _sz, _vp]),
    "attn_fwd_host_buffer_size": (_sz, [_c_int] * 6),
    "attn_fwd_host": (_c_int, [_vp, _vp, _vp, _vp, _vp] + [_c_int] * 7 + [_c_float, _vp, _sz, _vp]),
    "attn_fwd_q8_workspace_size": (_sz, [_c_int] * 6),
    "attn_fwd_q8": (_c_int, [_vp, _vp, _vp, _vp, _vp] + [_c_int] * 7 + [_c_float, _vp, _sz, _vp]),
    "attn_q8_prepass": (_c_int, [_vp, _vp, _vp] + [_c_int] * 6 + [_vp, _sz, _vp]),
    "attn_fwd_fp8": (_c_int, [_vp, _vp, _vp, _vp, _vp] + [_c_int] * 7 + [_c_float, _vp, _sz, _vp]),
    "attn_fp8_prepass": (_c_int, [_vp, _vp, _vp] + [_c_int] * 6 + [_vp, _sz, _vp]),
    "attn_q8_workspace_offsets": (_c_int, [_c_int] * 6 + [ctypes.POINTER(_sz)]),
    "attn_bwd_workspace_size": (_sz, [_c_int] * 6),
    "attn_bwd": (_c_int, [_vp] * 9 + [_c_int] * 7 + [_c_float, _vp, _sz, _vp]),
    "attn_bwd_varlen_workspace_size": (_sz, [_c_int] * 4),
    "attn_bwd_varlen": (_c_int, [_vp] * 11 + [_c_int] * 9 + [_c_float, _vp, _sz, _vp]),
    "attn_selftest_wait_timeout": (_c_int, [_c_int, _vp]),
    "attn_get_status": (_c_int, [_vp]),
    "attn_get_status_ex": (_c_int, [_vp, ctypes.POINTER(_c_int)]),
    "attn_set_timeout_ms": (_c_int, [_c_int]),
    "attn_status_string": (ctypes.c_char_p, [_c_int]),
    "attn_version": (_c_int, []),
    "attn_last_cuda_error": (_c_int, [ctypes.POINTER(ctypes.c_char_p)]),
}


def lib() -> ctypes.CDLL:
    """Load (once) and return the C library; raises if it was never built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"CUDA library not built: {LIB_PATH} is missing "
                    "(run `python -m exact_attention_134_b200.build`)")
            l = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in _SIGNATURES.items():
                fn = getattr(l, name)
                fn.restype = res
                fn.argtypes = args
            _lib = l
    return _lib


def _check(status: int, what: str):
    if status != 0:
        if status == 4:
            msg = ctypes.c_char_p()
            code = lib().attn_last_cuda_error(ctypes.byref(msg))
            what = f"{what} (cuda error {code}: {msg.value.decode() if msg.value else ''})"
        raise AttnError(status, what)


def _stream_handle(device=None) -> int:
    import torch
    return torch.cuda.current_stream(device).cuda_stream


def _shape_args(q, k, v):
    if q.dim() != 4 or k.dim() != 4 or v.dim() != 4:
        raise ValueError("q, k, v must be [B, H, N, d]")
    B, Hq, Nq, d = q.shape
    Bk, Hkv, Nkv, dk = k.shape
    if tuple(v.shape) != tuple(k.shape) or Bk != B or dk != d:
        raise ValueError(f"shape mismatch: q {tuple(q.shape)} k {tuple(k.shape)} v {tuple(v.shape)}")
    return B, Hq, Hkv, Nq, Nkv, d


def attn_fwd(q, k, v, causal: bool = False, scale: float | None = None, out=None, lse=None):
    """Fused exact attention forward on the GPU.

    q: bf16 cuda [B, Hq, Nq, d]; k, v: bf16 cuda [B, Hkv, Nkv, d] (contiguous).
    Returns (o bf16 [B, Hq, Nq, d], lse fp32 [B, Hq, Nq]) with
    lse = ln sum_j exp(scale * q.k_j) (scale defaults to 1/sqrt(d)).
    """
    import torch
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor")
    B, Hq, Hkv, Nq, Nkv, d = _shape_args(q, k, v)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    st = lib().attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                        B, Hq, Hkv, Nq, Nkv, d, int(bool(causal)), float(scale),
                        _stream_handle(q.device))
    _check(st, "attn_fwd")
    return out, lse


def _check_qkv(q, k, v):
    import torch
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor")
    return _shape_args(q, k, v)


def attn_fwd_partial(q, k, v, causal: bool = False, scale: float | None = None, kv_tail: int = 0,
                     out=None, lse=None, num_splits: int = 0, workspace=None):
    """Attention of all rows of q over the keys of k, v, which are one range of
    a longer key sequence with `kv_tail` more keys after it (the causal mask is
    that sequence's, bottom-right aligned). Returns the range's normalised
    partial result (o fp32 [B, Hq, Nq, d], lse fp32 [B, Hq, Nq]; -inf and
    O = 0 for a row that sees none of its keys), for merge_partials.

    num_splits: sub-ranges of the keys run as separate CTAs and merged on the
    device (attn_fwd_partial_splitkv); <= 0 picks one wave's worth, 1 is the
    single-launch attn_fwd_partial. workspace: a uint8 CUDA buffer of the
    library's attn_fwd_splitkv_workspace_size bytes (allocated here if None and
    needed)."""
    import torch
    B, Hq, Hkv, Nq, Nkv, d = _check_qkv(q, k, v)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((B, Hq, Nq, d), dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    need = 0 if num_splits == 1 else int(lib().attn_fwd_splitkv_workspace_size(B, Hq, Hkv, Nq, Nkv, d,
                                                                                 int(num_splits)))
    if need == 0:
        st = lib().attn_fwd_partial(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                    lse.data_ptr(), B, Hq, Hkv, Nq, Nkv, d, int(bool(causal)),
                                    float(scale), int(kv_tail), _stream_handle(q.device))
        _check(st, "attn_fwd_partial")
        return out, lse
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    st = lib().attn_fwd_partial_splitkv(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                        lse.data_ptr(), B, Hq, Hkv, Nq, Nkv, d, int(bool(causal)),
                                        float(scale), int(kv_tail), int(num_splits),
                                        workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                        _stream_handle(q.device))
    _check(st, "attn_fwd_partial_splitkv")
    return out, lse


def merge_partials(o_parts, lse_parts, out=None, lse=None):
    """Exact merge of partial results over disjoint key ranges:
    o_parts fp32 cuda [S, B, Hq, Nq, d], lse_parts fp32 cuda [S, B, Hq, Nq]
    -> (o bf16 [B, Hq, Nq, d], lse fp32 [B, Hq, Nq])."""
    import torch
    if o_parts.dtype != torch.float32 or lse_parts.dtype != torch.float32 or \
            not o_parts.is_cuda or not lse_parts.is_cuda or \
            not o_parts.is_contiguous() or not lse_parts.is_contiguous():
        raise ValueError("o_parts and lse_parts must be contiguous fp32 CUDA tensors")
    if o_parts.dim() != 5 or tuple(lse_parts.shape) != tuple(o_parts.shape[:4]):
        raise ValueError("o_parts must be [S, B, Hq, Nq, d] and lse_parts [S, B, Hq, Nq]")
    S, B, Hq, Nq, d = o_parts.shape
    if out is None:
        out = torch.empty((B, Hq, Nq, d), dtype=torch.bfloat16, device=o_parts.device)
    if lse is None:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=o_parts.device)
    st = lib().attn_merge_partials(o_parts.data_ptr(), lse_parts.data_ptr(), S, B, Hq, Nq, d,
                                   out.data_ptr(), lse.data_ptr(), _stream_handle(o_parts.device))
    _check(st, "attn_merge_partials")
    return out, lse


def partial_packed_floats(B, Hq, Nq, d) -> int:
    """Floats per part of the packed partial layout: fp32 O [B, Hq, Nq, d], then
    fp32 LSE [B, Hq, Nq], padded to a multiple of 4."""
    return int(lib().attn_partial_packed_floats(B, Hq, Nq, d))


def merge_partials_packed(parts, B, Hq, Nq, d, out=None, lse=None):
    """merge_partials over parts packed one after another (fp32 cuda
    [S, partial_packed_floats(B, Hq, Nq, d)], each part = O then LSE), the layout
    one all-gather of every rank's packed partial produces.
    -> (o bf16 [B, Hq, Nq, d], lse fp32 [B, Hq, Nq])."""
    import torch
    stride = partial_packed_floats(B, Hq, Nq, d)
    if parts.dtype != torch.float32 or not parts.is_cuda or not parts.is_contiguous() or \
            parts.dim() != 2 or parts.shape[1] != stride:
        raise ValueError(f"parts must be a contiguous fp32 CUDA tensor [S, {stride}]")
    if out is None:
        out = torch.empty((B, Hq, Nq, d), dtype=torch.bfloat16, device=parts.device)
    if lse is None:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=parts.device)
    st = lib().attn_merge_partials_packed(parts.data_ptr(), parts.shape[0], B, Hq, Nq, d,
                                          out.data_ptr(), lse.data_ptr(), _stream_handle(parts.device))
    _check(st, "attn_merge_partials_packed")
    return out, lse


def splitkv_num_splits(B, Hq, Hkv, Nq, Nkv, d, num_splits: int = 0) -> int:
    """Key ranges attn_fwd_splitkv uses (num_splits <= 0: its automatic choice)."""
    return int(lib().attn_fwd_splitkv_num_splits(B, Hq, Hkv, Nq, Nkv, d, int(num_splits)))


def attn_fwd_splitkv(q, k, v, causal: bool = False, scale: float | None = None,
                     num_splits: int = 0, workspace=None, out=None, lse=None):
    """attn_fwd with the keys split into ranges computed by separate CTAs and
    merged (for few query rows per head against many keys). Same tensors and
    results as attn_fwd (d = 64, 96 or 128)."""
    import torch
    B, Hq, Hkv, Nq, Nkv, d = _check_qkv(q, k, v)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    need = int(lib().attn_fwd_splitkv_workspace_size(B, Hq, Hkv, Nq, Nkv, d, int(num_splits)))
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_len = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = lib().attn_fwd_splitkv(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                lse.data_ptr(), B, Hq, Hkv, Nq, Nkv, d, int(bool(causal)),
                                float(scale), int(num_splits), ws_ptr, ws_len,
                                _stream_handle(q.device))
    _check(st, "attn_fwd_splitkv")
    return out, lse


def attn_fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int, causal: bool = False,
                    scale: float | None = None, out=None, lse=None):
    """Packed variable-length attention on the GPU.

    q: bf16 cuda [total_q, Hq, d]; k, v: bf16 cuda [total_k, Hkv, d];
    cu_seqlens_q / cu_seqlens_k: int32 cuda [num_seqs + 1] row offsets.
    Returns (o bf16 [total_q, Hq, d], lse fp32 [Hq, total_q]).
    """
    import torch
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous() or t.dim() != 3:
            raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor [total, H, d]")
    for name, t in (("cu_seqlens_q", cu_seqlens_q), ("cu_seqlens_k", cu_seqlens_k)):
        if t.dtype != torch.int32 or not t.is_cuda or not t.is_contiguous() or t.dim() != 1:
            raise ValueError(f"{name} must be a contiguous int32 CUDA vector")
    if cu_seqlens_q.numel() != cu_seqlens_k.numel() or cu_seqlens_q.numel() < 2:
        raise ValueError("cu_seqlens_q and cu_seqlens_k must both hold num_seqs + 1 offsets")
    total_q, Hq, d = q.shape
    total_k, Hkv, dk = k.shape
    if tuple(v.shape) != tuple(k.shape) or dk != d:
        raise ValueError("shape mismatch between q and k/v")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((Hq, total_q), dtype=torch.float32, device=q.device)
    st = lib().attn_fwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                               cu_seqlens_q.data_ptr(), cu_seqlens_k.data_ptr(),
                               cu_seqlens_q.numel() - 1, int(max_seqlen_q), total_q, total_k, Hq, Hkv, d,
                               int(bool(causal)), float(scale), _stream_handle(q.device))
    _check(st, "attn_fwd_varlen")
    return out, lse


def bwd_workspace_size(B, Hq, Hkv, Nq, Nkv, d) -> int:
    return int(lib().attn_bwd_workspace_size(B, Hq, Hkv, Nq, Nkv, d))


def attn_bwd(q, k, v, o, lse, dout, causal: bool = False, scale: float | None = None,
             workspace=None, dq=None, dk=None, dv=None):
    """Gradients of attn_fwd on the GPU.

    q, o, dout: bf16 cuda [B, Hq, Nq, d]; k, v: bf16 cuda [B, Hkv, Nkv, d];
    lse: fp32 cuda [B, Hq, Nq] (the forward's). Returns (dq, dk, dv) in the
    layouts of q, k, v. `workspace` (uint8 cuda, >= bwd_workspace_size bytes)
    is allocated when not given.
    """
    import torch
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dout", dout)):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor")
    B, Hq, Hkv, Nq, Nkv, d = _shape_args(q, k, v)
    if tuple(o.shape) != tuple(q.shape) or tuple(dout.shape) != tuple(q.shape):
        raise ValueError("o and dout must have the shape of q")
    if lse.dtype != torch.float32 or not lse.is_cuda or not lse.is_contiguous() or \
            tuple(lse.shape) != (B, Hq, Nq):
        raise ValueError("lse must be a contiguous fp32 CUDA tensor [B, Hq, Nq]")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    need = bwd_workspace_size(B, Hq, Hkv, Nq, Nkv, d)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    st = lib().attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                        dout.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                        B, Hq, Hkv, Nq, Nkv, d, int(bool(causal)), float(scale),
                        workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                        _stream_handle(q.device))
    _check(st, "attn_bwd")
    return dq, dk, dv


def attn_bwd_varlen(q, k, v, o, lse, dout, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int,
                    max_seqlen_k: int, causal: bool = False, scale: float | None = None,
                    workspace=None, dq=None, dk=None, dv=None):
    """Gradients of attn_fwd_varlen on the GPU (packed sequences).

    q, o, dout: bf16 cuda [total_q, Hq, d]; k, v: [total_k, Hkv, d]; lse: fp32
    [Hq, total_q] (the varlen forward's); cu_seqlens_*: int32 cuda
    [num_seqs + 1]. Returns (dq, dk, dv) in the layouts of q, k, v.
    """
    import torch
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dout", dout)):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous() or t.dim() != 3:
            raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor [total, H, d]")
    for name, t in (("cu_seqlens_q", cu_seqlens_q), ("cu_seqlens_k", cu_seqlens_k)):
        if t.dtype != torch.int32 or not t.is_cuda or not t.is_contiguous() or t.dim() != 1:
            raise ValueError(f"{name} must be a contiguous int32 CUDA vector")
    if cu_seqlens_q.numel() != cu_seqlens_k.numel() or cu_seqlens_q.numel() < 2:
        raise ValueError("cu_seqlens_q and cu_seqlens_k must both hold num_seqs + 1 offsets")
    total_q, Hq, d = q.shape
    total_k, Hkv, dk_ = k.shape
    if tuple(v.shape) != tuple(k.shape) or dk_ != d or tuple(o.shape) != tuple(q.shape) or \
            tuple(dout.shape) != tuple(q.shape):
        raise ValueError("shape mismatch")
    if lse.dtype != torch.float32 or not lse.is_cuda or tuple(lse.shape) != (Hq, total_q):
        raise ValueError("lse must be a contiguous fp32 CUDA tensor [Hq, total_q]")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    n = cu_seqlens_q.numel() - 1
    if workspace is None:
        need = int(lib().attn_bwd_varlen_workspace_size(n, Hq, int(max_seqlen_q), d))
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    st = lib().attn_bwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                               dout.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                               cu_seqlens_q.data_ptr(), cu_seqlens_k.data_ptr(), n, int(max_seqlen_q),
                               int(max_seqlen_k), total_q, total_k, Hq, Hkv, d, int(bool(causal)),
                               float(scale), workspace.data_ptr(),
                               workspace.numel() * workspace.element_size(), _stream_handle(q.device))
    _check(st, "attn_bwd_varlen")
    return dq, dk, dv


_AUTOGRAD_FN = None


def _autograd_fn():
    """torch.autograd.Function over attn_fwd / attn_bwd (created on first use
    so that importing this module does not import torch)."""
    global _AUTOGRAD_FN
    if _AUTOGRAD_FN is None:
        import torch

        class _Attention(torch.autograd.Function):
            @staticmethod
            def forward(ctx, q, k, v, causal, scale):
                o, lse = attn_fwd(q, k, v, causal=causal, scale=scale)
                ctx.save_for_backward(q, k, v, o, lse)
                ctx.causal, ctx.scale = causal, scale
                return o

            @staticmethod
            def backward(ctx, do):
                q, k, v, o, lse = ctx.saved_tensors
                dq, dk, dv = attn_bwd(q, k, v, o, lse, do.contiguous(), causal=ctx.causal, scale=ctx.scale)
                return dq, dk, dv, None, None

        _AUTOGRAD_FN = _Attention
    return _AUTOGRAD_FN


_AUTOGRAD_VARLEN_FN = None


def _autograd_varlen_fn():
    global _AUTOGRAD_VARLEN_FN
    if _AUTOGRAD_VARLEN_FN is None:
        import torch

        class _AttentionVarlen(torch.autograd.Function):
            @staticmethod
            def forward(ctx, q, k, v, cu_q, cu_k, max_q, max_k, causal, scale):
                o, lse = attn_fwd_varlen(q, k, v, cu_q, cu_k, max_q, causal=causal, scale=scale)
                ctx.save_for_backward(q, k, v, o, lse, cu_q, cu_k)
                ctx.args = (max_q, max_k, causal, scale)
                return o

            @staticmethod
            def backward(ctx, do):
                q, k, v, o, lse, cu_q, cu_k = ctx.saved_tensors
                max_q, max_k, causal, scale = ctx.args
                dq, dk, dv = attn_bwd_varlen(q, k, v, o, lse, do.contiguous(), cu_q, cu_k, max_q, max_k,
                                             causal=causal, scale=scale)
                return dq, dk, dv, None, None, None, None, None, None

        _AUTOGRAD_VARLEN_FN = _AttentionVarlen
    return _AUTOGRAD_VARLEN_FN


def attention_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int, max_seqlen_k: int,
                     causal: bool = False, scale: float | None = None):
    """Differentiable attention over packed variable-length sequences: forward
    attn_fwd_varlen, backward attn_bwd_varlen (d = 64, 96 or 128)."""
    return _autograd_varlen_fn().apply(q, k, v, cu_seqlens_q, cu_seqlens_k, int(max_seqlen_q),
                                       int(max_seqlen_k), causal, scale)


def attention(q, k, v, causal: bool = False, scale: float | None = None):
    """Differentiable exact attention for training: the forward is attn_fwd
    (O only; LSE is kept for the backward), the backward attn_bwd. Same
    tensors and head dims as attn_bwd (d = 64, 96 or 128)."""
    return _autograd_fn().apply(q, k, v, causal, scale)


def q8_workspace_size(B, Hq, Hkv, Nq, Nkv, d) -> int:
    return int(lib().attn_fwd_q8_workspace_size(B, Hq, Hkv, Nq, Nkv, d))


def q8_workspace_offsets(B, Hq, Hkv, Nq, Nkv, d) -> list[int]:
    """Byte offsets of the 8-bit workspace regions (q8, k8, v8, sq, sk, sv,
    kbar, qk, K partial sums, V partial maxima) and the total size."""
    arr = (_sz * 11)()
    _check(lib().attn_q8_workspace_offsets(B, Hq, Hkv, Nq, Nkv, d, arr), "attn_q8_workspace_offsets")
    return [int(x) for x in arr]


def attn_fwd_q8(q, k, v, causal: bool = False, scale: float | None = None, workspace=None,
                out=None, lse=None, qk_format: str = "int8"):
    """8-bit attention forward: INT8 Q K^T after K smoothing (``qk_format="int8"``)
    or FP8 e4m3 Q K^T with block scales and no smoothing (``"fp8"``); FP8 P V.

    Same tensors as ``attn_fwd``; ``workspace`` is a uint8 cuda tensor of at
    least ``q8_workspace_size`` bytes (allocated here if None). Returns (o, lse).
    """
    import torch
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor")
    B, Hq, Hkv, Nq, Nkv, d = _shape_args(q, k, v)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if workspace is None:
        workspace = torch.empty(q8_workspace_size(B, Hq, Hkv, Nq, Nkv, d), dtype=torch.uint8,
                                device=q.device)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    if qk_format not in ("int8", "fp8"):
        raise ValueError("qk_format must be 'int8' or 'fp8'")
    fn = lib().attn_fwd_q8 if qk_format == "int8" else lib().attn_fwd_fp8
    st = fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
            B, Hq, Hkv, Nq, Nkv, d, int(bool(causal)), float(scale),
            workspace.data_ptr(), workspace.numel(), _stream_handle(q.device))
    _check(st, "attn_fwd_q8" if qk_format == "int8" else "attn_fwd_fp8")
    return out, lse


def q8_prepass(q, k, v, workspace, qk_format: str = "int8"):
    """Run only the 8-bit prepass (K mean, scales, quantisation) into ``workspace``."""
    B, Hq, Hkv, Nq, Nkv, d = _shape_args(q, k, v)
    fn = lib().attn_q8_prepass if qk_format == "int8" else lib().attn_fp8_prepass
    st = fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), B, Hq, Hkv, Nq, Nkv, d,
            workspace.data_ptr(), workspace.numel(), _stream_handle(q.device))
    _check(st, "8-bit prepass")


def host_buffer_size(B, Hq, Hkv, Nq, Nkv, d) -> int:
    return int(lib().attn_fwd_host_buffer_size(B, Hq, Hkv, Nq, Nkv, d))


def attn_fwd_host(q, k, v, causal: bool = False, scale: float | None = None, dev_buf=None,
                  out=None, lse=None):
    """Same operation on HOST (CPU, ideally pinned) bf16 tensors: the library
    copies inputs to the device buffer ``dev_buf`` (a uint8 cuda tensor of at
    least ``host_buffer_size`` bytes; allocated here if None), computes, copies
    O and LSE back and synchronises. Returns CPU tensors (o, lse)."""
    import torch
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.dtype != torch.bfloat16 or t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous bf16 CPU tensor")
    B, Hq, Hkv, Nq, Nkv, d = _shape_args(q, k, v)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    need = host_buffer_size(B, Hq, Hkv, Nq, Nkv, d)
    if dev_buf is None:
        dev_buf = torch.empty(need, dtype=torch.uint8, device="cuda")
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32)
    st = lib().attn_fwd_host(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                             B, Hq, Hkv, Nq, Nkv, d, int(bool(causal)), float(scale),
                             dev_buf.data_ptr(), dev_buf.numel(), _stream_handle(dev_buf.device))
    _check(st, "attn_fwd_host")
    return out, lse


def selftest_wait_timeout(budget_us: int) -> None:
    """Queue the failure-detection self-test (a bounded wait that must time out
    after budget_us and record ATTN_ERR_TIMEOUT, where = 0xF00)."""
    _check(lib().attn_selftest_wait_timeout(int(budget_us), _stream_handle()), "attn_selftest_wait_timeout")


def get_status(stream: int | None = None) -> tuple[int, int]:
    """Synchronise the stream and return (status, where) from the device status word."""
    where = ctypes.c_int(0)
    s = lib().attn_get_status_ex(_stream_handle() if stream is None else stream, ctypes.byref(where))
    return int(s), int(where.value)


def set_timeout_ms(ms: int):
    _check(lib().attn_set_timeout_ms(int(ms)), "attn_set_timeout_ms")


def version() -> int:
    return int(lib().attn_version())
