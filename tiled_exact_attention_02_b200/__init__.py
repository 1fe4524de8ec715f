"""Python binding of libtiledattn.so: argument marshalling only.

Every step of the computation runs in the CUDA kernels behind the C ABI
(include/tiledattn.h).  PyTorch provides device memory and the current
stream.  There is no CPU fallback: if the library is missing, importing the
binding raises.
"""

from __future__ import annotations

import ctypes
import math
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libtiledattn.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "tiledattn.h")

ATTN_OK = 0
ATTN_ERR_INVALID_ARG = 1
ATTN_ERR_UNSUPPORTED = 2
ATTN_ERR_CUDA = 3
ATTN_ERR_TIMEOUT = 4


class AttnError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        msg = f"{what}: {status_string(status)} ({status})"
        if status == ATTN_ERR_CUDA:
            msg += f" [{lib.attn_last_cuda_error().decode()}]"
        super().__init__(msg)


class AttnMask(ctypes.Structure):
    """The C ABI's attn_mask."""
    _fields_ = [("causal", ctypes.c_int), ("window", ctypes.c_int), ("global_head", ctypes.c_int),
                ("global_tail", ctypes.c_int), ("seqlens_q", ctypes.c_void_p), ("seqlens_k", ctypes.c_void_p),
                ("sparse_block", ctypes.c_int)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is not built; run `python tiled_exact_attention_02_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.attn_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, i, vp]
    lib.attn_fwd.restype = i
    lib.attn_fwd_split.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, i, i, vp, sz, vp]
    lib.attn_fwd_split.restype = i
    lib.attn_fwd_split_workspace_size.argtypes = [i, i, i, i, i, i, i]
    lib.attn_fwd_split_workspace_size.restype = sz
    lib.attn_fwd_split_default.argtypes = [i, i, i, i, i, i, i, i]
    lib.attn_fwd_split_default.restype = i
    lib.attn_fwd_varlen.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, i, vp]
    lib.attn_fwd_varlen.restype = i
    lib.attn_bwd_varlen.argtypes = [vp] * 11 + [i] * 6 + [f, i, i, vp, sz, vp]
    lib.attn_bwd_varlen.restype = i
    lib.attn_bwd_main_varlen.argtypes = [vp] * 9 + [i] * 6 + [f, i, i, vp, sz, vp]
    lib.attn_bwd_main_varlen.restype = i
    mp = ctypes.POINTER(AttnMask)
    lib.attn_fwd_ex.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, mp, i, vp, sz, vp]
    lib.attn_fwd_ex.restype = i
    lib.attn_bwd_ex.argtypes = [vp] * 9 + [i] * 6 + [f, mp, vp, sz, vp]
    lib.attn_bwd_ex.restype = i
    lib.attn_bwd_workspace_size.argtypes = [i, i, i, i, i, i]
    lib.attn_bwd_workspace_size.restype = sz
    lib.attn_bwd.argtypes = [vp] * 9 + [i] * 6 + [f, i, i, vp, sz, vp]
    lib.attn_bwd.restype = i
    lib.attn_bwd_preprocess.argtypes = [vp, vp, i, i, i, i, vp, sz, vp]
    lib.attn_bwd_preprocess.restype = i
    lib.attn_bwd_main.argtypes = [vp] * 7 + [i] * 6 + [f, i, i, vp, sz, vp]
    lib.attn_bwd_main.restype = i
    lib.attn_bwd_finalize.argtypes = [vp, i, i, i, i, f, vp, sz, vp]
    lib.attn_bwd_finalize.restype = i
    lib.attn_step_host_buffer_size.argtypes = [i, i, i, i, i, i, i]
    lib.attn_step_host_buffer_size.restype = sz
    lib.attn_step_host.argtypes = [vp] * 9 + [i] * 6 + [f, i, i, vp, sz, vp]
    lib.attn_step_host.restype = i
    lib.attn_last_cuda_error.argtypes = []
    lib.attn_last_cuda_error.restype = ctypes.c_char_p
    lib.attn_status_string.argtypes = [i]
    lib.attn_status_string.restype = ctypes.c_char_p
    lib.attn_get_device_error.argtypes = [vp, ctypes.POINTER(i)]
    lib.attn_get_device_error.restype = i
    lib.attn_selftest_wait_timeout.argtypes = [ctypes.c_int64, vp]
    lib.attn_selftest_wait_timeout.restype = i
    lib.attn_fwd_accumulate.argtypes = [vp] * 5 + [i] * 6 + [f, i, i, i, vp]
    lib.attn_fwd_accumulate.restype = i
    lib.attn_fwd_accumulate_finalize.argtypes = [vp] * 4 + [i] * 4 + [vp]
    lib.attn_fwd_accumulate_finalize.restype = i
    lib.attn_bwd_accumulate.argtypes = [vp] * 7 + [i] * 6 + [f, i, i, i, vp, sz, vp]
    lib.attn_bwd_accumulate.restype = i
    lib.attn_accumulator_to_bf16.argtypes = [vp, vp, sz, vp]
    lib.attn_accumulator_to_bf16.restype = i
    lib.attn_selftest_bwd_abort.argtypes = [vp] * 9 + [i] * 6 + [f, i, i, i, ctypes.c_int64, vp, sz, vp]
    lib.attn_selftest_bwd_abort.restype = i
    lib.attn_selftest_step_host_fail_at.argtypes = [i]
    lib.attn_selftest_step_host_fail_at.restype = i
    return lib


lib = _load()


def status_string(status: int) -> str:
    return lib.attn_status_string(int(status)).decode()


def _stream_ptr(stream) -> int:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


def _check(status: int, what: str) -> None:
    if status != ATTN_OK:
        raise AttnError(status, what)


def _shapes(q, k):
    B, Hq, Lq, d = q.shape
    Bk, Hkv, Lk, dk = k.shape
    if Bk != B or dk != d:
        raise ValueError(f"shape mismatch q{tuple(q.shape)} k{tuple(k.shape)}")
    return B, Hq, Hkv, Lq, Lk, d


def _require(t, name, dtype=None):
    import torch
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")


def _causal_code(causal) -> int:
    """The ABI's mask code: False/0 none, True/1 top-left, 2 or "bottom_right"
    bottom-right alignment (query i at key position i + Lk - Lq)."""
    if isinstance(causal, str):
        codes = {"none": 0, "top_left": 1, "bottom_right": 2}
        if causal not in codes:
            raise ValueError(f"causal must be one of {sorted(codes)}, got {causal!r}")
        return codes[causal]
    return 2 if causal == 2 and not isinstance(causal, bool) else int(bool(causal))


def _lens(seqlens, B, name):
    """Device pointer of optional per-sequence lengths (int32 CUDA tensor [B])."""
    import torch
    if seqlens is None:
        return None
    _require(seqlens, name, torch.int32)
    if tuple(seqlens.shape) != (B,):
        raise ValueError(f"{name} must have shape ({B},)")
    return seqlens.data_ptr()


def fwd(q, k, v, o, lse, causal: bool = False, window: int = 0, scale: float | None = None, stream=None,
        seqlens_q=None, seqlens_k=None, global_head: int = 0, global_tail: int = 0, sparse_block: int = 0):
    """attn_fwd on torch tensors (bf16 q/k/v/o, fp32 lse), asynchronous on
    `stream`; with seqlens_q / seqlens_k (int32 CUDA [B]) attn_fwd_varlen."""
    import torch
    for n, t in (("q", q), ("k", k), ("v", v), ("o", o)):
        _require(t, n, torch.bfloat16)
    _require(lse, "lse", torch.float32)
    B, Hq, Hkv, Lq, Lk, d = _shapes(q, k)
    if tuple(v.shape) != tuple(k.shape) or tuple(o.shape) != tuple(q.shape) or tuple(lse.shape) != (B, Hq, Lq):
        raise ValueError("v/o/lse shape mismatch")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    lq, lk = _lens(seqlens_q, B, "seqlens_q"), _lens(seqlens_k, B, "seqlens_k")
    if global_head or global_tail or sparse_block:
        m = AttnMask(_causal_code(causal), int(window), int(global_head), int(global_tail), lq, lk, int(sparse_block))
        st = lib.attn_fwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                             B, Hq, Hkv, Lq, Lk, d, scale, ctypes.byref(m), 1, None, 0, _stream_ptr(stream))
        _check(st, "attn_fwd_ex")
        return
    if lq is None and lk is None:
        st = lib.attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                          B, Hq, Hkv, Lq, Lk, d, scale, _causal_code(causal), int(window), _stream_ptr(stream))
        _check(st, "attn_fwd")
        return
    st = lib.attn_fwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), lq, lk,
                             B, Hq, Hkv, Lq, Lk, d, scale, _causal_code(causal), int(window), _stream_ptr(stream))
    _check(st, "attn_fwd_varlen")


def bwd_workspace_size(B, Hq, Hkv, Lq, Lk, d) -> int:
    return int(lib.attn_bwd_workspace_size(B, Hq, Hkv, Lq, Lk, d))


def bwd(q, k, v, o, lse, do, dq, dk, dv, workspace, causal: bool = False, window: int = 0,
        scale: float | None = None, stream=None, seqlens_q=None, seqlens_k=None, global_head: int = 0,
        global_tail: int = 0, sparse_block: int = 0):
    """attn_bwd on torch tensors; `workspace` is a uint8 CUDA tensor; with
    seqlens_q / seqlens_k attn_bwd_varlen."""
    import torch
    for n, t in (("q", q), ("k", k), ("v", v), ("o", o), ("do", do), ("dq", dq), ("dk", dk), ("dv", dv)):
        _require(t, n, torch.bfloat16)
    _require(lse, "lse", torch.float32)
    _require(workspace, "workspace")
    B, Hq, Hkv, Lq, Lk, d = _shapes(q, k)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    lq, lk = _lens(seqlens_q, B, "seqlens_q"), _lens(seqlens_k, B, "seqlens_k")
    wsp, wsb = workspace.data_ptr(), workspace.numel() * workspace.element_size()
    if global_head or global_tail or sparse_block:
        m = AttnMask(_causal_code(causal), int(window), int(global_head), int(global_tail), lq, lk, int(sparse_block))
        st = lib.attn_bwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), do.data_ptr(),
                             dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, Hq, Hkv, Lq, Lk, d, scale,
                             ctypes.byref(m), wsp, wsb, _stream_ptr(stream))
        _check(st, "attn_bwd_ex")
        return
    if lq is None and lk is None:
        st = lib.attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), do.data_ptr(),
                          dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, Hq, Hkv, Lq, Lk, d, scale,
                          _causal_code(causal), int(window), wsp, wsb, _stream_ptr(stream))
        _check(st, "attn_bwd")
        return
    st = lib.attn_bwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), do.data_ptr(),
                             dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), lq, lk, B, Hq, Hkv, Lq, Lk, d, scale,
                             _causal_code(causal), int(window), wsp, wsb, _stream_ptr(stream))
    _check(st, "attn_bwd_varlen")


def bwd_phases(q, k, v, o, lse, do, dq, dk, dv, workspace, causal: bool = False, window: int = 0,
               scale: float | None = None, stream=None, between=None):
    """attn_bwd as its three C-ABI phases; `between(i)` (optional) is called
    before phase i (0..2) and after the last (i = 3), e.g. to record events."""
    B, Hq, Hkv, Lq, Lk, d = _shapes(q, k)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    ws, wsb, sp = workspace.data_ptr(), workspace.numel() * workspace.element_size(), _stream_ptr(stream)
    hook = between or (lambda i: None)
    hook(0)
    _check(lib.attn_bwd_preprocess(o.data_ptr(), do.data_ptr(), B, Hq, Lq, d, ws, wsb, sp), "attn_bwd_preprocess")
    hook(1)
    _check(lib.attn_bwd_main(q.data_ptr(), k.data_ptr(), v.data_ptr(), lse.data_ptr(), do.data_ptr(),
                             dk.data_ptr(), dv.data_ptr(), B, Hq, Hkv, Lq, Lk, d, scale, _causal_code(causal),
                             int(window), ws, wsb, sp), "attn_bwd_main")
    hook(2)
    _check(lib.attn_bwd_finalize(dq.data_ptr(), B, Hq, Lq, d, scale, ws, wsb, sp), "attn_bwd_finalize")
    hook(3)


def step_host_buffer_size(B, Hq, Hkv, Lq, Lk, d, with_backward: bool = True) -> int:
    return int(lib.attn_step_host_buffer_size(B, Hq, Hkv, Lq, Lk, d, int(bool(with_backward))))


def step_host(q, k, v, o, lse, buf, do=None, dq=None, dk=None, dv=None, causal: bool = False, window: int = 0,
              scale: float | None = None, stream=None) -> None:
    """attn_step_host: q, k, v (do) and the outputs o, lse (dq, dk, dv) are
    contiguous CPU tensors (pinned for overlapped copies); `buf` is a CUDA
    uint8 tensor of at least step_host_buffer_size bytes.  Asynchronous on
    `stream`: synchronise it before reading the outputs."""
    import torch
    B, Hq, Hkv, Lq, Lk, d = _shapes(q, k)
    host = [("q", q), ("k", k), ("v", v), ("o", o)] + ([("do", do), ("dq", dq), ("dk", dk), ("dv", dv)]
                                                     if do is not None else [])
    for name, t in host:
        if t is None or t.is_cuda or not t.is_contiguous() or t.dtype != torch.bfloat16:
            raise ValueError(f"{name} must be a contiguous bf16 CPU tensor")
    if lse.is_cuda or not lse.is_contiguous() or lse.dtype != torch.float32:
        raise ValueError("lse must be a contiguous float32 CPU tensor")
    _require(buf, "buf", torch.uint8)
    sc = d ** -0.5 if scale is None else scale
    ptr = lambda t: None if t is None else t.data_ptr()
    _check(lib.attn_step_host(q.data_ptr(), k.data_ptr(), v.data_ptr(), ptr(do), o.data_ptr(), lse.data_ptr(),
                              ptr(dq), ptr(dk), ptr(dv), B, Hq, Hkv, Lq, Lk, d, sc, _causal_code(causal),
                              int(window), buf.data_ptr(), buf.numel(), _stream_ptr(stream)), "attn_step_host")


def device_error(stream=None) -> tuple[int, int]:
    """(status, site) of the current device's error word; clears it."""
    site = ctypes.c_int(0)
    st = lib.attn_get_device_error(_stream_ptr(stream), ctypes.byref(site))
    return st, site.value


def attention(q, k, v, causal: bool = False, window: int = 0, scale: float | None = None, seqlens_q=None,
              seqlens_k=None, global_head: int = 0, global_tail: int = 0, sparse_block: int = 0):
    """Allocate O and LSE with torch and run the forward pass."""
    import torch
    B, Hq, Hkv, Lq, Lk, d = _shapes(q, k)
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device=q.device)
    fwd(q, k, v, o, lse, causal, window, scale, seqlens_q=seqlens_q, seqlens_k=seqlens_k, global_head=global_head,
        global_tail=global_tail, sparse_block=sparse_block)
    return o, lse


def fwd_split(q, k, v, o, lse, n_split: int, workspace, causal: bool = False, window: int = 0,
              scale: float | None = None, stream=None):
    """attn_fwd_split: the key range of every query tile cut into n_split
    slices computed by separate CTAs, then merged exactly."""
    B, Hq, Hkv, Lq, Lk, d = _shapes(q, k)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    ws = workspace.data_ptr() if workspace is not None else None
    wsb = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib.attn_fwd_split(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                              B, Hq, Hkv, Lq, Lk, d, scale, _causal_code(causal), int(window), int(n_split), ws, wsb,
                              _stream_ptr(stream)), "attn_fwd_split")


def attention_split(q, k, v, causal: bool = False, window: int = 0, scale: float | None = None,
                    n_split: int | None = None):
    """Allocate O, LSE and the workspace with torch and run the split-KV
    forward (n_split None: the library's suggestion for this shape)."""
    import torch
    B, Hq, Hkv, Lq, Lk, d = _shapes(q, k)
    if n_split is None:
        n_split = lib.attn_fwd_split_default(B, Hq, Hkv, Lq, Lk, d, _causal_code(causal), int(window))
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device=q.device)
    nbytes = lib.attn_fwd_split_workspace_size(B, Hq, Hkv, Lq, Lk, d, int(n_split))
    ws = torch.empty(max(256, nbytes), dtype=torch.uint8, device=q.device)
    fwd_split(q, k, v, o, lse, n_split, ws, causal, window, scale)
    return o, lse


def attention_backward(q, k, v, o, lse, do, causal: bool = False, window: int = 0, scale: float | None = None,
                       seqlens_q=None, seqlens_k=None, global_head: int = 0, global_tail: int = 0,
                       sparse_block: int = 0):
    """Allocate dQ/dK/dV and the workspace with torch and run the backward pass."""
    import torch
    B, Hq, Hkv, Lq, Lk, d = _shapes(q, k)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(max(1, bwd_workspace_size(B, Hq, Hkv, Lq, Lk, d)), dtype=torch.uint8, device=q.device)
    bwd(q, k, v, o, lse, do, dq, dk, dv, ws, causal, window, scale, seqlens_q=seqlens_q, seqlens_k=seqlens_k,
        global_head=global_head, global_tail=global_tail, sparse_block=sparse_block)
    return dq, dk, dv


def _autograd_function():
    import torch

    class TiledAttention(torch.autograd.Function):
        """autograd wrapper: forward saves O and LSE; backward recomputes."""

        @staticmethod
        def forward(ctx, q, k, v, causal=False, window=0, scale=None):
            o, lse = attention(q, k, v, causal, window, scale)
            ctx.save_for_backward(q, k, v, o, lse)
            ctx.args = (causal, window, scale)
            return o

        @staticmethod
        def backward(ctx, do):
            q, k, v, o, lse = ctx.saved_tensors
            dq, dk, dv = attention_backward(q, k, v, o, lse, do.contiguous(), *ctx.args)
            return dq, dk, dv, None, None, None

    return TiledAttention


def tiled_attention(q, k, v, causal: bool = False, window: int = 0, scale: float | None = None):
    """Differentiable attention (torch autograd) backed by the CUDA kernels."""
    global _TiledAttention
    try:
        fn = _TiledAttention
    except NameError:
        fn = _TiledAttention = _autograd_function()
    return fn.apply(q, k, v, causal, window, scale)
