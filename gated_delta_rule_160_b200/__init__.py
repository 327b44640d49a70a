"""libgdn2: the Gated DeltaNet-2 state recurrence on B200 (sm_100a).

This package is a thin ctypes binding over the C ABI declared in ``include/gdn2.h``; every
step of the recurrence runs in the CUDA kernels of ``libgdn2.so``. PyTorch provides device
memory and streams only. There is no CPU fallback: if the library is missing or fails to
load, importing the functions below raises.

    gdn2_chunk_fwd(q, k, v, log_alpha, b, w, S0=None, cu_seqlens=None, ...) -> (o, S_T)
        (prologue=True: raw projections in, the pre-processing fused)
    gdn2_decode_step(q, k, v, log_alpha, b, w, S, o=None) -> o     (S updated in place)
    gdn2_decode_multi(q, k, v, log_alpha, b, w, S_pool, slots=None, ...) -> (o, S_steps)
    gdn2_chunk_bwd(q, k, v, log_alpha, b, w, dO, S0=None, dS_T=None, ...)
        -> (dq, dk, dv, dlog_alpha, db, dw, dS0)
    gdn2_device_status(stream=None) -> int   (device-side error bits, read and cleared)
"""
from __future__ import annotations

import contextlib
import ctypes
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libgdn2.so")

GDN2_F32, GDN2_BF16 = 0, 1
GDN2_DECODE_MAX_TOKENS = 8  # tokens per sequence in one gdn2_decode_multi call (gdn2.h)
STATUS = {0: "GDN2_OK", 1: "GDN2_ERR_INVALID_ARG", 2: "GDN2_ERR_UNSUPPORTED", 3: "GDN2_ERR_CUDA"}
ABI_FUNCTIONS = ("gdn2_chunk_fwd_workspace_size", "gdn2_chunk_fwd", "gdn2_chunk_fwd_prologue",
                 "gdn2_chunk_fwd_noalloc", "gdn2_decode_step", "gdn2_decode_multi",
                 "gdn2_decode_multi_prologue", "gdn2_chunk_bwd_workspace_size", "gdn2_chunk_bwd",
                 "gdn2_device_status", "gdn2_testing_set_wait_limit", "gdn2_last_error_string",
                 "gdn2_version")
# bits of the device status word (gdn2_device_status)
GDN2_DEVICE_WAIT_TIMEOUT, GDN2_DEVICE_BAD_SEQLENS, GDN2_DEVICE_BAD_ORDER = 0x1, 0x2, 0x4
GDN2_DEVICE_DECAY_RANGE = 0x8  # a pair was recomputed token by token (valid, slower)


class Gdn2Error(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status


class Shape(ctypes.Structure):
    _fields_ = [("n_seq", ctypes.c_int), ("T_total", ctypes.c_int), ("h_qk", ctypes.c_int),
                ("h_v", ctypes.c_int), ("dk", ctypes.c_int), ("dv", ctypes.c_int),
                ("dtype", ctypes.c_int), ("o_dtype", ctypes.c_int)]


_lib = None


def load_library(path: str = LIB_PATH):
    """Load libgdn2.so (built by ``python -m gated_delta_rule_160_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} is not built; run `python -m gated_delta_rule_160_b200.build`")
    lib = ctypes.CDLL(path)
    vp, sz = ctypes.c_void_p, ctypes.c_size_t
    lib.gdn2_chunk_fwd_workspace_size.restype = sz
    lib.gdn2_chunk_fwd_workspace_size.argtypes = [ctypes.POINTER(Shape), ctypes.c_int]
    lib.gdn2_chunk_fwd.restype = ctypes.c_int
    lib.gdn2_chunk_fwd.argtypes = [ctypes.POINTER(Shape)] + [vp] * 10 + [vp, sz, vp]
    lib.gdn2_chunk_fwd_noalloc.restype = ctypes.c_int
    lib.gdn2_chunk_fwd_noalloc.argtypes = [ctypes.POINTER(Shape)] + [vp] * 10 + [vp]
    lib.gdn2_decode_step.restype = ctypes.c_int
    lib.gdn2_decode_step.argtypes = [ctypes.POINTER(Shape)] + [vp] * 9
    lib.gdn2_decode_multi.restype = ctypes.c_int
    lib.gdn2_decode_multi.argtypes = ([ctypes.POINTER(Shape), ctypes.c_int] + [vp] * 8
                                      + [ctypes.c_int, vp, vp, vp])
    lib.gdn2_decode_multi_prologue.restype = ctypes.c_int
    lib.gdn2_decode_multi_prologue.argtypes = lib.gdn2_decode_multi.argtypes
    lib.gdn2_chunk_fwd_prologue.restype = ctypes.c_int
    lib.gdn2_chunk_fwd_prologue.argtypes = lib.gdn2_chunk_fwd.argtypes
    lib.gdn2_chunk_bwd_workspace_size.restype = sz
    lib.gdn2_chunk_bwd_workspace_size.argtypes = [ctypes.POINTER(Shape)]
    lib.gdn2_chunk_bwd.restype = ctypes.c_int
    lib.gdn2_chunk_bwd.argtypes = [ctypes.POINTER(Shape)] + [vp] * 17 + [vp, sz, vp]
    lib.gdn2_device_status.restype = ctypes.c_int
    lib.gdn2_device_status.argtypes = [ctypes.POINTER(ctypes.c_uint), vp]
    lib.gdn2_testing_set_wait_limit.restype = None
    lib.gdn2_testing_set_wait_limit.argtypes = [ctypes.c_ulonglong, ctypes.c_int]
    lib.gdn2_last_error_string.restype = ctypes.c_char_p
    lib.gdn2_last_error_string.argtypes = []
    lib.gdn2_version.restype = ctypes.c_int
    _lib = lib
    return lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _on(stream):
    """Tensors allocated inside belong to ``stream``, the stream the call's kernels run on:
    torch's caching allocator then hands a freed workspace (or output) only to later work
    on that stream, never to another stream's work while the kernels still use it."""
    return torch.cuda.stream(stream) if isinstance(stream, torch.cuda.Stream) else contextlib.nullcontext()


def _check(status: int):
    if status != 0:
        msg = load_library().gdn2_last_error_string().decode()
        raise Gdn2Error(status, msg)


def _expect(name, t, shape, dtype=None, device=None, optional=False):
    """Argument check before any launch: the kernels take raw pointers and read each tensor
    densely at the shape the call implies, so a tensor of another shape, strided, on the
    host or of another type would be read out of bounds or misread."""
    if t is None:
        if optional:
            return
        raise ValueError(f"{name} is required")
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if tuple(t.shape) != tuple(int(x) for x in shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(int(x) for x in shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} is {t.dtype}, expected {dtype}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


def _expect_tokens(q, k, v, log_alpha, b, w, lead, prologue=False):
    """q, k [*lead, Hqk, dk]; v, w [*lead, Hv, dv]; log_alpha, b [*lead, Hv, dk], one element
    type for q, k, v, b, w (and for the decay pre-activation with the fused
    pre-processing; log_alpha is fp32 otherwise), all on q's device."""
    for name, t in (("q", q), ("v", v)):
        if not isinstance(t, torch.Tensor) or not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if t.dim() != len(lead) + 2 or tuple(t.shape[:len(lead)]) != tuple(lead):
            raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(lead)} + (heads, channels)")
    h_qk, dk = q.shape[-2:]
    h_v, dv = v.shape[-2:]
    dt, dev = q.dtype, q.device
    _expect("q", q, (*lead, h_qk, dk), dt, dev)
    _expect("k", k, (*lead, h_qk, dk), dt, dev)
    _expect("v", v, (*lead, h_v, dv), dt, dev)
    _expect("log_alpha", log_alpha, (*lead, h_v, dk), dt if prologue else torch.float32, dev)
    _expect("b", b, (*lead, h_v, dk), dt, dev)
    _expect("w", w, (*lead, h_v, dv), dt, dev)
    return h_qk, dk, h_v, dv, dev


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.bfloat16:
        return GDN2_BF16
    if dt == torch.float32:
        return GDN2_F32
    raise TypeError(f"unsupported element type {dt}; use bfloat16 or float32")


def make_shape(q, v, n_seq: int, out_dtype=torch.float32) -> Shape:
    T, h_qk, dk = q.shape
    _, h_v, dv = v.shape
    return Shape(int(n_seq), int(T), int(h_qk), int(h_v), int(dk), int(dv), _dtype_code(v.dtype),
                 _dtype_code(out_dtype))


def gdn2_chunk_fwd_workspace_size(shape: Shape, varlen: bool) -> int:
    return int(load_library().gdn2_chunk_fwd_workspace_size(ctypes.byref(shape), int(bool(varlen))))


def gdn2_chunk_fwd(q, k, v, log_alpha, b, w, S0=None, cu_seqlens=None, n_seq=None,
                   o=None, S_T=None, want_state: bool = True, workspace=None, stream=None,
                   out_dtype=torch.float32, prologue: bool = False):
    """Prefill: run the recurrence over whole (packed) sequences on the GPU.

    q,k [T,Hqk,dk]; v,w [T,Hv,dv]; log_alpha (fp32), b [T,Hv,dk]; S0 fp32 [N,Hv,dk,dv] or
    None; cu_seqlens int32 [N+1] or None (then ``n_seq`` equal sequences, default 1).
    Returns (o [T,Hv,dv] in ``out_dtype`` (or o's dtype when given), S_T fp32 [N,Hv,dk,dv] or
    None). Tensors must be contiguous CUDA tensors; nothing is converted or copied here.
    With ``prologue=True`` q, k, b, w are raw projections and ``log_alpha`` holds the decay
    pre-activation a (same dtype as q): the kernel L2-normalises q and k, takes
    log_alpha = -softplus(a) and sigmoid b, w (gdn2_chunk_fwd_prologue).
    """
    lib = load_library()
    n = (cu_seqlens.numel() - 1) if cu_seqlens is not None else (1 if n_seq is None else int(n_seq))
    if o is not None:
        out_dtype = o.dtype
    T = v.shape[0] if isinstance(v, torch.Tensor) else 0
    h_qk, dk, h_v, dv, dev = _expect_tokens(q, k, v, log_alpha, b, w, (T,), prologue)
    _expect("S0", S0, (n, h_v, dk, dv), torch.float32, dev, optional=True)
    _expect("cu_seqlens", cu_seqlens, (n + 1,), torch.int32, dev, optional=True)
    _expect("o", o, (T, h_v, dv), None, dev, optional=True)
    _expect("S_T", S_T, (n, h_v, dk, dv), torch.float32, dev, optional=True)
    shape = make_shape(q, v, n, out_dtype)
    with _on(stream):
        if o is None:
            o = torch.empty((T, h_v, dv), dtype=out_dtype, device=v.device)
        if S_T is None and want_state:
            S_T = torch.empty((n, h_v, q.shape[2], dv), dtype=torch.float32, device=v.device)
        need = gdn2_chunk_fwd_workspace_size(shape, cu_seqlens is not None)
        if need and workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=v.device)
        ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
        fn = lib.gdn2_chunk_fwd_prologue if prologue else lib.gdn2_chunk_fwd
        _check(fn(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha),
                  _ptr(b), _ptr(w), _ptr(S0), _ptr(cu_seqlens), _ptr(o), _ptr(S_T),
                  _ptr(workspace), ctypes.c_size_t(ws_bytes), _stream_handle(stream)))
    return o, S_T


def gdn2_chunk_fwd_noalloc(q, k, v, log_alpha, b, w, S0=None, cu_seqlens=None, n_seq=None,
                           o=None, S_T=None, stream=None):
    """gdn2_chunk_fwd without a workspace, for callers that cannot allocate device memory:
    the library keeps its packed-batch scratch in a static device array (at most 16384
    sequences per call; calls that run concurrently on the GPU must not overlap). ``o`` and
    ``S_T`` are required here -- this entry point allocates nothing."""
    lib = load_library()
    if o is None or S_T is None:
        raise ValueError("gdn2_chunk_fwd_noalloc writes into caller-provided o and S_T")
    n = (cu_seqlens.numel() - 1) if cu_seqlens is not None else (1 if n_seq is None else int(n_seq))
    T = v.shape[0] if isinstance(v, torch.Tensor) else 0
    h_qk, dk, h_v, dv, dev = _expect_tokens(q, k, v, log_alpha, b, w, (T,))
    _expect("S0", S0, (n, h_v, dk, dv), torch.float32, dev, optional=True)
    _expect("cu_seqlens", cu_seqlens, (n + 1,), torch.int32, dev, optional=True)
    _expect("o", o, (T, h_v, dv), None, dev)
    _expect("S_T", S_T, (n, h_v, dk, dv), torch.float32, dev)
    shape = make_shape(q, v, n, o.dtype)
    _check(lib.gdn2_chunk_fwd_noalloc(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha),
                                      _ptr(b), _ptr(w), _ptr(S0), _ptr(cu_seqlens), _ptr(o), _ptr(S_T),
                                      _stream_handle(stream)))
    return o, S_T


def gdn2_decode_step(q, k, v, log_alpha, b, w, S, o=None, stream=None, out_dtype=torch.float32):
    """One decode token per sequence: q,k [N,Hqk,dk]; v,w [N,Hv,dv]; log_alpha, b [N,Hv,dk];
    S fp32 [N,Hv,dk,dv] updated in place. Returns o [N,Hv,dv] in ``out_dtype``."""
    lib = load_library()
    if o is not None:
        out_dtype = o.dtype
    N = v.shape[0] if isinstance(v, torch.Tensor) else 0
    h_qk, dk, h_v, dv, dev = _expect_tokens(q, k, v, log_alpha, b, w, (N,))
    _expect("S", S, (N, h_v, dk, dv), torch.float32, dev)
    _expect("o", o, (N, h_v, dv), None, dev, optional=True)
    shape = make_shape(q, v, q.shape[0], out_dtype)
    with _on(stream):
        if o is None:
            o = torch.empty(v.shape, dtype=out_dtype, device=v.device)
        _check(lib.gdn2_decode_step(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha),
                                    _ptr(b), _ptr(w), _ptr(S), _ptr(o), _stream_handle(stream)))
    return o


def gdn2_decode_multi(q, k, v, log_alpha, b, w, S_pool, slots=None, o=None, S_steps=None,
                      want_steps: bool = False, stream=None, out_dtype=torch.float32, prologue: bool = False):
    """Serving decode: n_tok new tokens for each of N sequences whose states sit in a pool.

    q,k [N,n_tok,Hqk,dk]; v,w [N,n_tok,Hv,dv]; log_alpha (fp32), b [N,n_tok,Hv,dk];
    S_pool fp32 [n_slots,Hv,dk,dv], updated in place; slots int32 [N] (slot of each
    sequence; negative = inactive, skipped) or None (slot n). Returns (o [N,n_tok,Hv,dv],
    S_steps fp32 [N,n_tok,Hv,dk,dv] -- the state after each token -- or None). ``prologue`` as
    for gdn2_chunk_fwd (gdn2_decode_multi_prologue)."""
    lib = load_library()
    if o is not None:
        out_dtype = o.dtype
    N, n_tok = (v.shape[0], v.shape[1]) if isinstance(v, torch.Tensor) and v.dim() == 4 else (0, 0)
    h_qk, dk, h_v, dv, dev = _expect_tokens(q, k, v, log_alpha, b, w, (N, n_tok), prologue)
    if not isinstance(S_pool, torch.Tensor) or S_pool.dim() != 4:
        raise ValueError("S_pool must be a CUDA tensor [n_slots, Hv, dk, dv]")
    _expect("S_pool", S_pool, (S_pool.shape[0], h_v, dk, dv), torch.float32, dev)
    _expect("slots", slots, (N,), torch.int32, dev, optional=True)
    _expect("o", o, (N, n_tok, h_v, dv), None, dev, optional=True)
    _expect("S_steps", S_steps, (N, n_tok, h_v, dk, dv), torch.float32, dev, optional=True)
    shape = Shape(int(N), int(N * n_tok), int(h_qk), int(h_v), int(dk), int(dv), _dtype_code(v.dtype),
                  _dtype_code(out_dtype))
    with _on(stream):
        if o is None:
            o = torch.empty((N, n_tok, h_v, dv), dtype=out_dtype, device=v.device)
        if S_steps is None and want_steps:
            S_steps = torch.empty((N, n_tok, h_v, dk, dv), dtype=torch.float32, device=v.device)
        fn = lib.gdn2_decode_multi_prologue if prologue else lib.gdn2_decode_multi
        _check(fn(ctypes.byref(shape), int(n_tok), _ptr(slots), _ptr(q), _ptr(k), _ptr(v),
                  _ptr(log_alpha), _ptr(b), _ptr(w), _ptr(S_pool), int(S_pool.shape[0]),
                  _ptr(o), _ptr(S_steps), _stream_handle(stream)))
    return o, S_steps


def gdn2_chunk_bwd(q, k, v, log_alpha, b, w, dO, S0=None, dS_T=None, cu_seqlens=None, n_seq=None,
                   want_dS0: bool = True, workspace=None, stream=None):
    """Gradients of sum(o * dO) + sum(S_T * dS_T) with respect to the forward's inputs.
    Shapes as for gdn2_chunk_fwd; dO fp32 [T,Hv,dv]. Returns fp32 tensors
    (dq, dk, dv, dlog_alpha, db, dw, dS0 or None)."""
    lib = load_library()
    n = (cu_seqlens.numel() - 1) if cu_seqlens is not None else (1 if n_seq is None else int(n_seq))
    T = v.shape[0] if isinstance(v, torch.Tensor) else 0
    h_qk, dk, h_v, dv, dev = _expect_tokens(q, k, v, log_alpha, b, w, (T,))
    _expect("dO", dO, (T, h_v, dv), torch.float32, dev)
    _expect("S0", S0, (n, h_v, dk, dv), torch.float32, dev, optional=True)
    _expect("dS_T", dS_T, (n, h_v, dk, dv), torch.float32, dev, optional=True)
    _expect("cu_seqlens", cu_seqlens, (n + 1,), torch.int32, dev, optional=True)
    shape = make_shape(q, v, n, torch.float32)
    with _on(stream):
        f = lambda t: torch.empty(t.shape, dtype=torch.float32, device=dev)
        dq, dk, dv, dla, db, dw = f(q), f(k), f(v), f(log_alpha), f(b), f(w)
        dS0 = (torch.empty((n, v.shape[1], q.shape[2], v.shape[2]), dtype=torch.float32, device=dev)
               if want_dS0 else None)
        need = int(lib.gdn2_chunk_bwd_workspace_size(ctypes.byref(shape)))
        if workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=dev)
        ws_bytes = workspace.numel() * workspace.element_size()
        _check(lib.gdn2_chunk_bwd(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b),
                                  _ptr(w), _ptr(S0), _ptr(cu_seqlens), _ptr(dO), _ptr(dS_T), _ptr(dq), _ptr(dk),
                                  _ptr(dv), _ptr(dla), _ptr(db), _ptr(dw), _ptr(dS0), _ptr(workspace),
                                  ctypes.c_size_t(ws_bytes), _stream_handle(stream)))
    return dq, dk, dv, dla, db, dw, dS0


class _ChunkFn(torch.autograd.Function):
    """gdn2_chunk_fwd forward, gdn2_chunk_bwd backward (which recomputes the states from the
    saved inputs and S0, so nothing but the inputs is kept)."""

    @staticmethod
    def forward(ctx, q, k, v, log_alpha, b, w, S0, cu_seqlens, n_seq):
        o, S_T = gdn2_chunk_fwd(q, k, v, log_alpha, b, w, S0=S0, cu_seqlens=cu_seqlens, n_seq=n_seq)
        ctx.save_for_backward(q, k, v, log_alpha, b, w, S0, cu_seqlens)
        ctx.n_seq = n_seq
        return o, S_T

    @staticmethod
    def backward(ctx, dO, dS_T):
        q, k, v, log_alpha, b, w, S0, cu_seqlens = ctx.saved_tensors
        dO = torch.zeros(v.shape, dtype=torch.float32, device=v.device) if dO is None else dO.float().contiguous()
        dS_T = None if dS_T is None else dS_T.float().contiguous()
        dq, dk, dv, dla, db, dw, dS0 = gdn2_chunk_bwd(
            q, k, v, log_alpha, b, w, dO, S0=S0, dS_T=dS_T, cu_seqlens=cu_seqlens, n_seq=ctx.n_seq,
            want_dS0=S0 is not None and ctx.needs_input_grad[6])
        like = lambda g_, x: g_.to(x.dtype)
        return (like(dq, q), like(dk, k), like(dv, v), like(dla, log_alpha), like(db, b), like(dw, w), dS0,
                None, None)


def gdn2_chunk(q, k, v, log_alpha, b, w, S0=None, cu_seqlens=None, n_seq=None):
    """gdn2_chunk_fwd as a differentiable op: returns (o fp32, S_T) and, under autograd,
    takes the gradients of every input (and of S0) from gdn2_chunk_bwd, cast to each
    input's dtype. Same shapes and rules as gdn2_chunk_fwd."""
    return _ChunkFn.apply(q, k, v, log_alpha, b, w, S0, cu_seqlens, n_seq)


def gdn2_device_status(stream=None) -> int:
    """Wait for the work queued on ``stream`` (default: the current stream) and return, then
    clear, the device status bits set since the last call (GDN2_DEVICE_* above; 0 = none)."""
    flags = ctypes.c_uint(0)
    _check(load_library().gdn2_device_status(ctypes.byref(flags), _stream_handle(stream)))
    return int(flags.value)
