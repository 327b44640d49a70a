"""The oracle: a plain fp64 CPU statement of the Gated DeltaNet-2 recurrence.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s
CPU-baseline leg may import this package. The CUDA library never loads it and shares no
code with it; the two meet only through the seeded input generators.

The arithmetic lives in ``gdn2_ref.c`` (one token at a time, fp64); this module only builds
that file with gcc and marshals numpy arrays to it through ctypes. Which passage of the
pages each step follows is stated in ``gdn2_ref.c``.

``prologue_ref`` states the fused pre-processing (raw projections to q, k, log_alpha, b, w)
in numpy, fp64; ``tests/test_oracle_prologue.py`` pins it.

Parity status: every step is pinned by ``tests/test_oracle_pins.py`` (the delta-rule post's
worked example, closed forms, invariants and brute force); the one reading the pages leave
open -- which side of the erase term carries b -- is pinned to the adopted form only by a
hand-computed case.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn2_ref.c")
_SO = os.path.join(_HERE, "libgdn2_ref.so")
_lib = None

F32, BF16 = 0, 1


def build(force: bool = False) -> str:
    """Compile gdn2_ref.c into libgdn2_ref.so with gcc (OpenMP). Returns the .so path."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", _SO, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _SO


def load():
    """Load the oracle library. GDN2_ORACLE_LIB names another build of gdn2_ref.c to load
    instead (the mutation test uses it to check that the pins catch planted mistakes)."""
    global _lib
    if _lib is None:
        override = os.environ.get("GDN2_ORACLE_LIB")
        if not override:
            build()
        lib = ctypes.CDLL(override or _SO)
        lib.gdn2_fwd_ref.restype = ctypes.c_int
        vp = ctypes.c_void_p
        lib.gdn2_fwd_ref.argtypes = [ctypes.c_int, ctypes.c_int, vp, ctypes.c_int, ctypes.c_int,
                                     ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                     vp, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_int]
        lib.gdn2_ref_max_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def max_threads() -> int:
    return int(load().gdn2_ref_max_threads())


def _as_buffer(x, dtype_code):
    """Return a C-contiguous numpy array whose raw bytes are fp32 or bf16 bit patterns."""
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor: take its exact bits, never round
        import torch
        x = x.detach().cpu().contiguous()
        if x.dtype == torch.bfloat16:
            return np.ascontiguousarray(x.view(torch.int16).numpy().view(np.uint16))
        return np.ascontiguousarray(x.to(torch.float32).numpy())
    x = np.asarray(x)
    if dtype_code == BF16:
        if x.dtype != np.uint16:
            raise TypeError("bf16 oracle inputs must be uint16 bit patterns or torch bf16")
        return np.ascontiguousarray(x)
    return np.ascontiguousarray(x, dtype=np.float32)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def fwd_ref(q, k, v, log_alpha, b, w, S0=None, cu_seqlens=None, n_seq=None,
            bf16=None, n_threads: int = 0, want_state: bool = True):
    """Run the oracle. Shapes: q,k [T,Hqk,dk]; v,w [T,Hv,dv]; log_alpha,b [T,Hv,dk];
    S0 [N,Hv,dk,dv] or None. Returns (o [T,Hv,dv] float64, S_T [N,Hv,dk,dv] float64 or None).

    ``bf16`` selects the element type of q,k,v,b,w (inferred from torch tensors when None).
    ``cu_seqlens`` [N+1] int32 packs N sequences; without it the T tokens are split into
    ``n_seq`` equal sequences (default 1).
    """
    if bf16 is None:
        bf16 = hasattr(q, "dtype") and str(q.dtype) == "torch.bfloat16"
    code = BF16 if bf16 else F32
    qa, ka, va, ba, wa = (_as_buffer(t, code) for t in (q, k, v, b, w))
    la = _as_buffer(log_alpha, F32).astype(np.float32, copy=False)
    s0 = None if S0 is None else _as_buffer(S0, F32).astype(np.float32, copy=False)
    T, h_qk, dk = qa.shape
    _, h_v, dv = va.shape
    if cu_seqlens is not None:
        cu = np.ascontiguousarray(np.asarray(
            cu_seqlens.cpu() if hasattr(cu_seqlens, "cpu") else cu_seqlens, dtype=np.int32))
        n = cu.shape[0] - 1
    else:
        cu = None
        n = 1 if n_seq is None else int(n_seq)
    o = np.empty((T, h_v, dv), dtype=np.float64)
    st = np.empty((n, h_v, dk, dv), dtype=np.float64) if want_state else None
    rc = load().gdn2_fwd_ref(n, T, _ptr(cu), h_qk, h_v, dk, dv, code,
                             _ptr(qa), _ptr(ka), _ptr(va), _ptr(la), _ptr(ba), _ptr(wa),
                             _ptr(s0), _ptr(o), _ptr(st), int(n_threads))
    if rc != 0:
        raise ValueError(f"gdn2_fwd_ref rejected its arguments (status {rc})")
    return o, st


def _f64(x):
    if hasattr(x, "detach"):
        return x.detach().double().cpu().numpy()
    return np.asarray(x, dtype=np.float64)


def prologue_ref(q_raw, k_raw, a_raw, b_raw, w_raw, eps: float = 1e-12):
    """The fused pre-processing, fp64: from raw projections to the recurrence's inputs.

      q = q_raw / max(|q_raw|_2, eps), k likewise, per token and head over the key axis.
          The delta-rule post (ai-systems-engineering.com, section on the correction
          strength beta) notes that re-reading the correction with the same key scales it by
          k^T k, so the edit lands exactly only for unit-length keys.
      log_alpha = -softplus(a_raw) = -log(1 + e^a): a decay alpha = 1 / (1 + e^a) in (0, 1).
      b = sigmoid(b_raw), w = sigmoid(w_raw): gates in (0, 1), computed from the input (the
          same section: the strength is produced from the input rather than fixed).
    The pages name no activation functions; softplus and sigmoid are the reading adopted
    here. Inputs: q_raw, k_raw [T, Hqk, dk]; a_raw, b_raw [T, Hv, dk]; w_raw [T, Hv, dv]
    (torch tensors or arrays). Returns float64 arrays (q, k, log_alpha, b, w)."""
    q, k, a, b, w = (_f64(x) for x in (q_raw, k_raw, a_raw, b_raw, w_raw))
    qn = q / np.maximum(np.sqrt(np.sum(q * q, axis=-1, keepdims=True)), eps)
    kn = k / np.maximum(np.sqrt(np.sum(k * k, axis=-1, keepdims=True)), eps)
    log_alpha = -np.logaddexp(0.0, a)
    with np.errstate(over="ignore"):
        bs = 1.0 / (1.0 + np.exp(-b))
        ws = 1.0 / (1.0 + np.exp(-w))
    return qn, kn, log_alpha, bs, ws


def _recurrence_torch(q, k, v, log_alpha, b, w, S0):
    """The recurrence for one sequence in plain torch ops (fp64), token by token, as the
    note on Gated DeltaNet-2 (section "Gated DeltaNet-2 design point") orders its steps:
    decay on the key axis, key read of the decayed state, erase with b on the key axis,
    write with w on the value axis; the delta-rule post has the query read the updated
    state. Shapes: q, k [T, H, dk]; v, w [T, H, dv]; log_alpha, b [T, H, dk]; S0 [H, dk, dv]
    (value heads H; q and k already expanded to them). Returns (o [T, H, dv], S_T)."""
    import torch
    S = S0
    outs = []
    for t in range(q.shape[0]):
        S = torch.exp(log_alpha[t])[:, :, None] * S                       # S' = Diag(alpha) S
        r = torch.einsum("hc,hcm->hm", k[t], S)                           # r = S'^T k
        S = S - (b[t] * k[t])[:, :, None] * r[:, None, :] + k[t][:, :, None] * (w[t] * v[t])[:, None, :]
        outs.append(torch.einsum("hc,hcm->hm", q[t], S))                  # o = S^T q
    return torch.stack(outs), S


def bwd_ref(q, k, v, log_alpha, b, w, dO, S0=None, dS_T=None, cu_seqlens=None, n_seq=None):
    """Gradients of the recurrence by reverse-mode differentiation of its plain fp64
    statement (_recurrence_torch): the loss is sum(o * dO) + sum(S_T * dS_T).

    Shapes as for fwd_ref (q, k [T, Hqk, dk]; v, w [T, Hv, dv]; log_alpha, b [T, Hv, dk];
    S0, dS_T [N, Hv, dk, dv] or None; dO [T, Hv, dv]). Returns float64 arrays
    (dq, dk [T, Hqk, dk]; dv, dw [T, Hv, dv]; dlog_alpha, db [T, Hv, dk]; dS0 [N, Hv, dk, dv]).
    A query/key head's gradient sums over the value heads that read it. Small sizes only."""
    import torch
    f = lambda x: torch.as_tensor(_f64(x))
    q, k, v, la, b, w, dO = (f(x).requires_grad_(True) if i < 6 else f(x)
                             for i, x in enumerate((q, k, v, log_alpha, b, w, dO)))
    T, h_qk, dk = q.shape
    _, h_v, dv = v.shape
    grp = h_v // h_qk
    if cu_seqlens is not None:
        cu = [int(c) for c in np.asarray(cu_seqlens.cpu() if hasattr(cu_seqlens, "cpu") else cu_seqlens)]
    else:
        n = 1 if n_seq is None else int(n_seq)
        cu = [i * (T // n) for i in range(n + 1)]
    N = len(cu) - 1
    S0_t = (f(S0) if S0 is not None else torch.zeros(N, h_v, dk, dv, dtype=torch.float64)).requires_grad_(True)
    loss = 0.0
    for n in range(N):
        s, e = cu[n], cu[n + 1]
        qe = q[s:e].repeat_interleave(grp, dim=1)
        ke = k[s:e].repeat_interleave(grp, dim=1)
        if e > s:
            o, S_T = _recurrence_torch(qe, ke, v[s:e], la[s:e], b[s:e], w[s:e], S0_t[n])
            loss = loss + (o * dO[s:e]).sum()
        else:
            S_T = S0_t[n]
        if dS_T is not None:
            loss = loss + (S_T * f(dS_T)[n]).sum()
    grads = torch.autograd.grad(loss, (q, k, v, la, b, w, S0_t), allow_unused=True)
    return tuple(np.zeros(x.shape) if g_ is None else g_.numpy()
                 for g_, x in zip(grads, (q, k, v, la, b, w, S0_t)))
