"""Seeded synthetic inputs for the Gated DeltaNet-2 recurrence.

This module is shared by the GPU path's tests, the benchmark and the oracle checks; it holds
none of the recurrence's arithmetic. Inputs follow the stated recipe: q, k ~ N(0,1) then
L2-normalised per head; v ~ N(0,1); log_alpha = -softplus(N(0,1)) per key channel in fp32;
b, w = sigmoid(N(0,1)) per key / value channel; S0 either zero or N(0, std) in fp32. The
pages fix only the grouped-head counts (16 query/key heads shared by 32 value heads, head
dimension 128, from the Gated DeltaNet wiki page, section "How it works") and the model
scale; everything else is this recipe. Random numbers come from torch's Philox generator
on the target device, seeded per workload, so the same seed gives the same tensors on
every run of the same device type.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch
import torch.nn.functional as F


@dataclass(frozen=True)
class Workload:
    name: str
    description: str
    n_seq: int
    h_qk: int
    h_v: int
    dk: int
    dv: int
    dtype: torch.dtype
    T: int = 0                  # tokens per sequence (fixed-length workloads)
    len_range: tuple = ()       # (lo, hi) inclusive, for packed variable-length workloads
    S0_std: float = 0.0         # 0: zero initial state
    decode_steps: int = 0       # > 0: a decode workload of this many consecutive steps
    seed: int = 0

    @property
    def varlen(self) -> bool:
        return bool(self.len_range)


WORKLOADS = {
    w.name: w for w in [
        Workload("tiny_fp32", "batch 1, 2 heads, T=256, dk=dv=64, fp32, S0=0",
                 n_seq=1, h_qk=2, h_v=2, dk=64, dv=64, dtype=torch.float32, T=256, seed=1001),
        Workload("prefill_b8_h16_t4096", "batch 8, 16 heads, T=4096, dk=dv=128, bf16, S0=0",
                 n_seq=8, h_qk=16, h_v=16, dk=128, dv=128, dtype=torch.bfloat16, T=4096, seed=1002),
        Workload("grouped_b2_qk16_v32_t32768",
                 "batch 2, 16 query/key heads shared by 32 value heads, T=32768, d=128, bf16, S0~N(0,0.02)",
                 n_seq=2, h_qk=16, h_v=32, dk=128, dv=128, dtype=torch.bfloat16, T=32768,
                 S0_std=0.02, seed=1003),
        Workload("varlen_64seq_h16", "64 packed sequences, lengths U[128,8192], 16 heads, d=128, bf16",
                 n_seq=64, h_qk=16, h_v=16, dk=128, dv=128, dtype=torch.bfloat16,
                 len_range=(128, 8192), seed=1004),
        Workload("decode_256seq_h32", "decode: 256 sequences x 32 heads, d=128, S~N(0,0.05), 512 steps",
                 n_seq=256, h_qk=32, h_v=32, dk=128, dv=128, dtype=torch.bfloat16,
                 S0_std=0.05, decode_steps=512, seed=1005),
    ]
}


def seq_lengths(wl: Workload, n_seq: int | None = None) -> list:
    n = wl.n_seq if n_seq is None else n_seq
    if wl.varlen:
        lo, hi = wl.len_range
        return [int(x) for x in np.random.default_rng(wl.seed).integers(lo, hi + 1, size=n)]
    return [wl.T] * n


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _normal(shape, g, device):
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32)


def token_inputs(T: int, h_qk: int, h_v: int, dk: int, dv: int, dtype, device, seed: int):
    """Per-token inputs of the recipe for T packed tokens."""
    g = _gen(device, seed)
    q = F.normalize(_normal((T, h_qk, dk), g, device), dim=-1).to(dtype)
    k = F.normalize(_normal((T, h_qk, dk), g, device), dim=-1).to(dtype)
    v = _normal((T, h_v, dv), g, device).to(dtype)
    log_alpha = -F.softplus(_normal((T, h_v, dk), g, device))
    b = torch.sigmoid(_normal((T, h_v, dk), g, device)).to(dtype)
    w = torch.sigmoid(_normal((T, h_v, dv), g, device)).to(dtype)
    return dict(q=q.contiguous(), k=k.contiguous(), v=v.contiguous(), log_alpha=log_alpha.contiguous(),
                b=b.contiguous(), w=w.contiguous())


def state_input(n_seq: int, h_v: int, dk: int, dv: int, std: float, device, seed: int):
    if std == 0.0:
        return None
    g = _gen(device, seed + 7919)
    return (std * _normal((n_seq, h_v, dk, dv), g, device)).contiguous()


def prefill_inputs(wl: Workload, device="cuda", n_seq: int | None = None, T: int | None = None):
    """Inputs of a prefill workload. ``n_seq`` / ``T`` shrink it (same recipe and seed) for
    tests; varlen workloads take their first ``n_seq`` lengths."""
    n = wl.n_seq if n_seq is None else int(n_seq)
    lens = seq_lengths(wl, n)
    if T is not None:
        lens = [min(L, int(T)) for L in lens] if wl.varlen else [int(T)] * n
    T_total = int(sum(lens))
    d = token_inputs(T_total, wl.h_qk, wl.h_v, wl.dk, wl.dv, wl.dtype, device, wl.seed)
    d["S0"] = state_input(n, wl.h_v, wl.dk, wl.dv, wl.S0_std, device, wl.seed)
    if wl.varlen:
        cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
        d["cu_seqlens"] = torch.from_numpy(cu).to(device)
        d["n_seq"] = None
    else:
        d["cu_seqlens"] = None
        d["n_seq"] = n
    d["lengths"] = lens
    return d


def decode_state(wl: Workload, device="cuda", n_seq: int | None = None):
    n = wl.n_seq if n_seq is None else int(n_seq)
    return state_input(n, wl.h_v, wl.dk, wl.dv, wl.S0_std, device, wl.seed)


def decode_inputs(wl: Workload, step: int, device="cuda", n_seq: int | None = None):
    """Inputs of decode step ``step``: one token for each sequence."""
    n = wl.n_seq if n_seq is None else int(n_seq)
    return token_inputs(n, wl.h_qk, wl.h_v, wl.dk, wl.dv, wl.dtype, device, wl.seed * 100003 + step)


def algorithmic_bytes_per_token_head(wl: Workload) -> int:
    """Bytes a prefill token of one value head must move at least once: q, k (per value head,
    as the unfused layout reads them), v, w, b, log_alpha (fp32) and o."""
    es = torch.finfo(wl.dtype).bits // 8
    return es * (2 * wl.dk + 3 * wl.dv + wl.dk) + 4 * wl.dk
