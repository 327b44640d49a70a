"""Helpers for comparing the CUDA path with the oracle (test infrastructure).

Tolerances are the acceptance bounds for this recurrence: max|delta| / rms(reference)
<= 1e-4 for fp32 inputs and <= 2e-2 for bf16 inputs, for the outputs o and for the final
state, with rms taken over the whole compared tensor.
"""
import numpy as np
import torch

TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}


def rel_err(got, ref) -> float:
    """max|got - ref| / rms(ref); got may be a torch tensor (any device), ref numpy fp64."""
    if hasattr(got, "detach"):
        got = got.detach().float().cpu().numpy()
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    if ref.size == 0:
        return 0.0
    rms = float(np.sqrt(np.mean(ref * ref)))
    if rms == 0.0:
        return float(np.abs(got - ref).max())
    assert np.isfinite(got).all(), "non-finite values in the GPU result"
    return float(np.abs(got - ref).max() / rms)


def oracle_on(oracle, d, seqs=None, qk_heads=None, S0=None, n_threads=0):
    """Run the oracle on sequences ``seqs`` and query/key heads ``qk_heads`` (with their value
    heads) of the packed inputs ``d`` (as made by workloads.prefill_inputs). Returns
    {(n, h): (o [len, dv], S_T [dk, dv])} keyed by value head."""
    q, k, v = d["q"], d["k"], d["v"]
    T, h_qk, _ = q.shape
    h_v = v.shape[1]
    grp = h_v // h_qk
    lens = d["lengths"]
    starts = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    seqs = range(len(lens)) if seqs is None else seqs
    qk_heads = range(h_qk) if qk_heads is None else qk_heads
    S0 = d.get("S0") if S0 is None else S0
    out = {}
    for n in seqs:
        a, z = int(starts[n]), int(starts[n + 1])
        for g in qk_heads:
            hs = slice(g * grp, (g + 1) * grp)
            sub = lambda x, sl: x[a:z, sl].detach().cpu().contiguous()
            s0 = None if S0 is None else S0[n:n + 1, hs].detach().cpu().contiguous()
            o, st = oracle.fwd_ref(sub(q, slice(g, g + 1)), sub(k, slice(g, g + 1)), sub(v, hs),
                                   sub(d["log_alpha"], hs), sub(d["b"], hs), sub(d["w"], hs),
                                   S0=s0, n_threads=n_threads)
            for j in range(grp):
                out[(n, g * grp + j)] = (o[:, j], st[0, j])
    return out
