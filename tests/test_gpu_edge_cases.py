"""Degenerate and extreme inputs of the recurrence, and run-to-run determinism, on the CUDA
path (through the C ABI) against the fp64 oracle.

The chunked kernel takes every decayed operand relative to the chunk's mid-point decay, so
its fp32 factors reach e^(+-(the chunk's total log-decay) / 2): the strong-decay case puts
about 145 nats of decay in each 64-token chunk (factors near e^72, inside fp32's range);
past ~166 nats the kernel recomputes that (sequence, head) token by token in fp32 and
flags the call in the device status word.
"""
import numpy as np
import pytest
import torch

from gated_delta_rule_160_b200 import workloads as W
from tests.parity import TOL, oracle_on, rel_err

pytestmark = pytest.mark.gpu

H = 2          # value (= query/key) heads
LENS = [200, 64, 131]


@pytest.fixture(scope="module")
def g():
    import gated_delta_rule_160_b200 as g
    g.load_library()
    assert torch.cuda.is_available()
    return g


def _inputs(seed=11, S0_std=0.05):
    T = sum(LENS)
    d = W.token_inputs(T, H, H, 128, 128, torch.bfloat16, "cuda", seed=seed)
    d["S0"] = W.state_input(len(LENS), H, 128, 128, S0_std, "cuda", seed=seed)
    d["cu_seqlens"] = torch.tensor(np.concatenate([[0], np.cumsum(LENS)]), dtype=torch.int32, device="cuda")
    d["n_seq"] = None
    d["lengths"] = list(LENS)
    return d


def _run(g, d):
    o, st = g.gdn2_chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], S0=d["S0"],
                             cu_seqlens=d["cu_seqlens"])
    torch.cuda.synchronize()
    return o, st


def _check(g, oracle_mod, d, label):
    o, st = _run(g, d)
    ref = oracle_on(oracle_mod, d)
    starts = np.concatenate([[0], np.cumsum(d["lengths"])])
    eo = rel_err(torch.cat([o[starts[n]:starts[n + 1], h].float() for (n, h) in ref]),
                 np.concatenate([ref[key][0] for key in ref]))
    es = rel_err(torch.stack([st[n, h] for (n, h) in ref]), np.stack([ref[key][1] for key in ref]))
    tol = TOL[torch.bfloat16]
    print(f"{label}: o err {eo:.3e}, S_T err {es:.3e} (tol {tol})")
    assert eo <= tol and es <= tol, label
    return o, st


def test_deterministic(g):
    d = _inputs()
    o1, s1 = _run(g, d)
    o2, s2 = _run(g, d)
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


def test_no_erase_no_write(g, oracle_mod):
    """b = 0 and w = 0: the state only decays, S_T[c][m] = exp(G_T[c]) S0[c][m]."""
    d = _inputs()
    d["b"] = torch.zeros_like(d["b"])
    d["w"] = torch.zeros_like(d["w"])
    _, st = _check(g, oracle_mod, d, "b = w = 0")
    starts = np.concatenate([[0], np.cumsum(LENS)])
    for n in range(len(LENS)):
        g_T = d["log_alpha"][starts[n]:starts[n + 1]].double().sum(0)        # [H, dk]
        want = torch.exp(g_T)[:, :, None] * d["S0"][n].double()
        torch.testing.assert_close(st[n].double(), want, rtol=1e-4, atol=1e-7)


def test_zero_decay(g, oracle_mod):
    """log_alpha = 0: no forgetting at all."""
    d = _inputs(seed=12)
    d["log_alpha"] = torch.zeros_like(d["log_alpha"])
    _check(g, oracle_mod, d, "zero decay")


def test_strong_decay(g, oracle_mod):
    """log_alpha = -2.3 per token: ~145 nats of decay across a chunk, inside the range of the
    chunk kernel's factors, so the device status stays clear."""
    d = _inputs(seed=13)
    d["log_alpha"] = torch.full_like(d["log_alpha"], -2.3)
    g.gdn2_device_status()
    o, st = _check(g, oracle_mod, d, "strong decay")
    assert torch.isfinite(o).all() and torch.isfinite(st).all()
    assert g.gdn2_device_status() == 0


def _check_pairs_fp32(d, o, st, ref, pairs, label):
    """The recomputed pairs run the recurrence in fp32 on the bf16 inputs: the fp32 bound."""
    starts = np.concatenate([[0], np.cumsum(d["lengths"])])
    eo = rel_err(torch.cat([o[starts[n]:starts[n + 1], h] for (n, h) in pairs]),
                 np.concatenate([ref[key][0] for key in pairs]))
    es = rel_err(torch.stack([st[n, h] for (n, h) in pairs]), np.stack([ref[key][1] for key in pairs]))
    print(f"{label}: o err {eo:.3e}, S_T err {es:.3e} (tol {TOL[torch.float32]})")
    assert eo <= TOL[torch.float32] and es <= TOL[torch.float32], (eo, es)


def test_decay_beyond_the_factor_range_is_recomputed(g, oracle_mod):
    """log_alpha = -5 per token on some channels: ~320 nats across a 64-token chunk, past
    what the chunk kernel's mid-point factors e^(+-(G - Gref)) hold in fp32. Every
    (sequence, head) is then recomputed token by token in fp32 inside the same launch: the
    bf16 call matches the oracle to the fp32 bound and reports GDN2_DEVICE_DECAY_RANGE. The
    fp32 path (fp32 inputs) takes the same decay exactly."""
    d = _inputs(seed=15)
    la = d["log_alpha"].clone()
    la[..., :8] = -5.0
    d["log_alpha"] = la
    g.gdn2_device_status()
    o, st = _run(g, d)
    assert o.dtype == torch.float32
    assert g.gdn2_device_status() & g.GDN2_DEVICE_DECAY_RANGE
    ref = oracle_on(oracle_mod, d)
    _check_pairs_fp32(d, o, st, ref, list(ref), "decay past the range, bf16 call")
    d32 = dict(d)
    for k_ in ("q", "k", "v", "b", "w"):
        d32[k_] = d[k_].float()
    o, st = g.gdn2_chunk_fwd(d32["q"], d32["k"], d32["v"], d32["log_alpha"], d32["b"], d32["w"], S0=d32["S0"],
                             cu_seqlens=d32["cu_seqlens"])
    torch.cuda.synchronize()
    assert g.gdn2_device_status() == 0
    _check_pairs_fp32(d32, o, st, oracle_on(oracle_mod, d32), list(ref), "decay past the range, fp32 path")


def test_only_the_out_of_range_pair_is_recomputed(g, oracle_mod):
    """The decay leaves the range in one chunk of one (sequence, head) only (sequence 0,
    tokens 128..191, value head 1, eight channels), so the kernel meets it in the middle of
    that pair's walk. That pair matches the oracle to the fp32 bound; every other pair is
    bit for bit what the same launch gives without the strong decay; bf16 outputs too."""
    d = _inputs(seed=16)
    base_o, base_st = _run(g, d)
    base_o16, _ = g.gdn2_chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], S0=d["S0"],
                                   cu_seqlens=d["cu_seqlens"], out_dtype=torch.bfloat16)
    la = d["log_alpha"].clone()
    la[128:192, 1, :8] = -5.0
    d["log_alpha"] = la
    g.gdn2_device_status()
    o, st = _run(g, d)
    assert g.gdn2_device_status() & g.GDN2_DEVICE_DECAY_RANGE
    ref = oracle_on(oracle_mod, d, seqs=[0])
    _check_pairs_fp32(d, o, st, ref, [(0, 1)], "one pair past the range")
    starts = np.concatenate([[0], np.cumsum(d["lengths"])])
    for n in range(len(LENS)):
        for h in range(H):
            if (n, h) == (0, 1):
                continue
            assert torch.equal(o[starts[n]:starts[n + 1], h], base_o[starts[n]:starts[n + 1], h]), (n, h)
            assert torch.equal(st[n, h], base_st[n, h]), (n, h)
    o16, st16 = g.gdn2_chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], S0=d["S0"],
                                 cu_seqlens=d["cu_seqlens"], out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert g.gdn2_device_status() & g.GDN2_DEVICE_DECAY_RANGE
    assert torch.equal(st16, st)
    # the recomputation's fp32 outputs, rounded to bf16 once
    assert torch.equal(o16[starts[0]:starts[1], 1], o[starts[0]:starts[1], 1].to(torch.bfloat16))
    keep = torch.ones(o16.shape[:2], dtype=torch.bool, device=o16.device)
    keep[starts[0]:starts[1], 1] = False
    assert torch.equal(o16[keep], base_o16[keep])


def test_recomputed_pair_without_final_state(g, oracle_mod):
    """The recomputation with no S_T buffer (only o asked for): o still matches the oracle to
    the fp32 bound for the pair past the range and the bf16 bound elsewhere."""
    d = _inputs(seed=18)
    la = d["log_alpha"].clone()
    la[200:264, 0, 16:24] = -6.0  # sequence 1 (tokens 200..263), value head 0
    d["log_alpha"] = la
    g.gdn2_device_status()
    o, none = g.gdn2_chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], S0=d["S0"],
                               cu_seqlens=d["cu_seqlens"], want_state=False)
    torch.cuda.synchronize()
    assert none is None and g.gdn2_device_status() & g.GDN2_DEVICE_DECAY_RANGE
    ref = oracle_on(oracle_mod, d)
    starts = np.concatenate([[0], np.cumsum(d["lengths"])])
    e1 = rel_err(o[starts[1]:starts[2], 0], ref[(1, 0)][0])
    rest = [key for key in ref if key != (1, 0)]
    e2 = rel_err(torch.cat([o[starts[n]:starts[n + 1], h] for (n, h) in rest]),
                 np.concatenate([ref[key][0] for key in rest]))
    print(f"no S_T: recomputed pair o err {e1:.3e}, other pairs {e2:.3e}")
    assert e1 <= TOL[torch.float32] and e2 <= TOL[torch.bfloat16]


def test_state_updated_in_place(g):
    """S_T may be S0: each (sequence, head) reads its initial state before it writes the final
    one, on the tensor-core path, on its token-by-token recomputation (strong decay in one
    pair) and on the fp32 path; the results are bit for bit those of separate buffers."""
    d = _inputs(seed=17)
    la = d["log_alpha"].clone()
    la[64:128, 0, :8] = -5.0  # sequence 0, value head 0: recomputed
    d["log_alpha"] = la
    cases = [d, dict(d, **{k_: d[k_].float() for k_ in ("q", "k", "v", "b", "w")})]
    for c in cases:
        names = ("q", "k", "v", "log_alpha", "b", "w")
        o, st = g.gdn2_chunk_fwd(*(c[k_] for k_ in names), S0=c["S0"], cu_seqlens=c["cu_seqlens"])
        S = c["S0"].clone()
        o2, st2 = g.gdn2_chunk_fwd(*(c[k_] for k_ in names), S0=S, S_T=S, cu_seqlens=c["cu_seqlens"])
        torch.cuda.synchronize()
        assert st2.data_ptr() == S.data_ptr()
        assert torch.equal(o2, o) and torch.equal(S, st)
    g.gdn2_device_status()


def test_decay_mixed_per_channel(g, oracle_mod):
    """Half the key channels barely decay, half decay hard: the per-channel reference frame."""
    d = _inputs(seed=14)
    la = d["log_alpha"].clone()
    la[..., :64] = -1e-3
    la[..., 64:] = -2.0
    d["log_alpha"] = la
    _check(g, oracle_mod, d, "mixed decay")
