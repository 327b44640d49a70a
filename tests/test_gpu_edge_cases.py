"""Degenerate and extreme inputs of the recurrence, and run-to-run determinism, on the CUDA
path (through the C ABI) against the fp64 oracle.

The chunked kernel takes every decayed operand relative to the chunk's mid-point decay, so
its fp32 factors reach e^(+-(the chunk's total log-decay) / 2): the strong-decay case puts
about 145 nats of decay in each 64-token chunk (factors near e^72, inside fp32's range).
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
    """log_alpha = -2.3 per token: ~145 nats of decay across a chunk."""
    d = _inputs(seed=13)
    d["log_alpha"] = torch.full_like(d["log_alpha"], -2.3)
    o, st = _check(g, oracle_mod, d, "strong decay")
    assert torch.isfinite(o).all() and torch.isfinite(st).all()


def test_decay_mixed_per_channel(g, oracle_mod):
    """Half the key channels barely decay, half decay hard: the per-channel reference frame."""
    d = _inputs(seed=14)
    la = d["log_alpha"].clone()
    la[..., :64] = -1e-3
    la[..., 64:] = -2.0
    d["log_alpha"] = la
    _check(g, oracle_mod, d, "mixed decay")
