"""Gradients of the recurrence on the GPU (gdn2_chunk_bwd, through the C ABI) against the
oracle's reverse-mode differentiation of its plain fp64 statement."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_160_b200 import workloads as W
from tests.parity import rel_err

pytestmark = pytest.mark.gpu

TOL = 1e-4  # the backward kernel's arithmetic is fp32 for every input dtype


@pytest.fixture(scope="module")
def g():
    import gated_delta_rule_160_b200 as g
    g.load_library()
    assert torch.cuda.is_available()
    return g


@pytest.mark.parametrize("dtype,d,h_qk,h_v,lens", [
    (torch.float32, 64, 1, 2, [37, 64, 1, 0, 90]),
    (torch.bfloat16, 128, 2, 2, [70, 129]),
])
def test_backward_matches_oracle(g, dtype, d, h_qk, h_v, lens):
    T = sum(lens)
    inp = W.token_inputs(T, h_qk, h_v, d, d, dtype, "cuda", seed=51)
    S0 = W.state_input(len(lens), h_v, d, d, 0.05, "cuda", seed=51)
    gen = torch.Generator(device="cuda").manual_seed(52)
    dO = torch.randn(T, h_v, d, generator=gen, device="cuda")
    dS = torch.randn(len(lens), h_v, d, d, generator=gen, device="cuda")
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device="cuda")
    got = g.gdn2_chunk_bwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["b"], inp["w"], dO, S0=S0,
                           dS_T=dS, cu_seqlens=cu)
    torch.cuda.synchronize()
    ref = oracle.bwd_ref(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["b"], inp["w"], dO, S0=S0,
                         dS_T=dS, cu_seqlens=cu.cpu())
    for name, a, r in zip(["dq", "dk", "dv", "dlog_alpha", "db", "dw", "dS0"], got, ref):
        err = rel_err(a, r)
        print(f"backward {dtype} d={d}: {name} err {err:.3e}")
        assert err <= TOL, name


def test_backward_without_final_state_gradient(g):
    """dS_T omitted = zero; dS0 not requested."""
    T, H, d = 100, 2, 64
    inp = W.token_inputs(T, H, H, d, d, torch.float32, "cuda", seed=53)
    dO = torch.randn(T, H, d, generator=torch.Generator(device="cuda").manual_seed(54), device="cuda")
    got = g.gdn2_chunk_bwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["b"], inp["w"], dO, n_seq=1,
                           want_dS0=False)
    torch.cuda.synchronize()
    ref = oracle.bwd_ref(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["b"], inp["w"], dO, n_seq=1)
    assert got[6] is None
    for a, r in zip(got[:6], ref[:6]):
        assert rel_err(a, r) <= TOL
