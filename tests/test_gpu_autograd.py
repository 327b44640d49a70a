"""gdn2_chunk, the differentiable pairing of gdn2_chunk_fwd and gdn2_chunk_bwd: its outputs
are gdn2_chunk_fwd's bit for bit, and torch's backward through it gives gdn2_chunk_bwd's
gradients (checked against the oracle in test_gpu_backward.py) cast to each input's dtype,
for a loss on o and S_T, on packed sequences with grouped heads and an initial state."""
import numpy as np
import pytest
import torch

from gated_delta_rule_160_b200 import workloads as W

pytestmark = pytest.mark.gpu

NAMES = ("q", "k", "v", "log_alpha", "b", "w")


@pytest.fixture(scope="module")
def g():
    import gated_delta_rule_160_b200 as g
    g.load_library()
    assert torch.cuda.is_available()
    return g


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_autograd_matches_the_direct_calls(g, dtype):
    lens = [150, 64, 1, 97]
    d = W.token_inputs(sum(lens), 2, 4, 128, 128, dtype, "cuda", seed=91)
    S0 = W.state_input(len(lens), 4, 128, 128, 0.05, "cuda", seed=91)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device="cuda")
    gen = torch.Generator(device="cuda").manual_seed(92)
    dO = torch.randn(d["v"].shape, generator=gen, device="cuda")
    dS_T = torch.randn(S0.shape, generator=gen, device="cuda")

    leaves = {k_: d[k_].clone().requires_grad_(True) for k_ in NAMES}
    S0_leaf = S0.clone().requires_grad_(True)
    o, S_T = g.gdn2_chunk(*(leaves[k_] for k_ in NAMES), S0=S0_leaf, cu_seqlens=cu)
    ((o * dO).sum() + (S_T * dS_T).sum()).backward()
    torch.cuda.synchronize()

    o_ref, S_T_ref = g.gdn2_chunk_fwd(*(d[k_] for k_ in NAMES), S0=S0, cu_seqlens=cu)
    grads = g.gdn2_chunk_bwd(*(d[k_] for k_ in NAMES), dO, S0=S0, dS_T=dS_T, cu_seqlens=cu)
    torch.cuda.synchronize()
    assert torch.equal(o.detach(), o_ref) and torch.equal(S_T.detach(), S_T_ref)
    for k_, gr in zip(NAMES, grads[:6]):
        assert leaves[k_].grad.dtype == d[k_].dtype
        assert torch.equal(leaves[k_].grad, gr.to(d[k_].dtype)), k_
    assert torch.equal(S0_leaf.grad, grads[6])


def test_autograd_loss_on_o_only(g):
    """A loss on o alone (S_T's gradient is None in the backward); no initial state."""
    d = W.token_inputs(130, 1, 1, 128, 128, torch.bfloat16, "cuda", seed=93)
    leaves = {k_: d[k_].clone().requires_grad_(True) for k_ in NAMES}
    o, _ = g.gdn2_chunk(*(leaves[k_] for k_ in NAMES), n_seq=1)
    o.square().sum().backward()
    grads = g.gdn2_chunk_bwd(*(d[k_] for k_ in NAMES), 2.0 * o.detach(), n_seq=1, want_dS0=False)
    torch.cuda.synchronize()
    for k_, gr in zip(NAMES, grads[:6]):
        assert torch.equal(leaves[k_].grad, gr.to(d[k_].dtype)), k_
