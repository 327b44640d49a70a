"""The seeded input generators (gated_delta_rule_160_b200/workloads.py) follow the stated
recipe and are deterministic: q, k unit-length per token and head; v ~ N(0, 1);
log_alpha = -softplus(N(0, 1)) < 0 in fp32; b, w = sigmoid(N(0, 1)) in (0, 1); packed
lengths in [128, 8192]; the same seed gives the same tensors."""
import numpy as np
import torch

from gated_delta_rule_160_b200 import workloads as W


def test_token_recipe_and_determinism():
    a = W.token_inputs(300, 2, 4, 64, 32, torch.float32, "cpu", seed=7)
    b = W.token_inputs(300, 2, 4, 64, 32, torch.float32, "cpu", seed=7)
    c = W.token_inputs(300, 2, 4, 64, 32, torch.float32, "cpu", seed=8)
    for key in a:
        assert torch.equal(a[key], b[key]), key
        assert not torch.equal(a[key], c[key]), key
    assert a["q"].shape == (300, 2, 64) and a["v"].shape == (300, 4, 32)
    assert a["log_alpha"].shape == (300, 4, 64) and a["log_alpha"].dtype == torch.float32
    assert a["b"].shape == (300, 4, 64) and a["w"].shape == (300, 4, 32)
    for key in ("q", "k"):
        assert torch.allclose(a[key].norm(dim=-1), torch.ones(300, 2), atol=1e-5), key
    assert (a["log_alpha"] < 0).all()
    for key in ("b", "w"):
        assert ((a[key] > 0) & (a[key] < 1)).all(), key
    v = a["v"].double()
    assert abs(v.mean().item()) < 0.05 and abs(v.std().item() - 1.0) < 0.05


def test_bf16_inputs_are_the_rounded_recipe():
    f = W.token_inputs(64, 1, 1, 128, 128, torch.float32, "cpu", seed=3)
    h = W.token_inputs(64, 1, 1, 128, 128, torch.bfloat16, "cpu", seed=3)
    for key in ("q", "k", "v", "b", "w"):
        assert h[key].dtype == torch.bfloat16
        assert torch.equal(h[key], f[key].to(torch.bfloat16)), key
    assert h["log_alpha"].dtype == torch.float32  # the decay stays fp32


def test_workload_shapes_and_lengths():
    wl = W.WORKLOADS["varlen_64seq_h16"]
    lens = W.seq_lengths(wl)
    assert len(lens) == 64 and min(lens) >= 128 and max(lens) <= 8192
    assert lens == W.seq_lengths(wl)  # seeded
    assert 200_000 < sum(lens) < 330_000
    pre = W.WORKLOADS["prefill_b8_h16_t4096"]
    assert (pre.n_seq, pre.h_qk, pre.h_v, pre.dk, pre.dv, pre.T) == (8, 16, 16, 128, 128, 4096)
    grp = W.WORKLOADS["grouped_b2_qk16_v32_t32768"]
    assert (grp.n_seq, grp.h_qk, grp.h_v, grp.T) == (2, 16, 32, 32768) and grp.S0_std == 0.02
    dec = W.WORKLOADS["decode_256seq_h32"]
    assert (dec.n_seq, dec.h_v, dec.decode_steps, dec.S0_std) == (256, 32, 512, 0.05)


def test_states():
    assert W.state_input(2, 3, 8, 8, 0.0, "cpu", seed=1) is None
    s = W.state_input(64, 4, 32, 32, 0.05, "cpu", seed=1)
    assert s.shape == (64, 4, 32, 32) and s.dtype == torch.float32
    assert abs(s.double().std().item() - 0.05) < 0.005
    assert torch.equal(s, W.state_input(64, 4, 32, 32, 0.05, "cpu", seed=1))
    np.testing.assert_array_equal(W.prefill_inputs(W.WORKLOADS["tiny_fp32"], "cpu")["lengths"], [256])
