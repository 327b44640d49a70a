"""Pins of the oracle's fused pre-processing (oracle.prologue_ref) against closed forms,
identities and an independent implementation (torch, fp64)."""
import math

import numpy as np
import torch

import oracle


def _run(q=None, k=None, a=None, b=None, w=None, shape=(3, 2, 8)):
    z = np.zeros(shape)
    return oracle.prologue_ref(*(z if x is None else x for x in (q, k, a, b, w)))


def test_gates_at_zero():
    _, _, la, b, w = _run()
    assert np.allclose(la, -math.log(2.0), rtol=0, atol=1e-15)
    assert np.allclose(b, 0.5, rtol=0, atol=0) and np.allclose(w, 0.5, rtol=0, atol=0)


def test_decay_is_the_complementary_sigmoid():
    """exp(-softplus(a)) = 1 / (1 + e^a) = sigmoid(-a), and large |a| follows the asymptotes."""
    a = np.linspace(-30.0, 30.0, 121).reshape(11, 1, 11)
    _, _, la, _, _ = _run(a=a, shape=a.shape)
    assert np.allclose(np.exp(la), 1.0 / (1.0 + np.exp(a)), rtol=1e-13, atol=0)
    big = np.array([40.0, -40.0, 700.0, -700.0]).reshape(1, 1, 4)
    _, _, la, _, _ = _run(a=big, shape=big.shape)
    assert np.allclose(la[0, 0, :3:2], -big[0, 0, :3:2], rtol=1e-15)       # -softplus(a) -> -a
    assert np.allclose(la[0, 0, 1], -math.exp(-40.0), rtol=1e-12)           # -softplus(a) -> -e^a
    assert la[0, 0, 3] <= 0.0 and la[0, 0, 3] > -1e-300


def test_sigmoid_symmetry_and_range():
    x = np.linspace(-50.0, 50.0, 101).reshape(101, 1, 1)
    _, _, _, b, w = _run(b=x, w=x, shape=x.shape)
    assert np.all((b >= 0.0) & (b <= 1.0))
    assert np.allclose(b + b[::-1], 1.0, rtol=0, atol=1e-15)  # sigmoid(x) + sigmoid(-x) = 1
    assert np.array_equal(b, w)


def test_normalisation():
    g = np.random.default_rng(0)
    q = g.standard_normal((5, 3, 128)) * 7.0
    qn, kn, *_ = _run(q=q, k=-2.0 * q, shape=q.shape)
    assert np.allclose(np.linalg.norm(qn, axis=-1), 1.0, rtol=1e-14)
    assert np.allclose(qn, -kn, rtol=1e-14)                     # direction kept, scale removed
    assert np.allclose(qn * np.linalg.norm(q, axis=-1, keepdims=True), q, rtol=1e-13)
    zero = np.zeros((1, 1, 16))
    qz, *_ = _run(q=zero, shape=zero.shape)
    assert np.array_equal(qz, zero)                             # the zero vector stays zero


def test_against_torch_fp64():
    g = torch.Generator().manual_seed(5)
    t = {n: torch.randn((7, 2, 64), generator=g, dtype=torch.float64) * 3 for n in "qkabw"}
    q, k, la, b, w = oracle.prologue_ref(t["q"], t["k"], t["a"], t["b"], t["w"])
    F = torch.nn.functional
    assert np.allclose(q, F.normalize(t["q"], dim=-1).numpy(), rtol=1e-13)
    assert np.allclose(k, F.normalize(t["k"], dim=-1).numpy(), rtol=1e-13)
    assert np.allclose(la, -F.softplus(t["a"]).numpy(), rtol=1e-13)
    assert np.allclose(b, torch.sigmoid(t["b"]).numpy(), rtol=1e-13)
    assert np.allclose(w, torch.sigmoid(t["w"]).numpy(), rtol=1e-13)
