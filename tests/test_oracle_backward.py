"""Pins of the oracle's backward (oracle.bwd_ref): its plain torch statement of the forward
agrees with the C oracle, and its gradients agree with central finite differences of the C
oracle's forward."""
import numpy as np
import torch

import oracle


def _inputs(T, h_qk, h_v, d, seed):
    g = torch.Generator().manual_seed(seed)
    n = lambda *s: torch.randn(*s, generator=g, dtype=torch.float64)
    q = torch.nn.functional.normalize(n(T, h_qk, d), dim=-1)
    k = torch.nn.functional.normalize(n(T, h_qk, d), dim=-1)
    return dict(q=q, k=k, v=n(T, h_v, d), log_alpha=-torch.nn.functional.softplus(n(T, h_v, d)),
                b=torch.sigmoid(n(T, h_v, d)), w=torch.sigmoid(n(T, h_v, d)))


def test_torch_statement_matches_c_oracle():
    d = _inputs(23, 1, 2, 8, seed=1)
    S0 = 0.3 * torch.randn(2, 2, 8, 8, dtype=torch.float64, generator=torch.Generator().manual_seed(2))
    cu = np.array([0, 9, 23], dtype=np.int32)
    o_c, s_c = oracle.fwd_ref(*(d[x].float() for x in ("q", "k", "v", "log_alpha", "b", "w")),
                              S0=S0.float(), cu_seqlens=cu)
    f32 = {x: d[x].float().double() for x in d}  # the C oracle reads fp32 inputs
    for n, (s, e) in enumerate([(0, 9), (9, 23)]):
        qe, ke = (f32[x][s:e].repeat_interleave(2, dim=1) for x in ("q", "k"))
        o, S = oracle._recurrence_torch(qe, ke, f32["v"][s:e], f32["log_alpha"][s:e], f32["b"][s:e],
                                        f32["w"][s:e], S0[n].float().double())
        assert np.allclose(o.numpy(), o_c[s:e], rtol=1e-12, atol=1e-12)
        assert np.allclose(S.numpy(), s_c[n], rtol=1e-12, atol=1e-12)


def test_gradients_match_finite_differences():
    T, h_qk, h_v, d = 7, 1, 2, 4
    inp = _inputs(T, h_qk, h_v, d, seed=3)
    g = torch.Generator().manual_seed(4)
    S0 = 0.5 * torch.randn(1, h_v, d, d, dtype=torch.float64, generator=g)
    dO = torch.randn(T, h_v, d, dtype=torch.float64, generator=g)
    dS = torch.randn(1, h_v, d, d, dtype=torch.float64, generator=g)
    grads = oracle.bwd_ref(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["b"], inp["w"], dO,
                           S0=S0, dS_T=dS)

    def loss(vals):
        # the C oracle's forward in float64 arithmetic from float32 inputs: perturbations must
        # survive the float32 widening, so the step is large and the check relative
        o, s = oracle.fwd_ref(*(vals[x].float() for x in ("q", "k", "v", "log_alpha", "b", "w")),
                              S0=vals["S0"].float())
        return float((torch.as_tensor(o) * dO).sum() + (torch.as_tensor(s) * dS).sum())

    names = ["q", "k", "v", "log_alpha", "b", "w", "S0"]
    base = dict(inp, S0=S0)
    rng = np.random.default_rng(5)
    h = 1e-3
    for name, gr in zip(names, grads):
        x = base[name]
        for _ in range(4):  # a few random coordinates of each input
            idx = tuple(int(rng.integers(0, s)) for s in x.shape)
            plus, minus = dict(base), dict(base)
            plus[name] = x.clone(); plus[name][idx] += h
            minus[name] = x.clone(); minus[name][idx] -= h
            fd = (loss(plus) - loss(minus)) / (2 * h)
            assert abs(fd - gr[idx]) <= 2e-3 * max(1.0, abs(fd)), (name, idx, fd, gr[idx])
