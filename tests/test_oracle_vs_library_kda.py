"""The oracle pinned to a third-party implementation on the special case where the recurrence
reduces to Kimi Delta Attention (KDA): with uniform gates b = w = beta (a scalar per token
and head) and alpha = exp(g),

    S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,   o_t = S_t^T q_t,

which is the recurrence flash-linear-attention's plain torch reference
(fla.ops.kda.naive.naive_recurrent_kda) evaluates, here with query scale 1. That library is
run, not copied; it computes in fp32 internally, hence the 1e-5 tolerance, far below what any
dropped term, wrong sign or transposed operand in the oracle would produce. Skipped where the
library is not installed."""
import numpy as np
import pytest

naive = pytest.importorskip("fla.ops.kda.naive")
torch = pytest.importorskip("torch")


@pytest.mark.parametrize("T,H,HV,K,V,with_S0", [(37, 2, 2, 8, 6, True), (64, 1, 1, 16, 16, False),
                                                 (5, 3, 3, 4, 10, True), (16, 2, 4, 8, 6, True)])
def test_oracle_equals_library_kda_reference(oracle_mod, T, H, HV, K, V, with_S0):
    """The last case has two value heads per query/key head: the library groups them the
    way the oracle does (value head h reads query/key head h // (HV / H))."""
    rng = np.random.default_rng(T * 31 + H + HV)
    f32 = lambda x: np.asarray(x, np.float32)
    q = rng.standard_normal((T, H, K))
    k = rng.standard_normal((T, H, K))
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((T, HV, V))
    la = -np.log1p(np.exp(rng.standard_normal((T, HV, K))))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((T, HV))))
    S0 = 0.3 * rng.standard_normal((1, HV, K, V)) if with_S0 else None
    q, k, v, la, beta = map(f32, (q, k, v, la, beta))
    S0 = None if S0 is None else f32(S0)
    b = np.repeat(beta[:, :, None], K, axis=2)
    w = np.repeat(beta[:, :, None], V, axis=2)
    o_ref, s_ref = oracle_mod.fwd_ref(q, k, v, la, b, w, S0=S0, bf16=False)
    t = lambda x: torch.from_numpy(np.asarray(x, np.float64))[None]
    o, s = naive.naive_recurrent_kda(t(q), t(k), t(v), t(la), t(beta), scale=1.0,
                                     initial_state=None if S0 is None else torch.from_numpy(S0.astype(np.float64)),
                                     output_final_state=True)
    assert np.abs(o[0].numpy() - o_ref).max() <= 1e-5 * max(1.0, np.abs(o_ref).max())
    assert np.abs(s.numpy() - s_ref).max() <= 1e-5 * max(1.0, np.abs(s_ref).max())


def test_backward_oracle_equals_library_kda_autograd(oracle_mod):
    """The oracle's gradients (oracle.bwd_ref) at uniform gates against torch's reverse mode
    through the library's KDA reference: dq, dk, dv, dlog_alpha, dS0 directly, and the
    scalar gate's gradient as the sum of the erase and write gates' (beta feeds both)."""
    rng = np.random.default_rng(5)
    T, H, K, V = 20, 2, 8, 6
    f32 = lambda x: np.asarray(x, np.float32)
    q = rng.standard_normal((T, H, K))
    k = rng.standard_normal((T, H, K))
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((T, H, V))
    la = -np.log1p(np.exp(rng.standard_normal((T, H, K))))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((T, H))))
    S0 = 0.3 * rng.standard_normal((1, H, K, V))
    dO, dS_T = rng.standard_normal((T, H, V)), rng.standard_normal((1, H, K, V))
    q, k, v, la, beta, S0 = map(f32, (q, k, v, la, beta, S0))
    b = np.repeat(beta[:, :, None], K, axis=2)
    w = np.repeat(beta[:, :, None], V, axis=2)
    ref = oracle_mod.bwd_ref(q, k, v, la, b, w, dO, S0=S0, dS_T=dS_T, n_seq=1)
    t = lambda x: torch.from_numpy(np.asarray(x, np.float64))[None].requires_grad_(True)
    tq, tk, tv, tg, tb = t(q), t(k), t(v), t(la), t(beta)
    ts0 = torch.from_numpy(S0.astype(np.float64)).requires_grad_(True)
    o, s = naive.naive_recurrent_kda(tq, tk, tv, tg, tb, scale=1.0, initial_state=ts0, output_final_state=True)
    loss = (o * torch.from_numpy(dO)[None]).sum() + (s * torch.from_numpy(dS_T)).sum()
    gq, gk, gv, gg, gbeta, gs0 = torch.autograd.grad(loss, (tq, tk, tv, tg, tb, ts0))
    pairs = [(gq[0], ref[0]), (gk[0], ref[1]), (gv[0], ref[2]), (gg[0], ref[3]),
             (gbeta[0], np.asarray(ref[4]).sum(-1) + np.asarray(ref[5]).sum(-1)), (gs0, ref[6])]
    for a, r in pairs:
        a, r = a.detach().numpy(), np.asarray(r, dtype=np.float64)
        assert np.abs(a - r).max() <= 1e-5 * max(1.0, np.abs(r).max())
