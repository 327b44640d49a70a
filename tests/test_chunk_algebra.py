"""The chunkwise-parallel form of the Gated DeltaNet-2 recurrence, in fp64 numpy, must
equal the sequential oracle. This checks the algebra the CUDA chunk kernel implements
before any kernel numerics enter.

Derivation (per sequence and value head, a chunk of C tokens with state S on entry).
Write e_i = b_i(.)k_i, x_i = w_i(.)v_i, G_i = sum_{m<=i} log_alpha_m (inclusive, per key
channel), and divide the state by its accumulated decay, S~_i = Diag(exp(-G_i)) S_i. Then
    S~_i = S - sum_{j<=i} (e_j(.)exp(-G_j)) r_j^T + sum_{j<=i} (k_j(.)exp(-G_j)) x_j^T,
and the key read r_i = (Diag(alpha_i) S_{i-1})^T k_i = S~_{i-1}^T (k_i(.)exp(G_i)) gives
    (I + A) R = Khat S + B X,   A_ij = sum_c k_ic e_jc exp(G_ic - G_jc)   (j < i)
                                B_ij = sum_c k_ic k_jc exp(G_ic - G_jc)   (j < i)
with Khat = K(.)exp(G). So R = T (Khat S + B X), T = (I + A)^-1 (the gated UT transform).
The query read of the updated state is
    O = Qhat S + P X - Qm R,   P_ij = sum_c q_ic k_jc exp(G_ic - G_jc)    (j <= i)
                               Qm_ij = sum_c q_ic e_jc exp(G_ic - G_jc)   (j <= i)
and the state leaving the chunk is
    S' = Diag(exp(G_C)) S + (K(.)exp(G_C - G))^T X - (E(.)exp(G_C - G))^T R.
"""
import numpy as np
import pytest

from tests.test_oracle_pins import _rand_inputs


def chunked_forward(q, k, v, la, b, w, S0, C):
    """fp64 chunked form for one (sequence, head): q,k,la,b [T,dk]; v,w [T,dv]."""
    T, dk = k.shape
    dv = v.shape[1]
    S = np.zeros((dk, dv)) if S0 is None else S0.astype(np.float64).copy()
    out = np.zeros((T, dv))
    for c0 in range(0, T, C):
        c1 = min(T, c0 + C)
        Kc, Qc, Lc = k[c0:c1], q[c0:c1], la[c0:c1]
        Ec = b[c0:c1] * Kc
        Xc = w[c0:c1] * v[c0:c1]
        G = np.cumsum(Lc, axis=0)
        n = c1 - c0
        ratio = np.exp(G[:, None, :] - G[None, :, :])          # [i, j, c] = exp(G_ic - G_jc)
        strict = np.tril(np.ones((n, n)), -1)
        incl = np.tril(np.ones((n, n)))
        # masked entries may be huge (exp of a positive sum): mask by selection
        A = np.where(strict > 0, np.einsum("ic,jc,ijc->ij", Kc, Ec, np.where(strict[..., None] > 0, ratio, 0)), 0)
        B = np.where(strict > 0, np.einsum("ic,jc,ijc->ij", Kc, Kc, np.where(strict[..., None] > 0, ratio, 0)), 0)
        P = np.where(incl > 0, np.einsum("ic,jc,ijc->ij", Qc, Kc, np.where(incl[..., None] > 0, ratio, 0)), 0)
        Qm = np.where(incl > 0, np.einsum("ic,jc,ijc->ij", Qc, Ec, np.where(incl[..., None] > 0, ratio, 0)), 0)
        Tm = np.linalg.inv(np.eye(n) + A)
        Khat, Qhat = Kc * np.exp(G), Qc * np.exp(G)
        R = Tm @ (Khat @ S + B @ Xc)
        out[c0:c1] = Qhat @ S + P @ Xc - Qm @ R
        tail = np.exp(G[-1][None, :] - G)
        S = np.exp(G[-1])[:, None] * S + (Kc * tail).T @ Xc - (Ec * tail).T @ R
    return out, S


@pytest.mark.parametrize("T", [1, 5, 63, 64, 65, 130])
@pytest.mark.parametrize("C", [4, 8, 64])
def test_chunked_equals_sequential(oracle_mod, T, C):
    rng = np.random.default_rng(100 + T * 7 + C)
    dk, dv = 8, 6
    q, k, v, la, b, w, S0 = _rand_inputs(rng, T, 1, 1, dk, dv, S0_scale=0.3)
    o, st = oracle_mod.fwd_ref(q, k, v, la, b, w, S0=S0, bf16=False)
    f = lambda x: x[:, 0].astype(np.float64)
    oc, sc = chunked_forward(f(q), f(k), f(v), f(la), f(b), f(w), S0[0, 0], C)
    scale = max(1.0, np.abs(o).max())
    assert np.abs(oc - o[:, 0]).max() <= 1e-11 * scale
    assert np.abs(sc - st[0, 0]).max() <= 1e-11 * max(1.0, np.abs(st).max())
