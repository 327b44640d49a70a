"""The per-token adjoint that the CUDA backward evaluates, stated in fp64 numpy and compared
with the oracle's reverse-mode differentiation of the recurrence (oracle.bwd_ref).

For each token, with e = b (.) k, x = w (.) v, S' = Diag(alpha) S_prev, r = S'^T k, the
update S = S' - e r^T + k x^T, o = S^T q, and dS the adjoint of S (later tokens, dS_T):
    dS += q dO^T;  dx = dS^T k;  dr = -dS^T e;  de = -dS r
    dk = dS x + Diag(alpha) S_prev dr + de (.) b;  db = de (.) k
    dS' = dS + k dr^T;  dlog_alpha = alpha (.) rowsum(dS' (.) S_prev);  dq = S dO
    dw = dx (.) v;  dv = dx (.) w;  and Diag(alpha) dS' goes to the previous token.
A query/key head's dq, dk sum over its value heads."""
import numpy as np
import pytest

import oracle
from tests.test_oracle_pins import _rand_inputs


def token_adjoint(q, k, v, la, b, w, dO, S0, dS_T, cu):
    """q, k [T, Hqk, dk]; v, w, dO [T, Hv, dv]; la, b [T, Hv, dk]; S0, dS_T [N, Hv, dk, dv]."""
    T, h_qk, dk = q.shape
    h_v, dv = v.shape[1], v.shape[2]
    grp = h_v // h_qk
    f = lambda a: np.asarray(a, dtype=np.float64)
    q, k, v, la, b, w, dO = map(f, (q, k, v, la, b, w, dO))
    gq, gk = np.zeros_like(q), np.zeros_like(k)
    gv, gw, gla, gb = np.zeros_like(v), np.zeros_like(w), np.zeros_like(la), np.zeros_like(b)
    N = len(cu) - 1
    gS0 = np.zeros((N, h_v, dk, dv))
    for n in range(N):
        t0, t1 = cu[n], cu[n + 1]
        for h in range(h_v):
            g = h // grp
            S = np.zeros((dk, dv)) if S0 is None else f(S0[n, h]).copy()
            states = [S]
            for t in range(t0, t1):  # forward, keeping every state
                al = np.exp(la[t, h])
                Sp = al[:, None] * S
                r = Sp.T @ k[t, g]
                S = Sp - np.outer(b[t, h] * k[t, g], r) + np.outer(k[t, g], w[t, h] * v[t, h])
                states.append(S)
            dS = np.zeros((dk, dv)) if dS_T is None else f(dS_T[n, h]).copy()
            for t in range(t1 - 1, t0 - 1, -1):
                Sprev, Snew = states[t - t0], states[t - t0 + 1]
                al, kt, qt, bt = np.exp(la[t, h]), k[t, g], q[t, g], b[t, h]
                e, x = bt * kt, w[t, h] * v[t, h]
                r = (al[:, None] * Sprev).T @ kt
                dS = dS + np.outer(qt, dO[t, h])
                dx, dr = dS.T @ kt, -(dS.T @ e)
                de = -(dS @ r)
                gk[t, g] += dS @ x + al * (Sprev @ dr) + de * bt
                gb[t, h] = de * kt
                dSp = dS + np.outer(kt, dr)
                gla[t, h] = al * (dSp * Sprev).sum(1)
                gq[t, g] += Snew @ dO[t, h]
                gw[t, h], gv[t, h] = dx * v[t, h], dx * w[t, h]
                dS = al[:, None] * dSp
            gS0[n, h] = dS
    return gq, gk, gv, gla, gb, gw, gS0


@pytest.mark.parametrize("lens,h_qk,h_v", [([9], 1, 1), ([5, 0, 12], 1, 2), ([1, 7], 2, 2)])
def test_token_adjoint_equals_reverse_mode(lens, h_qk, h_v):
    rng = np.random.default_rng(sum(lens) + 10 * h_v)
    T, dk, dv = sum(lens), 6, 5
    q, k, v, la, b, w, _ = _rand_inputs(rng, T, h_qk, h_v, dk, dv)
    S0 = 0.3 * rng.standard_normal((len(lens), h_v, dk, dv))
    dO = rng.standard_normal((T, h_v, dv))
    dS_T = rng.standard_normal((len(lens), h_v, dk, dv))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    ref = oracle.bwd_ref(q, k, v, la, b, w, dO, S0=S0, dS_T=dS_T, cu_seqlens=cu)
    got = token_adjoint(q, k, v, la, b, w, dO, S0, dS_T, cu)
    for name, a, r in zip(["dq", "dk", "dv", "dlog_alpha", "db", "dw", "dS0"], got, ref):
        r = np.asarray(r, dtype=np.float64)
        assert np.abs(a - r).max() <= 1e-10 * max(1.0, np.abs(r).max()), name
