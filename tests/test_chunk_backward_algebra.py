"""The chunkwise form of the recurrence's gradients, in fp64 numpy, must equal the oracle's
reverse-mode differentiation of the sequential recurrence (oracle.bwd_ref). This is the
algebra a chunked (tensor-core) backward would implement, checked before any kernel
numerics enter; the per-token adjoint the CUDA backward runs today is checked against the
same oracle in the GPU tests.

Derivation, per sequence and value head, for one chunk of C tokens with entry state S and
the forward's chunk quantities (test_chunk_algebra.py): E = b (.) K, X = w (.) v, G the
inclusive cumulative log-decay, ratio_ijc = exp(G_ic - G_jc), the masked Gram blocks
A, B (j < i) and P, Qm (j <= i), T = (I + A)^-1, Khat = K (.) exp(G), Qhat = Q (.) exp(G),
Y = Khat S + B X, R = T Y, O = Qhat S + P X - Qm R, g = exp(G_last), tails
Kt = K (.) exp(G_last - G), Et = E (.) exp(G_last - G), and S_next = Diag(g) S + Kt^T X - Et^T R.
Given dO and the adjoint dS_next of the state leaving the chunk, reverse mode gives, in order:
    dS = Diag(g) dS_next,  dg = rowsum(dS_next (.) S),  dKt = X dS_next^T,  dEt = -R dS_next^T,
    dX = Kt dS_next,  dR = -Et dS_next                                      (state pass)
    dQhat = dO S^T,  dS += Qhat^T dO,  dP = mask(dO X^T),  dX += P^T dO,
    dQm = -mask(dO R^T),  dR -= Qm^T dO                                      (output)
    dT = dR Y^T,  dY = T^T dR,  dA = -mask(T^T dT T^T)                       (UT transform)
    dKhat = dY S^T,  dS += Khat^T dY,  dB = mask(dY X^T),  dX += B^T dY     (key reads)
and for each masked Gram block M_ij = sum_c U_ic V_jc ratio_ijc with its adjoint dM:
    dU_ic += sum_j dM_ij V_jc ratio_ijc,  dV_jc += sum_i dM_ij U_ic ratio_ijc,
    dG_ic += sum_j dM_ij U_ic V_jc ratio_ijc,  dG_jc -= sum_i dM_ij U_ic V_jc ratio_ijc
((U, V) = (K, E) for A, (K, K) for B, (Q, K) for P, (Q, E) for Qm); then
    dK += dKhat (.) exp(G) + dKt (.) exp(G_last - G) + dE (.) b,   db = dE (.) K,
    dQ += dQhat (.) exp(G),   dE += dEt (.) exp(G_last - G),
    dG += dKhat (.) Khat + dQhat (.) Qhat - (dKt (.) Kt + dEt (.) Et),
    dG_last += colsum(dKt (.) Kt + dEt (.) Et) + dg (.) g,
    dlog_alpha = reverse cumulative sum of dG over the chunk's tokens,
    dv = dX (.) w,  dw = dX (.) v,
and dS is the adjoint passed to the previous chunk (dS0 after the first). Every exponent in
the ratio form is <= 0 inside the masks, so no intermediate overflows; a kernel would
factor the ratios through a per-chunk reference frame as the forward does.
"""
import numpy as np
import pytest

import oracle
from tests.test_oracle_pins import _rand_inputs


def _chunk(Kc, Qc, Lc, Bc, Xc, S):
    n = Kc.shape[0]
    G = np.cumsum(Lc, axis=0)
    Ec = Bc * Kc
    strict = np.tril(np.ones((n, n)), -1)
    incl = np.tril(np.ones((n, n)))
    diff = G[:, None, :] - G[None, :, :]
    rs = np.where(strict[..., None] > 0, np.exp(np.where(strict[..., None] > 0, diff, 0.0)), 0.0)
    ri = np.where(incl[..., None] > 0, np.exp(np.where(incl[..., None] > 0, diff, 0.0)), 0.0)
    gram = lambda U, V, r: np.einsum("ic,jc,ijc->ij", U, V, r)
    A, B = gram(Kc, Ec, rs), gram(Kc, Kc, rs)
    P, Qm = gram(Qc, Kc, ri), gram(Qc, Ec, ri)
    Tm = np.linalg.inv(np.eye(n) + A)
    eG = np.exp(G)
    Khat, Qhat = Kc * eG, Qc * eG
    Y = Khat @ S + B @ Xc
    R = Tm @ Y
    O = Qhat @ S + P @ Xc - Qm @ R
    g = np.exp(G[-1])
    tail = np.exp(G[-1][None, :] - G)
    Kt, Et = Kc * tail, Ec * tail
    S_next = g[:, None] * S + Kt.T @ Xc - Et.T @ R
    return dict(G=G, E=Ec, strict=strict, incl=incl, rs=rs, ri=ri, A=A, B=B, P=P, Qm=Qm, T=Tm, eG=eG,
                Khat=Khat, Qhat=Qhat, Y=Y, R=R, O=O, g=g, tail=tail, Kt=Kt, Et=Et, S_next=S_next)


def _gram_bwd(dM, U, V, r):
    W = dM[:, :, None] * r
    t = W * U[:, None, :] * V[None, :, :]
    return np.einsum("ijc,jc->ic", W, V), np.einsum("ijc,ic->jc", W, U), t.sum(1) - t.sum(0)


def chunked_backward(q, k, v, la, b, w, S0, dO, dS_T, C):
    """fp64 chunked gradients for one (sequence, head): q,k,la,b [T,dk]; v,w,dO [T,dv];
    S0, dS_T [dk,dv] or None. Returns dq, dk, dv, dla, db, dw, dS0."""
    T, dk = k.shape
    dv = v.shape[1]
    X = w * v
    S = np.zeros((dk, dv)) if S0 is None else S0.copy()
    starts = list(range(0, T, C))
    entry = []
    for c0 in starts:  # forward: the state entering every chunk
        c1 = min(T, c0 + C)
        entry.append(S)
        S = _chunk(k[c0:c1], q[c0:c1], la[c0:c1], b[c0:c1], X[c0:c1], S)["S_next"]
    gq, gk, gla, gb, gX = (np.zeros_like(a) for a in (q, k, la, b, X))
    dS = np.zeros((dk, dv)) if dS_T is None else dS_T.copy()
    for ci in reversed(range(len(starts))):
        c0 = starts[ci]
        c1 = min(T, c0 + C)
        Kc, Qc, Bc, Xc, S = k[c0:c1], q[c0:c1], b[c0:c1], X[c0:c1], entry[ci]
        f = _chunk(Kc, Qc, la[c0:c1], Bc, Xc, S)
        dOc = dO[c0:c1]
        # state pass
        dSp = f["g"][:, None] * dS
        dg = (dS * S).sum(1)
        dKt, dEt = Xc @ dS.T, -(f["R"] @ dS.T)
        dXc = f["Kt"] @ dS
        dR = -(f["Et"] @ dS)
        # output
        dQhat = dOc @ S.T
        dSp += f["Qhat"].T @ dOc
        dP = f["incl"] * (dOc @ Xc.T)
        dXc += f["P"].T @ dOc
        dQm = -f["incl"] * (dOc @ f["R"].T)
        dR -= f["Qm"].T @ dOc
        # UT transform and key reads
        dTm = dR @ f["Y"].T
        dY = f["T"].T @ dR
        dA = -f["strict"] * (f["T"].T @ dTm @ f["T"].T)
        dKhat = dY @ S.T
        dSp += f["Khat"].T @ dY
        dB = f["strict"] * (dY @ Xc.T)
        dXc += f["B"].T @ dY
        # masked Gram blocks
        dKc, dQc, dEc, dG = (np.zeros_like(Kc) for _ in range(4))
        for dM, (U, V, r, tu, tv) in ((dA, (Kc, f["E"], f["rs"], "k", "e")), (dB, (Kc, Kc, f["rs"], "k", "k")),
                                       (dP, (Qc, Kc, f["ri"], "q", "k")), (dQm, (Qc, f["E"], f["ri"], "q", "e"))):
            dU, dV, dGc = _gram_bwd(dM, U, V, r)
            dG += dGc
            for name, dval in ((tu, dU), (tv, dV)):
                if name == "k":
                    dKc += dval
                elif name == "q":
                    dQc += dval
                else:
                    dEc += dval
        # scaled operands, tails, the chunk's total decay
        dKc += dKhat * f["eG"] + dKt * f["tail"]
        dQc += dQhat * f["eG"]
        dEc += dEt * f["tail"]
        tt = dKt * f["Kt"] + dEt * f["Et"]
        dG += dKhat * f["Khat"] + dQhat * f["Qhat"] - tt
        dG[-1] += tt.sum(0) + dg * f["g"]
        # E = b (.) K; G = cumsum(log_alpha)
        gb[c0:c1] = dEc * Kc
        dKc += dEc * Bc
        gla[c0:c1] = np.cumsum(dG[::-1], axis=0)[::-1]
        gq[c0:c1], gk[c0:c1], gX[c0:c1] = dQc, dKc, dXc
        dS = dSp
    return gq, gk, gX * w, gla, gb, gX * v, dS


@pytest.mark.parametrize("T", [1, 5, 63, 64, 65, 130])
@pytest.mark.parametrize("C", [4, 8, 64])
def test_chunked_backward_equals_reverse_mode(T, C):
    rng = np.random.default_rng(300 + T * 7 + C)
    dk, dv = 8, 6
    q, k, v, la, b, w, S0 = _rand_inputs(rng, T, 1, 1, dk, dv, S0_scale=0.3)
    dO = rng.standard_normal((T, 1, dv))
    dS_T = rng.standard_normal((1, 1, dk, dv))
    ref = oracle.bwd_ref(q, k, v, la, b, w, dO, S0=S0, dS_T=dS_T, n_seq=1)
    f = lambda x: x[:, 0].astype(np.float64)
    got = chunked_backward(f(q), f(k), f(v), f(la), f(b), f(w), S0[0, 0].astype(np.float64), dO[:, 0],
                           dS_T[0, 0], C)
    names = ["dq", "dk", "dv", "dlog_alpha", "db", "dw", "dS0"]
    for name, a, r in zip(names, got, ref):
        r = np.asarray(r, dtype=np.float64)
        r = r[:, 0] if name != "dS0" else r[0, 0]
        scale = max(1.0, np.abs(r).max())
        assert np.abs(a - r).max() <= 1e-9 * scale, (name, T, C, np.abs(a - r).max())


def test_chunked_backward_strong_decay():
    """Spans of ~100 nats inside a chunk: the ratio form keeps every exponent <= 0."""
    rng = np.random.default_rng(7)
    T, dk, dv = 64, 8, 6
    q, k, v, la, b, w, S0 = _rand_inputs(rng, T, 1, 1, dk, dv, S0_scale=0.3)
    la = (la * 0 - 1.6).astype(np.float32)
    dO = rng.standard_normal((T, 1, dv))
    ref = oracle.bwd_ref(q, k, v, la, b, w, dO, S0=S0, n_seq=1)
    f = lambda x: x[:, 0].astype(np.float64)
    got = chunked_backward(f(q), f(k), f(v), f(la), f(b), f(w), S0[0, 0].astype(np.float64), dO[:, 0], None, 64)
    for a, r in zip(got[:6], ref[:6]):
        r = np.asarray(r, dtype=np.float64)[:, 0]
        assert np.isfinite(a).all()
        assert np.abs(a - r).max() <= 1e-9 * max(1.0, np.abs(r).max())


def factored_backward(q, k, v, la, b, w, S0, dO, dS_T, C):
    """The same gradients in the factored form a tensor-core kernel evaluates: per chunk,
    operands scaled to the chunk's midpoint frame Gref = (G_0 + G_last) / 2 (Khat = K (.)
    exp(G - Gref), Qhat likewise, Kbar = K (.) exp(Gref - G), Ebar likewise, Sref = exp(Gref)
    (.) S), the Gram blocks and their adjoints as plain products of those operands, and the
    frame's own adjoint dGref = rowsum(dSref (.) Sref) - colsum(dKhat (.) Khat + dQhat (.) Qhat)
    + colsum(dKbar (.) Kbar + dEbar (.) Ebar), shared half and half by G_0 and G_last."""
    T, dk = k.shape
    dv = v.shape[1]
    X = w * v
    S = np.zeros((dk, dv)) if S0 is None else S0.copy()
    starts = list(range(0, T, C))
    entry = []
    for c0 in starts:
        c1 = min(T, c0 + C)
        entry.append(S)
        S = _chunk(k[c0:c1], q[c0:c1], la[c0:c1], b[c0:c1], X[c0:c1], S)["S_next"]
    gq, gk, gla, gb, gX = (np.zeros_like(a) for a in (q, k, la, b, X))
    dS = np.zeros((dk, dv)) if dS_T is None else dS_T.copy()
    for ci in reversed(range(len(starts))):
        c0 = starts[ci]
        c1 = min(T, c0 + C)
        n = c1 - c0
        K, Q, Bg, Xc, S = k[c0:c1], q[c0:c1], b[c0:c1], X[c0:c1], entry[ci]
        G = np.cumsum(la[c0:c1], axis=0)
        Gref = 0.5 * (G[0] + G[-1])
        E = Bg * K
        up, dn = np.exp(G - Gref), np.exp(Gref - G)
        Kh, Qh, Kb, Eb = K * up, Q * up, K * dn, E * dn
        Sref = np.exp(Gref)[:, None] * S
        strict, incl = np.tril(np.ones((n, n)), -1), np.tril(np.ones((n, n)))
        A, B = strict * (Kh @ Eb.T), strict * (Kh @ Kb.T)
        P, Qm = incl * (Qh @ Kb.T), incl * (Qh @ Eb.T)
        Tm = np.linalg.inv(np.eye(n) + A)
        Y = Kh @ Sref + B @ Xc
        R = Tm @ Y
        g = np.exp(G[-1])
        tail = np.exp(G[-1][None, :] - G)
        Kt, Et = K * tail, E * tail
        dOc = dO[c0:c1]
        dSp = g[:, None] * dS
        dg = (dS * S).sum(1)
        dKt, dEt = Xc @ dS.T, -(R @ dS.T)
        dXc = Kt @ dS
        dR = -(Et @ dS)
        dQh = dOc @ Sref.T
        dSref = Qh.T @ dOc
        dP = incl * (dOc @ Xc.T)
        dXc += P.T @ dOc
        dQm = -incl * (dOc @ R.T)
        dR -= Qm.T @ dOc
        dTm = dR @ Y.T
        dY = Tm.T @ dR
        dA = -strict * (Tm.T @ dTm @ Tm.T)
        dKh = dY @ Sref.T
        dSref += Kh.T @ dY
        dB = strict * (dY @ Xc.T)
        dXc += B.T @ dY
        dKh += dA @ Eb + dB @ Kb
        dEb = dA.T @ Kh + dQm.T @ Qh
        dKb = dB.T @ Kh + dP.T @ Qh
        dQh += dP @ Kb + dQm @ Eb
        dK = dKh * up + dKb * dn + dKt * tail
        dQ = dQh * up
        dE = dEb * dn + dEt * tail
        tt = dKt * Kt + dEt * Et
        dG = dKh * Kh + dQh * Qh - dKb * Kb - dEb * Eb - tt
        dG[-1] += tt.sum(0) + dg * g
        dGref = (dSref * Sref).sum(1) - (dKh * Kh + dQh * Qh).sum(0) + (dKb * Kb + dEb * Eb).sum(0)
        dG[0] += 0.5 * dGref
        dG[-1] += 0.5 * dGref
        dSp += np.exp(Gref)[:, None] * dSref
        gb[c0:c1] = dE * K
        gla[c0:c1] = np.cumsum(dG[::-1], axis=0)[::-1]
        gq[c0:c1], gk[c0:c1], gX[c0:c1] = dQ, dK + dE * Bg, dXc
        dS = dSp
    return gq, gk, gX * w, gla, gb, gX * v, dS


@pytest.mark.parametrize("T,C", [(1, 64), (63, 64), (130, 64), (37, 8)])
def test_factored_backward_equals_reverse_mode(T, C):
    rng = np.random.default_rng(500 + T + C)
    dk, dv = 8, 6
    q, k, v, la, b, w, S0 = _rand_inputs(rng, T, 1, 1, dk, dv, S0_scale=0.3)
    dO = rng.standard_normal((T, 1, dv))
    dS_T = rng.standard_normal((1, 1, dk, dv))
    ref = oracle.bwd_ref(q, k, v, la, b, w, dO, S0=S0, dS_T=dS_T, n_seq=1)
    f = lambda x: x[:, 0].astype(np.float64)
    got = factored_backward(f(q), f(k), f(v), f(la), f(b), f(w), S0[0, 0].astype(np.float64), dO[:, 0],
                            dS_T[0, 0], C)
    for name, a, r in zip(["dq", "dk", "dv", "dlog_alpha", "db", "dw", "dS0"], got, ref):
        r = np.asarray(r, dtype=np.float64)
        r = r[:, 0] if name != "dS0" else r[0, 0]
        assert np.abs(a - r).max() <= 1e-9 * max(1.0, np.abs(r).max()), name
