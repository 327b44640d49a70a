"""Pins for the oracle: checks against what the pages and the mathematics fix, not against
the oracle itself.

Each test names the passage it follows. Sources:
  * ai-systems-engineering.com, "Delta rule: correcting the state's associations toward
    the new Value" (the worked example, the beta rule, the re-read and other-query facts);
  * tilnote.io note on Gated DeltaNet-2, "Gated DeltaNet-2 design point" (decay, then
    erase on the key axis with b_t, then write on the value axis with w_t);
  * the causal weighted-sum identity of plain linear attention that the delta-rule post
    recalls in its opening paragraph.
"""
import os

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "delta_rule_worked_example.txt")


def _golden():
    vals = {}
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            name, rest = line.split(":", 1)
            nums = rest.split("|", 1)[0].split()
            vals[name.strip()] = np.array([float(x) for x in nums])
    return vals


def _one_token(oracle, S_old, k, v, q, beta_b, beta_w, log_alpha=(0.0, 0.0)):
    """One token through the oracle with dk = dv = 2 and fp32 inputs."""
    f = lambda x: np.asarray(x, dtype=np.float32).reshape(1, 1, 2)
    S0 = np.asarray(S_old, dtype=np.float32).reshape(1, 1, 2, 2)
    o, st = oracle.fwd_ref(f(q), f(k), f(v), f(log_alpha), f(beta_b), f(beta_w), S0=S0, bf16=False)
    return o[0, 0], st[0, 0]


# ---------------------------------------------------------------- worked example (exact)

def test_worked_example_full_correction(oracle_mod):
    """Delta-rule post, "Recording the difference ..." table and Figure 2 right: with the
    unit key [1,0], value [1,1] and full strength, the first state row becomes [1,1], the
    second stays [0,3], and reading back with the key gives [1,1]."""
    g = _golden()
    S_old = np.stack([g["S_old_row0"], g["S_old_row1"]])
    o, st = _one_token(oracle_mod, S_old, g["k"], g["v"], g["k"], [1, 1], [1, 1])
    np.testing.assert_array_equal(st[0], g["S_new_row0"])
    np.testing.assert_array_equal(st[1], g["S_new_row1"])
    np.testing.assert_array_equal(o, g["reread_delta"])
    # the correction written into row 0 is new value minus old read
    np.testing.assert_array_equal(st[0] - S_old[0], g["correction"])
    np.testing.assert_array_equal(g["v"] - g["correction"], g["read_old"])


def test_worked_example_plain_addition(oracle_mod):
    """Figure 2 left of the same post: adding k v^T without the edit reads back [3,1]. In
    the gated form that is erase gate 0 and write gate 1."""
    g = _golden()
    S_old = np.stack([g["S_old_row0"], g["S_old_row1"]])
    o, _ = _one_token(oracle_mod, S_old, g["k"], g["v"], g["k"], [0, 0], [1, 1])
    np.testing.assert_array_equal(o, g["reread_add"])


@pytest.mark.parametrize("beta,key", [(0.0, "beta0_row0"), (0.5, "beta05_row0"), (1.0, "beta1_row0")])
def test_worked_example_beta(oracle_mod, beta, key):
    """Delta-rule post, "Controlling the correction strength with beta", Figure 4: the
    first row becomes [2,0], [1.5,0.5], [1,1] for beta = 0, 0.5, 1 (erase = write = beta),
    and reading back with the unit key gives the same row."""
    g = _golden()
    S_old = np.stack([g["S_old_row0"], g["S_old_row1"]])
    o, st = _one_token(oracle_mod, S_old, g["k"], g["v"], g["k"], [beta] * 2, [beta] * 2)
    np.testing.assert_array_equal(st[0], g[key])
    np.testing.assert_array_equal(st[1], g["S_old_row1"])
    np.testing.assert_array_equal(o, g[key])


@pytest.mark.parametrize("qname", ["q_a", "q_b"])
def test_worked_example_other_queries(oracle_mod, qname):
    """Delta-rule post, "Effect of the state edit on other reads", Figure 5: query [0,1]
    reads [0,3] before and after; query [1,1] reads [2,3] before and [1,4] after. "Before"
    is a token with both gates 0, which leaves the state untouched."""
    g = _golden()
    S_old = np.stack([g["S_old_row0"], g["S_old_row1"]])
    q = g[qname]
    before, _ = _one_token(oracle_mod, S_old, g["k"], g["v"], q, [0, 0], [0, 0])
    after, _ = _one_token(oracle_mod, S_old, g["k"], g["v"], q, [1, 1], [1, 1])
    np.testing.assert_array_equal(before, g[qname + "_before"])
    np.testing.assert_array_equal(after, g[qname + "_after"])


# ---------------------------------------------------------------- invariants

def _rand_inputs(rng, T, h_qk, h_v, dk, dv, unit_k=True, S0_scale=0.0, positive_gates=True):
    q = rng.standard_normal((T, h_qk, dk)).astype(np.float32)
    k = rng.standard_normal((T, h_qk, dk)).astype(np.float32)
    if unit_k:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
        k = k.astype(np.float32)
        q = q.astype(np.float32)
    v = rng.standard_normal((T, h_v, dv)).astype(np.float32)
    la = (-np.log1p(np.exp(rng.standard_normal((T, h_v, dk))))).astype(np.float32)
    sig = lambda x: 1.0 / (1.0 + np.exp(-x))
    b = sig(rng.standard_normal((T, h_v, dk))).astype(np.float32)
    w = sig(rng.standard_normal((T, h_v, dv))).astype(np.float32)
    S0 = None
    if S0_scale:
        S0 = (S0_scale * rng.standard_normal((1, h_v, dk, dv))).astype(np.float32)
    return q, k, v, la, b, w, S0


def test_effect_on_other_queries_invariant(oracle_mod):
    """Delta-rule post, "Effect of the state edit on other reads": after adding
    beta k e^T (e = v - r), a query q reads beta (q.k) e^T more than before. Checked on a
    random 8x6 state with no decay and erase = write = beta."""
    rng = np.random.default_rng(1)
    dk, dv, beta = 8, 6, 0.37
    S_old = rng.standard_normal((dk, dv)).astype(np.float32)
    k = rng.standard_normal(dk).astype(np.float32)
    v = rng.standard_normal(dv).astype(np.float32)
    q = rng.standard_normal(dk).astype(np.float32)
    f = lambda x, d: np.asarray(x, dtype=np.float32).reshape(1, 1, d)
    run = lambda bb: oracle_mod.fwd_ref(f(q, dk), f(k, dk), f(v, dv), f(np.zeros(dk), dk),
                                        f(np.full(dk, bb), dk), f(np.full(dv, bb), dv),
                                        S0=S_old.reshape(1, 1, dk, dv), bf16=False)[0][0, 0]
    before, after = run(0.0), run(np.float32(beta))
    S64, k64, v64, q64 = (x.astype(np.float64) for x in (S_old, k, v, q))
    e = v64 - S64.T @ k64
    np.testing.assert_allclose(after - before, float(np.float32(beta)) * (q64 @ k64) * e,
                               rtol=1e-12, atol=1e-12)


def test_reread_unit_key_full_erase_returns_written_value(oracle_mod):
    """Delta-rule post, "Controlling the correction strength with beta": with a unit key
    and full correction the key reads back exactly the value written. In the gated form,
    erase gate b = 1 and a unit key make the key read back w (.) v after any history and
    any decay. Checked on the last token of a random 40-token sequence by reading with
    q_t = k_t."""
    rng = np.random.default_rng(2)
    T, dk, dv = 40, 16, 12
    q, k, v, la, b, w, S0 = _rand_inputs(rng, T, 1, 1, dk, dv, S0_scale=0.5)
    b[-1] = 1.0
    # an exactly unit key in fp32: +-0.5 on four channels, zero elsewhere
    k[-1] = 0.0
    chans = rng.choice(dk, size=4, replace=False)
    k[-1, 0, chans] = 0.5 * rng.choice([-1.0, 1.0], size=4)
    q[-1] = k[-1]
    o, _ = oracle_mod.fwd_ref(q, k, v, la, b, w, S0=S0, bf16=False)
    expect = w[-1, 0].astype(np.float64) * v[-1, 0].astype(np.float64)
    np.testing.assert_allclose(o[-1, 0], expect, rtol=1e-9, atol=1e-12)


def test_reread_general_invariant(oracle_mod):
    """Delta-rule post, same section: reading back with the key gives r + beta (k.k) e;
    the gated generalisation is S_t^T k_t = (1 - k.(b(.)k)) r_t + (k.k)(w(.)v), with r_t the
    key read of the decayed old state. The old state comes from the oracle run on the
    prefix; non-unit keys are used on purpose (the post notes the k.k factor)."""
    rng = np.random.default_rng(3)
    T, dk, dv = 25, 8, 5
    q, k, v, la, b, w, S0 = _rand_inputs(rng, T, 1, 1, dk, dv, unit_k=False, S0_scale=0.3)
    _, S_prev = oracle_mod.fwd_ref(q[:-1], k[:-1], v[:-1], la[:-1], b[:-1], w[:-1], S0=S0, bf16=False)
    q2 = q.copy()
    q2[-1] = k[-1]
    o, _ = oracle_mod.fwd_ref(q2, k, v, la, b, w, S0=S0, bf16=False)
    k64, b64 = k[-1, 0].astype(np.float64), b[-1, 0].astype(np.float64)
    x = w[-1, 0].astype(np.float64) * v[-1, 0].astype(np.float64)
    S_dec = np.exp(la[-1, 0].astype(np.float64))[:, None] * S_prev[0, 0]
    r = S_dec.T @ k64
    expect = (1.0 - k64 @ (b64 * k64)) * r + (k64 @ k64) * x
    np.testing.assert_allclose(o[-1, 0], expect, rtol=1e-10, atol=1e-10)


def test_no_erase_equals_decayed_causal_sum(oracle_mod):
    """With erase gate 0 the recurrence is plain gated accumulation, whose output has the
    closed form o_t = sum_{s<=t} sum_c q_tc k_sc exp(G_tc - G_sc) w_s(.)v_s
    + sum_c q_tc exp(G_tc) S0[c,:], G_t = cumulative log-decay. With no decay, w = 1 and
    S0 = 0 this is the causal weighted sum sum_{s<=t} (q_t.k_s) v_s that the delta-rule post
    recalls in its opening paragraph. Brute force O(T^2) in fp64."""
    rng = np.random.default_rng(4)
    T, dk, dv = 48, 8, 6
    q, k, v, la, b, w, S0 = _rand_inputs(rng, T, 1, 1, dk, dv, S0_scale=0.5)
    b[:] = 0.0
    o, st = oracle_mod.fwd_ref(q, k, v, la, b, w, S0=S0, bf16=False)
    q64, k64 = q[:, 0].astype(np.float64), k[:, 0].astype(np.float64)
    x = w[:, 0].astype(np.float64) * v[:, 0].astype(np.float64)
    G = np.cumsum(la[:, 0].astype(np.float64), axis=0)
    S0_64 = S0[0, 0].astype(np.float64)
    for t in range(T):
        acc = (q64[t] * np.exp(G[t])) @ S0_64
        for s in range(t + 1):
            acc = acc + np.sum(q64[t] * k64[s] * np.exp(G[t] - G[s])) * x[s]
        np.testing.assert_allclose(o[t, 0], acc, rtol=1e-9, atol=1e-12)
    # plain causal sum: no decay, w = 1, S0 = 0
    la0 = np.zeros_like(la)
    w1 = np.ones_like(w)
    o2, _ = oracle_mod.fwd_ref(q, k, v, la0, b, w1, bf16=False)
    v64 = v[:, 0].astype(np.float64)
    causal = np.array([sum((q64[t] @ k64[s]) * v64[s] for s in range(t + 1)) for t in range(T)])
    np.testing.assert_allclose(o2[:, 0], causal, rtol=1e-10, atol=1e-12)


def _delta_rule_textbook(q, k, v, beta, log_alpha=None):
    """The delta rule exactly as the delta-rule post states it, sections "Recording the
    difference ..." and "Controlling the correction strength with beta": r^T = k^T S,
    e^T = v^T - r^T, S <- S + beta k e^T, output read with the query from the updated state.
    With ``log_alpha`` the state is first decayed channel-wise (the KDA form the note on
    Gated DeltaNet-2 says the layer inherits)."""
    T, dk = k.shape
    dv = v.shape[1]
    S = np.zeros((dk, dv))
    out = np.zeros((T, dv))
    for t in range(T):
        if log_alpha is not None:
            S = np.exp(log_alpha[t])[:, None] * S
        e = v[t] - k[t] @ S
        S = S + beta[t] * np.outer(k[t], e)
        out[t] = q[t] @ S
    return out, S


@pytest.mark.parametrize("with_decay", [False, True])
def test_reduces_to_delta_rule_and_kda(oracle_mod, with_decay):
    """With erase gate = write gate = beta_t * 1 the recurrence must be the delta rule of the
    delta-rule post (no decay) or its KDA form (channel-wise decay first)."""
    rng = np.random.default_rng(5)
    T, dk, dv = 64, 16, 8
    q, k, v, la, b, w, _ = _rand_inputs(rng, T, 1, 1, dk, dv)
    beta = (1.0 / (1.0 + np.exp(-rng.standard_normal(T)))).astype(np.float32)
    bb = np.repeat(beta[:, None, None], dk, axis=2).astype(np.float32)
    ww = np.repeat(beta[:, None, None], dv, axis=2).astype(np.float32)
    if not with_decay:
        la = np.zeros_like(la)
    o, st = oracle_mod.fwd_ref(q, k, v, la, bb, ww, bf16=False)
    ref_o, ref_S = _delta_rule_textbook(q[:, 0].astype(np.float64), k[:, 0].astype(np.float64),
                                        v[:, 0].astype(np.float64), beta.astype(np.float64),
                                        la[:, 0].astype(np.float64) if with_decay else None)
    np.testing.assert_allclose(o[:, 0], ref_o, rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(st[0, 0], ref_S, rtol=1e-9, atol=1e-12)


def test_nonuniform_gates_hand_computed(oracle_mod):
    """Channel-wise erase and write gates, computed by hand from the adopted form
    S_t = (I - (b(.)k) k^T) Diag(alpha) S + k (w(.)v)^T (the reading of the note on Gated
    DeltaNet-2: b_t acts on the key axis, w_t on the value axis, after the decay).
      S_old = [[2,0],[0,3]], alpha = [0.5, 1], k = [0.6, 0.8], b = [1, 0.5],
      v = [1, 2], w = [1, 0.25].
      Diag(alpha) S_old = [[1,0],[0,3]];  r = [0.6, 2.4];  b(.)k = [0.6, 0.4]
      erase:  [[1,0],[0,3]] - [[0.36,1.44],[0.24,0.96]] = [[0.64,-1.44],[-0.24,2.04]]
      write:  + k (w(.)v)^T = + [[0.6,0.3],[0.8,0.4]]   -> [[1.24,-1.14],[0.56,2.44]]
    Query [1,0] reads [1.24,-1.14]; query [0,1] reads [0.56,2.44]. (The other reading,
    erasing with k (b(.)k)^T, would give row 0 = [0.52,-1.92].)"""
    S_old = [[2, 0], [0, 3]]
    la = [np.log(np.float32(0.5)), 0.0]
    k, b, v, w = [0.6, 0.8], [1.0, 0.5], [1.0, 2.0], [1.0, 0.25]
    o1, st = _one_token(oracle_mod, S_old, k, v, [1, 0], b, w, log_alpha=la)
    o2, _ = _one_token(oracle_mod, S_old, k, v, [0, 1], b, w, log_alpha=la)
    tol = dict(rtol=0, atol=2e-6)  # 0.6, 0.8 and log(0.5) are fp32-rounded inputs
    np.testing.assert_allclose(st, [[1.24, -1.14], [0.56, 2.44]], **tol)
    np.testing.assert_allclose(o1, [1.24, -1.14], **tol)
    np.testing.assert_allclose(o2, [0.56, 2.44], **tol)


# ---------------------------------------------------------------- structural properties

def test_value_columns_independent(oracle_mod):
    """The transition acts on the key axis only, so each value column of the state evolves
    on its own: running the value channels one at a time gives the same outputs and states."""
    rng = np.random.default_rng(6)
    T, dk, dv = 30, 8, 5
    q, k, v, la, b, w, S0 = _rand_inputs(rng, T, 1, 1, dk, dv, S0_scale=0.4)
    o, st = oracle_mod.fwd_ref(q, k, v, la, b, w, S0=S0, bf16=False)
    for j in range(dv):
        sl = slice(j, j + 1)
        oj, sj = oracle_mod.fwd_ref(q, k, np.ascontiguousarray(v[:, :, sl]), la, b,
                                    np.ascontiguousarray(w[:, :, sl]),
                                    S0=np.ascontiguousarray(S0[:, :, :, sl]), bf16=False)
        np.testing.assert_array_equal(oj[:, :, 0], o[:, :, j])
        np.testing.assert_array_equal(sj[..., 0], st[..., j])


def test_split_sequence_resume(oracle_mod):
    """The final state is a checkpoint: running [0,t0) then [t0,T) from the returned state
    reproduces one run over [0,T) (the fixed-size state of the note's opening sections)."""
    rng = np.random.default_rng(7)
    T, t0, dk, dv = 50, 21, 8, 6
    q, k, v, la, b, w, S0 = _rand_inputs(rng, T, 1, 1, dk, dv, S0_scale=0.2)
    o, st = oracle_mod.fwd_ref(q, k, v, la, b, w, S0=S0, bf16=False)
    oa, sa = oracle_mod.fwd_ref(q[:t0], k[:t0], v[:t0], la[:t0], b[:t0], w[:t0], S0=S0, bf16=False)
    ob, sb = oracle_mod.fwd_ref(q[t0:], k[t0:], v[t0:], la[t0:], b[t0:], w[t0:],
                                S0=sa.astype(np.float32), bf16=False)
    np.testing.assert_allclose(np.concatenate([oa, ob]), o, rtol=1e-6, atol=1e-6)
    np.testing.assert_allclose(sb, st, rtol=1e-6, atol=1e-6)


def test_varlen_equals_separate_and_grouped_heads(oracle_mod):
    """Packed sequences (cu_seqlens) equal separate runs, the state resets at each boundary,
    zero-length sequences return S0, and value head h reads query/key head h // (Hv/Hqk)
    (the grouped layout of the Gated DeltaNet wiki page: 16 query/key heads, 32 value heads)."""
    rng = np.random.default_rng(8)
    lens = [5, 0, 17, 1, 9]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T, h_qk, h_v, dk, dv = int(cu[-1]), 2, 4, 8, 4
    q, k, v, la, b, w, _ = _rand_inputs(rng, T, h_qk, h_v, dk, dv)
    S0 = (0.3 * rng.standard_normal((len(lens), h_v, dk, dv))).astype(np.float32)
    o, st = oracle_mod.fwd_ref(q, k, v, la, b, w, S0=S0, cu_seqlens=cu, bf16=False)
    for n in range(len(lens)):
        a, z = cu[n], cu[n + 1]
        for h in range(h_v):
            g = h // (h_v // h_qk)
            sl = lambda x, hh: np.ascontiguousarray(x[a:z, hh:hh + 1])
            on, sn = oracle_mod.fwd_ref(sl(q, g), sl(k, g), sl(v, h), sl(la, h), sl(b, h), sl(w, h),
                                        S0=np.ascontiguousarray(S0[n:n + 1, h:h + 1]), bf16=False)
            np.testing.assert_array_equal(on[:, 0], o[a:z, h])
            np.testing.assert_array_equal(sn[0, 0], st[n, h])
        if lens[n] == 0:
            np.testing.assert_array_equal(st[n], S0[n].astype(np.float64))


def test_bf16_inputs_widen_exactly(oracle_mod):
    """bf16 inputs are read as their exact values: the same numbers given as fp32 and as
    bf16 bit patterns produce bit-identical fp64 results."""
    rng = np.random.default_rng(9)
    T, dk, dv = 12, 4, 4
    q, k, v, la, b, w, _ = _rand_inputs(rng, T, 1, 1, dk, dv)
    to_bf16_bits = lambda x: (np.asarray(x, np.float32).view(np.uint32) >> 16).astype(np.uint16)
    from_bits = lambda u: (u.astype(np.uint32) << 16).view(np.float32)
    bq, bk, bv, bb, bw = (to_bf16_bits(x) for x in (q, k, v, b, w))
    o1, s1 = oracle_mod.fwd_ref(bq, bk, bv, la, bb, bw, bf16=True)
    o2, s2 = oracle_mod.fwd_ref(from_bits(bq), from_bits(bk), from_bits(bv), la, from_bits(bb),
                                from_bits(bw), bf16=False)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(s1, s2)


def test_rejects_bad_arguments(oracle_mod):
    """Malformed cu_seqlens and non-divisible head counts are rejected, not guessed."""
    rng = np.random.default_rng(10)
    q, k, v, la, b, w, _ = _rand_inputs(rng, 6, 2, 3, 4, 4)
    with pytest.raises(ValueError):
        oracle_mod.fwd_ref(q, k, v, la, b, w, bf16=False)      # 3 value heads, 2 qk heads
    q, k, v, la, b, w, _ = _rand_inputs(rng, 6, 1, 1, 4, 4)
    with pytest.raises(ValueError):
        oracle_mod.fwd_ref(q, k, v, la, b, w, cu_seqlens=np.array([0, 4, 3, 6], np.int32), bf16=False)
    with pytest.raises(ValueError):
        oracle_mod.fwd_ref(q, k, v, la, b, w, cu_seqlens=np.array([0, 4, 5], np.int32), bf16=False)
