"""Serving-style decode (gdn2_decode_multi): states in a slot pool, several tokens per step,
optional state after every token. Checked through the C ABI against the fp64 oracle run on
each active sequence's tokens from its slot's state, and against the single-token decode
and the prefill path on the same tokens."""
import numpy as np
import pytest
import torch

from gated_delta_rule_160_b200 import workloads as W
from tests.parity import TOL, rel_err

pytestmark = pytest.mark.gpu

D = 128


@pytest.fixture(scope="module")
def g():
    import gated_delta_rule_160_b200 as g
    g.load_library()
    assert torch.cuda.is_available()
    return g


def _tokens(N, n_tok, H, dtype, seed):
    d = W.token_inputs(N * n_tok, H, H, D, D, dtype, "cuda", seed=seed)
    return {k_: t.view(N, n_tok, *t.shape[1:]) for k_, t in d.items()}


def _oracle(oracle_mod, d, n, t_end, S0):
    """Oracle on tokens 0 .. t_end-1 of sequence n, from state S0 [H, dk, dv]."""
    sl = {k_: d[k_][n, :t_end].cpu() for k_ in ("q", "k", "v", "log_alpha", "b", "w")}
    o, st = oracle_mod.fwd_ref(sl["q"], sl["k"], sl["v"], sl["log_alpha"], sl["b"], sl["w"],
                               S0=S0[None].cpu(), n_seq=1)
    return o, st[0]


def test_slot_pool_multi_token_matches_oracle(g, oracle_mod):
    N, n_tok, H, n_slots = 5, 4, 2, 12
    slots = [7, 2, -1, 11, 0]
    d = _tokens(N, n_tok, H, torch.bfloat16, seed=31)
    pool = W.state_input(n_slots, H, D, D, 0.05, "cuda", seed=31)
    before = pool.clone()
    o = torch.full((N, n_tok, H, D), 123.0, device="cuda")
    slots_t = torch.tensor(slots, dtype=torch.int32, device="cuda")
    o, steps = g.gdn2_decode_multi(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], pool,
                                   slots=slots_t, o=o, want_steps=True)
    torch.cuda.synchronize()
    tol = TOL[torch.float32]  # the decode kernel's arithmetic is fp32 on bf16 inputs
    o_got, o_ref, s_got, s_ref = [], [], [], []
    for n, s in enumerate(slots):
        if s < 0:
            assert torch.all(o[n] == 123.0), "an inactive sequence's rows of o were written"
            continue
        ref_o, ref_s = _oracle(oracle_mod, d, n, n_tok, before[s])
        o_got.append(o[n])
        o_ref.append(ref_o)
        s_got.append(pool[s])
        s_ref.append(ref_s)
        for t in range(n_tok):  # the state after token t
            _, st = _oracle(oracle_mod, d, n, t + 1, before[s])
            assert rel_err(steps[n, t], st) <= tol, (n, t)
    eo = rel_err(torch.stack(o_got), np.stack(o_ref))
    es = rel_err(torch.stack(s_got), np.stack(s_ref))
    print(f"serving decode: o err {eo:.3e}, S err {es:.3e} (tol {tol})")
    assert eo <= tol and es <= tol
    untouched = [s for s in range(n_slots) if s not in slots]
    assert torch.equal(pool[untouched], before[untouched])


def test_single_token_equals_decode_step(g):
    N, H = 6, 2
    d = _tokens(N, 1, H, torch.bfloat16, seed=32)
    S = W.state_input(N, H, D, D, 0.05, "cuda", seed=32)
    S_a, S_b, S_c = S.clone(), S.clone(), S.clone()
    o_a = g.gdn2_decode_step(*(d[k_][:, 0] for k_ in ("q", "k", "v", "log_alpha", "b", "w")), S_a)
    o_b, _ = g.gdn2_decode_multi(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], S_b)
    o_c, steps = g.gdn2_decode_multi(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], S_c,
                                     want_steps=True)
    torch.cuda.synchronize()
    assert torch.equal(o_a, o_b[:, 0]) and torch.equal(S_a, S_b)
    torch.testing.assert_close(o_c[:, 0], o_a, rtol=1e-6, atol=1e-7)
    torch.testing.assert_close(S_c, S_a, rtol=1e-6, atol=1e-7)
    torch.testing.assert_close(steps[:, 0], S_a, rtol=1e-6, atol=1e-7)


def test_multi_token_equals_prefill(g):
    """n_tok decode tokens from a state == prefill of the same n_tok tokens from that state."""
    N, n_tok, H = 3, 8, 2
    d = _tokens(N, n_tok, H, torch.float32, seed=33)
    S0 = W.state_input(N, H, D, D, 0.05, "cuda", seed=33)
    pool = S0.clone()
    o_dec, _ = g.gdn2_decode_multi(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], pool)
    flat = {k_: t.reshape(N * n_tok, *t.shape[2:]) for k_, t in d.items()}
    o_pre, S_pre = g.gdn2_chunk_fwd(flat["q"], flat["k"], flat["v"], flat["log_alpha"], flat["b"], flat["w"],
                                    S0=S0, n_seq=N)
    torch.cuda.synchronize()
    torch.testing.assert_close(o_dec.reshape(N * n_tok, H, D), o_pre, rtol=1e-4, atol=1e-5)
    torch.testing.assert_close(pool, S_pre, rtol=1e-4, atol=1e-5)


@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 128), (128, 64)])
@pytest.mark.parametrize("n_tok", [1, 4, 8])
@pytest.mark.parametrize("want_steps", [False, True])
def test_narrow_heads_match_oracle(g, oracle_mod, dk, dv, n_tok, want_steps):
    """Every key/value width of the serving-decode kernels (64 and 128), 1, 4 and 8 tokens,
    with and without the per-token states, over a pool with inactive and out-of-range slots;
    element by element against the oracle run from each active slot's state."""
    N, H, n_slots = 6, 2, 9
    slots = [4, -1, 8, 0, 9, 2]  # -1 and 9 (>= n_slots) are skipped
    d = W.token_inputs(N * n_tok, H, H, dk, dv, torch.bfloat16, "cuda", seed=50 + dk + dv + n_tok)
    d = {k_: t.view(N, n_tok, *t.shape[1:]) for k_, t in d.items()}
    pool = W.state_input(n_slots, H, dk, dv, 0.05, "cuda", seed=51 + n_tok)
    before = pool.clone()
    o = torch.full((N, n_tok, H, dv), 123.0, device="cuda")
    slots_t = torch.tensor(slots, dtype=torch.int32, device="cuda")
    o, steps = g.gdn2_decode_multi(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], pool,
                                   slots=slots_t, o=o, want_steps=want_steps)
    torch.cuda.synchronize()
    tol = TOL[torch.float32]
    o_got, o_ref, s_got, s_ref = [], [], [], []
    for n, s in enumerate(slots):
        if not 0 <= s < n_slots:
            assert torch.all(o[n] == 123.0), "a skipped sequence's rows of o were written"
            continue
        ref_o, ref_s = _oracle(oracle_mod, d, n, n_tok, before[s])
        o_got.append(o[n])
        o_ref.append(ref_o)
        s_got.append(pool[s])
        s_ref.append(ref_s)
        if want_steps:
            for t in range(n_tok):
                _, st = _oracle(oracle_mod, d, n, t + 1, before[s])
                assert rel_err(steps[n, t], st) <= tol, (n, t)
    eo = rel_err(torch.stack(o_got), np.stack(o_ref))
    es = rel_err(torch.stack(s_got), np.stack(s_ref))
    assert eo <= tol and es <= tol, (eo, es)
    untouched = [s for s in range(n_slots) if s not in slots]
    assert torch.equal(pool[untouched], before[untouched])
