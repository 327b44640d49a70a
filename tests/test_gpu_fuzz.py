"""Seeded random configurations through the C ABI against the fp64 oracle: dtypes, key and
value widths, head groupings, ragged and empty packed sequences, initial states; decode over
a slot pool with inactive slots and 1..8 tokens; bursts of strong decay; and the gradients. Small sizes, so the
oracle sees whole tensors."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_160_b200 import workloads as W
from tests.parity import TOL, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    import gated_delta_rule_160_b200 as g
    g.load_library()
    assert torch.cuda.is_available()
    return g


def _config(seed):
    rng = np.random.default_rng(seed)
    dk, dv = int(rng.choice([64, 128])), int(rng.choice([64, 128]))
    dtype = torch.bfloat16 if rng.random() < 0.6 else torch.float32
    if rng.random() < 0.5:  # the tensor-core path's shape, more often
        dk = dv = 128
        dtype = torch.bfloat16
    h_qk = int(rng.choice([1, 2]))
    h_v = h_qk * int(rng.choice([1, 2]))
    n = int(rng.integers(1, 5))
    lens = [int(x) for x in rng.choice([0, 1, 17, 63, 64, 65, 100, 130], size=n)]
    return dict(dk=dk, dv=dv, dtype=dtype, h_qk=h_qk, h_v=h_v, lens=lens, with_S0=bool(rng.random() < 0.5))


@pytest.mark.parametrize("seed", range(12))
def test_fuzz_chunk_fwd(g, seed):
    c = _config(1000 + seed)
    T = sum(c["lens"])
    d = W.token_inputs(T, c["h_qk"], c["h_v"], c["dk"], c["dv"], c["dtype"], "cuda", seed=seed)
    S0 = W.state_input(len(c["lens"]), c["h_v"], c["dk"], c["dv"], 0.05, "cuda", seed=seed) if c["with_S0"] else None
    cu = torch.tensor(np.concatenate([[0], np.cumsum(c["lens"])]), dtype=torch.int32, device="cuda")
    o, st = g.gdn2_chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], S0=S0, cu_seqlens=cu)
    torch.cuda.synchronize()
    o_ref, s_ref = oracle.fwd_ref(*(d[k].cpu() for k in ("q", "k", "v", "log_alpha", "b", "w")),
                                  S0=None if S0 is None else S0.cpu(), cu_seqlens=cu.cpu())
    tol = TOL[c["dtype"]]
    eo, es = rel_err(o, o_ref), rel_err(st, s_ref)
    print(f"fuzz chunk {c}: o {eo:.2e}, S_T {es:.2e}")
    assert eo <= tol and es <= tol, c


@pytest.mark.parametrize("seed", range(6))
def test_fuzz_chunk_fwd_decay_spikes(g, seed):
    """The tensor-core shape with bursts of strong decay: random (token range, value head,
    channel) blocks at -2 .. -9 per token and single tokens at -20 .. -120, so that some
    (sequence, head) pairs leave the chunk frame's range (and are recomputed token by token)
    and others stay just inside it. Every pair is checked against the oracle."""
    rng = np.random.default_rng(3000 + seed)
    h_qk = int(rng.choice([1, 2]))
    h_v = h_qk * int(rng.choice([1, 2]))
    lens = [int(x) for x in rng.choice([1, 63, 64, 65, 130, 200], size=int(rng.integers(1, 4)))]
    T = sum(lens)
    d = W.token_inputs(T, h_qk, h_v, 128, 128, torch.bfloat16, "cuda", seed=seed)
    la = d["log_alpha"].clone()
    for _ in range(int(rng.integers(1, 4))):
        t0 = int(rng.integers(0, T))
        t1 = min(T, t0 + int(rng.integers(8, 80)))
        c0 = int(rng.integers(0, 120))
        la[t0:t1, int(rng.integers(0, h_v)), c0:c0 + int(rng.integers(1, 9))] = -float(rng.uniform(2.0, 9.0))
    for _ in range(int(rng.integers(0, 4))):
        la[int(rng.integers(0, T)), int(rng.integers(0, h_v)), int(rng.integers(0, 128))] = -float(rng.uniform(20, 120))
    d["log_alpha"] = la
    S0 = W.state_input(len(lens), h_v, 128, 128, 0.05, "cuda", seed=seed)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device="cuda")
    g.gdn2_device_status()
    o, st = g.gdn2_chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], S0=S0, cu_seqlens=cu)
    torch.cuda.synchronize()
    flags = g.gdn2_device_status()
    assert flags & ~g.GDN2_DEVICE_DECAY_RANGE == 0
    o_ref, s_ref = oracle.fwd_ref(*(d[k].cpu() for k in ("q", "k", "v", "log_alpha", "b", "w")),
                                  S0=S0.cpu(), cu_seqlens=cu.cpu())
    eo, es = rel_err(o, o_ref), rel_err(st, s_ref)
    print(f"fuzz decay spikes {seed}: lens {lens}, heads {h_qk}/{h_v}, recomputed {bool(flags)}: "
          f"o {eo:.2e}, S_T {es:.2e}")
    assert eo <= TOL[torch.bfloat16] and es <= TOL[torch.bfloat16]


@pytest.mark.parametrize("seed", range(8))
def test_fuzz_decode_multi(g, seed):
    rng = np.random.default_rng(2000 + seed)
    c = _config(2000 + seed)
    N, n_tok = int(rng.integers(1, 6)), int(rng.integers(1, 9))
    n_slots = N + int(rng.integers(0, 4))
    slots = [int(x) for x in rng.permutation(n_slots)[:N]]
    slots = [-1 if rng.random() < 0.2 else s for s in slots]  # some inactive sequences
    d = W.token_inputs(N * n_tok, c["h_qk"], c["h_v"], c["dk"], c["dv"], c["dtype"], "cuda", seed=seed)
    d = {k: t.view(N, n_tok, *t.shape[1:]) for k, t in d.items()}
    pool = W.state_input(n_slots, c["h_v"], c["dk"], c["dv"], 0.05, "cuda", seed=seed)
    before = pool.clone()
    want_steps = bool(rng.random() < 0.5)
    slots_t = torch.tensor(slots, dtype=torch.int32, device="cuda")
    o, steps = g.gdn2_decode_multi(*(d[k] for k in ("q", "k", "v", "log_alpha", "b", "w")), pool, slots=slots_t,
                                   want_steps=want_steps)
    torch.cuda.synchronize()
    tol = TOL[torch.float32]  # fp32 arithmetic
    for n, s in enumerate(slots):
        if s < 0:
            continue
        o_ref, s_ref = oracle.fwd_ref(*(d[k][n].cpu() for k in ("q", "k", "v", "log_alpha", "b", "w")),
                                      S0=before[s:s + 1].cpu())
        assert rel_err(o[n], o_ref) <= tol, (c, n)
        assert rel_err(pool[s], s_ref[0]) <= tol, (c, n)
        if want_steps:
            _, s_mid = oracle.fwd_ref(*(d[k][n, :1].cpu() for k in ("q", "k", "v", "log_alpha", "b", "w")),
                                      S0=before[s:s + 1].cpu())
            assert rel_err(steps[n, 0], s_mid[0]) <= tol, (c, n)
    untouched = [s for s in range(n_slots) if s not in slots]
    assert torch.equal(pool[untouched], before[untouched])


@pytest.mark.parametrize("seed", range(6))
def test_fuzz_backward(g, seed):
    c = _config(3000 + seed)
    c["lens"] = [min(L, 70) for L in c["lens"]]  # the oracle differentiates every token
    T = sum(c["lens"])
    d = W.token_inputs(T, c["h_qk"], c["h_v"], c["dk"], c["dv"], c["dtype"], "cuda", seed=seed)
    S0 = W.state_input(len(c["lens"]), c["h_v"], c["dk"], c["dv"], 0.05, "cuda", seed=seed) if c["with_S0"] else None
    gen = torch.Generator(device="cuda").manual_seed(seed)
    dO = torch.randn(T, c["h_v"], c["dv"], generator=gen, device="cuda")
    dS = torch.randn(len(c["lens"]), c["h_v"], c["dk"], c["dv"], generator=gen, device="cuda")
    cu = torch.tensor(np.concatenate([[0], np.cumsum(c["lens"])]), dtype=torch.int32, device="cuda")
    got = g.gdn2_chunk_bwd(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], dO, S0=S0, dS_T=dS, cu_seqlens=cu)
    torch.cuda.synchronize()
    ref = oracle.bwd_ref(*(d[k] for k in ("q", "k", "v", "log_alpha", "b", "w")), dO, S0=S0, dS_T=dS,
                         cu_seqlens=cu.cpu())
    for name, a, r in zip(["dq", "dk", "dv", "dlog_alpha", "db", "dw", "dS0"], got, ref):
        err = rel_err(a, r)
        assert err <= 1e-4, (c, name, err)
