"""Full-size parity of the backward, the fused pre-processing and the serving decode.

Each path runs on the GPU (through the C ABI) over the whole workload in the launch
configuration the benchmark times; the oracle recomputes sampled (sequence, head) pairs one
by one and the sampled outputs are compared element by element.
"""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_160_b200 import workloads as W
from tests.parity import TOL, rel_err

pytestmark = pytest.mark.gpu

PREFILL = "prefill_b8_h16_t4096"
DECODE = "decode_256seq_h32"


@pytest.fixture(scope="module")
def g():
    import gated_delta_rule_160_b200 as g
    g.load_library()
    assert torch.cuda.is_available()
    return g


def _slice(d, n, h, T):
    """Tokens of sequence n (all sequences T long) and value head h = query/key head h."""
    s = slice(n * T, (n + 1) * T)
    return {key: d[key][s, h:h + 1].cpu() for key in ("q", "k", "v", "log_alpha", "b", "w")}


def _S0(d, n, h):
    return None if d["S0"] is None else d["S0"][n:n + 1, h:h + 1].cpu()


def test_backward_full_size_sampled(g):
    """gdn2_chunk_bwd on all 8 x 16 x 4096 token-heads; the oracle differentiates (sequence,
    head) pairs (0, 0) and (7, 15) one at a time (query/key head = value head here)."""
    wl = W.WORKLOADS[PREFILL]
    d = W.prefill_inputs(wl, "cuda")
    dO = torch.randn(d["v"].shape, generator=torch.Generator(device="cuda").manual_seed(wl.seed + 29),
                     device="cuda")
    got = g.gdn2_chunk_bwd(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], dO, S0=d["S0"],
                           n_seq=d["n_seq"])
    torch.cuda.synchronize()
    names = ["dq", "dk", "dv", "dlog_alpha", "db", "dw"]
    cols = {name: ([], []) for name in names + ["dS0"]}
    T = wl.T
    for n, h in [(0, 0), (7, 15)]:
        x = _slice(d, n, h, T)
        ref = oracle.bwd_ref(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"],
                             dO[n * T:(n + 1) * T, h:h + 1].cpu(), S0=_S0(d, n, h), n_seq=1)
        for name, a, r in zip(names, got[:6], ref[:6]):
            cols[name][0].append(a[n * T:(n + 1) * T, h])
            cols[name][1].append(r[:, 0])
        cols["dS0"][0].append(got[6][n, h])
        cols["dS0"][1].append(ref[6][0, 0])
    for name, (a, r) in cols.items():
        err = rel_err(torch.stack(a), np.stack(r))
        print(f"backward full size: {name} err {err:.3e}")
        assert err <= 1e-4, name  # fp32 arithmetic


def test_prologue_full_size_sampled(g):
    """gdn2_chunk_fwd_prologue on the 8 x 16 x 4096 workload from raw bf16 projections (the
    recipe of the benchmark's fused pre-processing leg); oracle: prologue_ref then fwd_ref on
    (sequence, head) pairs (0, 0) and (7, 15)."""
    wl = W.WORKLOADS[PREFILL]
    d = W.prefill_inputs(wl, "cuda")
    T_all = int(sum(d["lengths"]))
    gen = torch.Generator(device="cuda").manual_seed(wl.seed + 17)
    rn = lambda *shp: torch.randn(*shp, generator=gen, device="cuda").to(wl.dtype)
    raw = dict(q=rn(T_all, wl.h_qk, wl.dk), k=rn(T_all, wl.h_qk, wl.dk), a=rn(T_all, wl.h_v, wl.dk),
               b=rn(T_all, wl.h_v, wl.dk), w=rn(T_all, wl.h_v, wl.dv))
    o, st = g.gdn2_chunk_fwd(raw["q"], raw["k"], d["v"], raw["a"], raw["b"], raw["w"], S0=d["S0"],
                             n_seq=d["n_seq"], prologue=True)
    torch.cuda.synchronize()
    T = wl.T
    f32 = lambda x: np.asarray(x, dtype=np.float32)
    o_got, o_ref, s_got, s_ref = [], [], [], []
    for n, h in [(0, 0), (7, 15)]:
        s = slice(n * T, (n + 1) * T)
        q, k, la, b, w = oracle.prologue_ref(raw["q"][s, h:h + 1], raw["k"][s, h:h + 1], raw["a"][s, h:h + 1],
                                             raw["b"][s, h:h + 1], raw["w"][s, h:h + 1])
        ro, rs = oracle.fwd_ref(f32(q), f32(k), d["v"][s, h:h + 1].float().cpu().numpy(), f32(la), f32(b), f32(w),
                                S0=_S0(d, n, h), n_seq=1, bf16=False)
        o_got.append(o[s, h])
        o_ref.append(ro[:, 0])
        s_got.append(st[n, h])
        s_ref.append(rs[0, 0])
    eo = rel_err(torch.stack(o_got), np.stack(o_ref))
    es = rel_err(torch.stack(s_got), np.stack(s_ref))
    tol = TOL[torch.bfloat16]
    print(f"prologue full size: o err {eo:.3e}, S_T err {es:.3e} (tol {tol})")
    assert eo <= tol and es <= tol


def test_serving_decode_full_size_sampled(g):
    """gdn2_decode_multi on all 256 x 32 states at seeded-random slots of a 512-state pool,
    4 tokens per sequence and step (the benchmark's serving leg), three steps; the oracle
    replays sampled (sequence, head) pairs as 12-token sequences from the slot's state."""
    wl = W.WORKLOADS[DECODE]
    N, n_tok, steps = wl.n_seq, 4, 3
    pool = torch.zeros((2 * N, wl.h_v, wl.dk, wl.dv), dtype=torch.float32, device="cuda")
    perm = torch.randperm(2 * N, generator=torch.Generator().manual_seed(wl.seed))[:N]
    S_init = W.decode_state(wl, "cuda")
    pool[perm.to("cuda")] = S_init
    slots = perm.to(torch.int32).to("cuda")
    ins, outs = [], []
    for s_ in range(steps):
        t_ = W.token_inputs(N * n_tok, wl.h_qk, wl.h_v, wl.dk, wl.dv, wl.dtype, "cuda", wl.seed * 7919 + s_)
        x = {key: t.view(N, n_tok, *t.shape[1:]) for key, t in t_.items()}
        o, _ = g.gdn2_decode_multi(*(x[key] for key in ("q", "k", "v", "log_alpha", "b", "w")), pool, slots=slots)
        ins.append(x)
        outs.append(o)
    torch.cuda.synchronize()
    tol = TOL[torch.float32]  # fp32 arithmetic in the decode kernel
    o_got, o_ref, s_got, s_ref = [], [], [], []
    for n, h in [(0, 0), (255, 31), (100, 17)]:
        seq = {key: torch.cat([x[key][n, :, h:h + 1] for x in ins]).cpu()
               for key in ("q", "k", "v", "log_alpha", "b", "w")}
        ro, rs = oracle.fwd_ref(seq["q"], seq["k"], seq["v"], seq["log_alpha"], seq["b"], seq["w"],
                                S0=S_init[n:n + 1, h:h + 1].cpu(), n_seq=1)
        o_got.append(torch.cat([o[n, :, h] for o in outs]))
        o_ref.append(ro[:, 0])
        s_got.append(pool[int(perm[n]), h])
        s_ref.append(rs[0, 0])
    eo = rel_err(torch.stack(o_got), np.stack(o_ref))
    es = rel_err(torch.stack(s_got), np.stack(s_ref))
    print(f"serving decode full size: o err {eo:.3e}, S err {es:.3e} (tol {tol})")
    assert eo <= tol and es <= tol


def test_prologue_full_size_every_pair_against_the_fp32_path(g):
    """Every output of gdn2_chunk_fwd_prologue at full size, against the fp32 per-token kernel
    given the activations written out in torch (fp32): q / max(|q|, eps), k likewise,
    -softplus(a), sigmoid(b), sigmoid(w)."""
    wl = W.WORKLOADS[PREFILL]
    d = W.prefill_inputs(wl, "cuda")
    T_all = int(sum(d["lengths"]))
    gen = torch.Generator(device="cuda").manual_seed(wl.seed + 17)
    rn = lambda *shp: torch.randn(*shp, generator=gen, device="cuda").to(wl.dtype)
    raw = dict(q=rn(T_all, wl.h_qk, wl.dk), k=rn(T_all, wl.h_qk, wl.dk), a=rn(T_all, wl.h_v, wl.dk),
               b=rn(T_all, wl.h_v, wl.dk), w=rn(T_all, wl.h_v, wl.dv))
    o, st = g.gdn2_chunk_fwd(raw["q"], raw["k"], d["v"], raw["a"], raw["b"], raw["w"], S0=d["S0"],
                             n_seq=d["n_seq"], prologue=True)
    unit = lambda x: x / x.norm(dim=-1, keepdim=True).clamp_min(1e-12)
    act = dict(q=unit(raw["q"].float()), k=unit(raw["k"].float()), v=d["v"].float(),
               log_alpha=-torch.nn.functional.softplus(raw["a"].float()), b=torch.sigmoid(raw["b"].float()),
               w=torch.sigmoid(raw["w"].float()))
    o32, st32 = g.gdn2_chunk_fwd(*(act[key] for key in ("q", "k", "v", "log_alpha", "b", "w")), S0=d["S0"],
                                 n_seq=d["n_seq"])
    torch.cuda.synchronize()
    eo = rel_err(o, o32.double().cpu().numpy())
    es = rel_err(st, st32.double().cpu().numpy())
    print(f"prologue full size, every pair against the fp32 path: o err {eo:.3e}, S_T err {es:.3e}")
    assert eo <= TOL[torch.bfloat16] and es <= TOL[torch.bfloat16], (eo, es)


def test_serving_decode_full_size_every_state_against_the_prefill(g):
    """gdn2_decode_multi on all 256 x 32 states of the serving workload (4 tokens, states at
    seeded-random slots of a 512-state pool) equals, for every state, the fp32 prefill of the
    same 4 tokens started from that state."""
    wl = W.WORKLOADS[DECODE]
    N, n_tok = wl.n_seq, 4
    pool = torch.zeros((2 * N, wl.h_v, wl.dk, wl.dv), dtype=torch.float32, device="cuda")
    perm = torch.randperm(2 * N, generator=torch.Generator().manual_seed(wl.seed))[:N]
    S_init = W.decode_state(wl, "cuda")
    pool[perm.to("cuda")] = S_init
    slots = perm.to(torch.int32).to("cuda")
    t_ = W.token_inputs(N * n_tok, wl.h_qk, wl.h_v, wl.dk, wl.dv, wl.dtype, "cuda", wl.seed * 7919)
    x = {key: t.view(N, n_tok, *t.shape[1:]) for key, t in t_.items()}
    o, _ = g.gdn2_decode_multi(*(x[key] for key in ("q", "k", "v", "log_alpha", "b", "w")), pool, slots=slots)
    f = {key: t_[key].float() for key in ("q", "k", "v", "log_alpha", "b", "w")}
    o_pre, S_pre = g.gdn2_chunk_fwd(*(f[key] for key in ("q", "k", "v", "log_alpha", "b", "w")), S0=S_init,
                                    n_seq=N)
    torch.cuda.synchronize()
    eo = rel_err(o.reshape(N * n_tok, wl.h_v, wl.dv), o_pre.double().cpu().numpy())
    es = rel_err(pool[perm.to("cuda")], S_pre.double().cpu().numpy())
    print(f"serving decode full size, every state against the prefill: o err {eo:.3e}, S err {es:.3e}")
    assert eo <= TOL[torch.float32] and es <= TOL[torch.float32], (eo, es)


def test_backward_full_size_directional_derivatives(g):
    """The gradients of the full-size backward over every (sequence, head) pair at once: o is
    linear in S0, in v, in w and in q, so for a random direction delta the central difference
    [L(x + delta) - L(x - delta)] / 2 of L = sum(o * dO) equals <dL/dx, delta> exactly (up to
    rounding), whatever delta's size; for k, b and log_alpha, extrapolated central differences
    at small steps. L is taken with the fp32 forward kernel on the same input values."""
    wl = W.WORKLOADS[PREFILL]
    d = W.prefill_inputs(wl, "cuda")
    names = ("q", "k", "v", "log_alpha", "b", "w")
    S0 = W.state_input(wl.n_seq, wl.h_v, wl.dk, wl.dv, 0.05, "cuda", seed=wl.seed + 5)
    gen = torch.Generator(device="cuda").manual_seed(wl.seed + 29)
    dO = torch.randn(d["v"].shape, generator=gen, device="cuda")
    dq, dk, dv, dla, db, dw, dS0 = g.gdn2_chunk_bwd(*(d[k_] for k_ in names), dO, S0=S0, n_seq=wl.n_seq)
    f32 = {k_: d[k_].float() for k_ in names}

    def loss(**over):
        x = dict(f32, **{k_: v_ for k_, v_ in over.items() if k_ != "S0"})
        o, _ = g.gdn2_chunk_fwd(*(x[k_] for k_ in names), S0=over.get("S0", S0), n_seq=wl.n_seq, want_state=False)
        return float((o.double() * dO.double()).sum())

    checks = []
    for name, grad, base in (("S0", dS0, S0), ("v", dv, f32["v"]), ("q", dq, f32["q"]), ("w", dw, f32["w"])):
        delta = torch.randn(base.shape, generator=gen, device="cuda") * base.abs().mean()
        fd = (loss(**{name: base + delta}) - loss(**{name: base - delta})) / 2.0
        an = float((grad.double() * delta.double()).sum())
        checks.append((name, fd, an, abs(fd - an) / abs(an)))
    # k, b and log_alpha enter non-linearly: central differences at steps h and 2h, combined
    # (Richardson) so that the h^2 term cancels, leave O(h^4)
    for name, grad, base, h in (("k", dk, f32["k"], 1e-2), ("b", db, f32["b"], 1e-2),
                                ("log_alpha", dla, f32["log_alpha"], 1e-2)):
        delta = torch.randn(base.shape, generator=gen, device="cuda") * base.abs().mean()
        cd = lambda s_: (loss(**{name: base + s_ * delta}) - loss(**{name: base - s_ * delta})) / (2.0 * s_)
        fd = (4.0 * cd(h) - cd(2.0 * h)) / 3.0
        an = float((grad.double() * delta.double()).sum())
        checks.append((name, fd, an, abs(fd - an) / abs(an)))
    for name, fd, an, rel in checks:
        print(f"backward full size, directional {name}: difference {fd:.6e}, gradient {an:.6e}, rel {rel:.2e}")
    # the linear ones to rounding; the others to the extrapolation's remainder
    assert all(rel <= (1e-4 if name in ("S0", "v", "q", "w") else 2e-3) for name, *_, rel in checks), checks
