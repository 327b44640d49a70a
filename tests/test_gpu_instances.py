"""Every compiled kernel instance under a GPU parity test.

The decode kernels are instantiated per key width and value width (64, 128), input element
type (fp32, bf16), output element type (fp32, bf16) and with or without the fused
pre-processing; one token without per-token states runs the single-token kernel, more tokens
the persistent multi-token one. The prefill runs the tensor-core kernel for bf16 inputs with
dk = dv = 128 (fp32 or bf16 output, raw or pre-processed inputs) and the fp32 recurrent
kernel otherwise. Each case here is small, includes an inactive sequence (decode) or an empty
one (prefill), and is compared element by element with the oracle (fp64) through the C ABI.
A bf16 output may carry one extra rounding: |o - o_ref| <= 2^-8 |o_ref| + tol rms(o_ref).
"""
import itertools

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


def _out_err(o, o_ref, out_dtype) -> float:
    """rel_err, allowing one bf16 rounding of each element for a bf16 output."""
    if out_dtype == torch.float32:
        return rel_err(o, o_ref)
    got = o.detach().double().cpu().numpy()
    ref = np.asarray(o_ref, dtype=np.float64)
    assert got.shape == ref.shape and np.isfinite(got).all()
    rms = float(np.sqrt(np.mean(ref * ref)))
    return float((np.abs(got - ref) - 2.0 ** -8 * np.abs(ref)).max() / rms)


def _raw(T, h_qk, h_v, dk, dv, dtype, seed):
    """Raw projections for the fused pre-processing: q, k away from unit length,
    pre-activations ~ N(0, 1)."""
    gen = torch.Generator(device="cuda").manual_seed(seed)
    n = lambda *s: torch.randn(*s, generator=gen, device="cuda")
    return dict(q=(3.0 * n(T, h_qk, dk)).to(dtype), k=(0.5 * n(T, h_qk, dk)).to(dtype),
                v=n(T, h_v, dv).to(dtype), log_alpha=n(T, h_v, dk).to(dtype), b=n(T, h_v, dk).to(dtype),
                w=n(T, h_v, dv).to(dtype))


def _oracle(d, pro, S0, cu_seqlens=None, n_seq=None):
    """The oracle on d's tokens (prologue_ref first when ``pro``; the recurrence then takes
    the activated values at fp32, as the kernels compute them)."""
    cpu = {k_: t.detach().cpu() for k_, t in d.items()}
    if pro:
        q, k, la, b, w = oracle.prologue_ref(cpu["q"], cpu["k"], cpu["log_alpha"], cpu["b"], cpu["w"])
        f32 = lambda x: np.asarray(x, dtype=np.float32)
        return oracle.fwd_ref(f32(q), f32(k), cpu["v"].float().numpy(), f32(la), f32(b), f32(w),
                              S0=S0, cu_seqlens=cu_seqlens, n_seq=n_seq, bf16=False)
    return oracle.fwd_ref(cpu["q"], cpu["k"], cpu["v"], cpu["log_alpha"], cpu["b"], cpu["w"], S0=S0,
                          cu_seqlens=cu_seqlens, n_seq=n_seq)


F32, BF16 = torch.float32, torch.bfloat16
DECODE_CASES = list(itertools.product([64, 128], [64, 128], [F32, BF16], [F32, BF16], [False, True], [1, 3]))


@pytest.mark.parametrize("dk,dv,in_dt,out_dt,pro,n_tok", DECODE_CASES,
                         ids=[f"dk{a}-dv{b}-{str(c)[6:]}-o{str(e)[6:]}-{'pro' if p else 'plain'}-t{n}"
                              for a, b, c, e, p, n in DECODE_CASES])
def test_decode_instance(g, dk, dv, in_dt, out_dt, pro, n_tok):
    N, h_qk, h_v, n_slots = 3, 1, 2, 5
    slots = [3, -1, 0]  # the second sequence is inactive
    seed = 7000 + dk + 3 * dv + 11 * n_tok + (1 if in_dt == BF16 else 0) + (2 if out_dt == BF16 else 0) + 5 * pro
    if pro:
        d = _raw(N * n_tok, h_qk, h_v, dk, dv, in_dt, seed)
    else:
        d = W.token_inputs(N * n_tok, h_qk, h_v, dk, dv, in_dt, "cuda", seed=seed)
    dm = {k_: t.view(N, n_tok, *t.shape[1:]) for k_, t in d.items()}
    pool = W.state_input(n_slots, h_v, dk, dv, 0.05, "cuda", seed=seed)
    before = pool.clone()
    o = torch.full((N, n_tok, h_v, dv), 123.0, dtype=out_dt, device="cuda")
    slots_t = torch.tensor(slots, dtype=torch.int32, device="cuda")
    o, _ = g.gdn2_decode_multi(dm["q"], dm["k"], dm["v"], dm["log_alpha"], dm["b"], dm["w"], pool,
                               slots=slots_t, o=o, prologue=pro)
    torch.cuda.synchronize()
    assert torch.all(o[1] == 123.0), "the inactive sequence's rows of o were written"
    tol = TOL[F32]  # the decode kernels compute in fp32
    o_got, o_ref, s_got, s_ref = [], [], [], []
    for n, s in enumerate(slots):
        if s < 0:
            continue
        dn = {k_: t[n] for k_, t in dm.items()}
        ro, rs = _oracle(dn, pro, before[s][None].cpu(), n_seq=1)
        o_got.append(o[n])
        o_ref.append(ro)
        s_got.append(pool[s])
        s_ref.append(rs[0])
    eo = _out_err(torch.stack(o_got), np.stack(o_ref), out_dt)
    es = rel_err(torch.stack(s_got), np.stack(s_ref))
    assert eo <= tol and es <= tol, (eo, es)
    untouched = [s for s in range(n_slots) if s not in slots]
    assert torch.equal(pool[untouched], before[untouched])


CHUNK_CASES = ([(F32, dk, dv, out, False) for dk in (64, 128) for dv in (64, 128) for out in (F32, BF16)]
               + [(BF16, dk, dv, out, False) for dk, dv in ((64, 64), (64, 128), (128, 64)) for out in (F32, BF16)]
               + [(BF16, 128, 128, out, pro) for out in (F32, BF16) for pro in (False, True)])


@pytest.mark.parametrize("in_dt,dk,dv,out_dt,pro", CHUNK_CASES,
                         ids=[f"{str(a)[6:]}-dk{b}-dv{c}-o{str(e)[6:]}-{'pro' if p else 'plain'}"
                              for a, b, c, e, p in CHUNK_CASES])
def test_prefill_instance(g, in_dt, dk, dv, out_dt, pro):
    lens = [70, 0, 131]
    T, h_qk, h_v = sum(lens), 1, 2
    seed = 7500 + dk + 3 * dv + (1 if in_dt == BF16 else 0) + (2 if out_dt == BF16 else 0) + 5 * pro
    if pro:
        d = _raw(T, h_qk, h_v, dk, dv, in_dt, seed)
    else:
        d = W.token_inputs(T, h_qk, h_v, dk, dv, in_dt, "cuda", seed=seed)
    S0 = W.state_input(len(lens), h_v, dk, dv, 0.05, "cuda", seed=seed)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device="cuda")
    o, st = g.gdn2_chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], S0=S0, cu_seqlens=cu,
                             out_dtype=out_dt, prologue=pro)
    torch.cuda.synchronize()
    assert o.dtype == out_dt
    o_ref, st_ref = _oracle(d, pro, S0.cpu(), cu_seqlens=cu.cpu())
    tol = TOL[in_dt]
    eo, es = _out_err(o, o_ref, out_dt), rel_err(st, st_ref)
    assert eo <= tol and es <= tol, (eo, es)
    torch.testing.assert_close(st[1], S0[1], rtol=0, atol=0)  # the empty sequence
