"""Fused pre-processing (gdn2_chunk_fwd_prologue, gdn2_decode_multi_prologue): raw projections
in, the recurrence on L2-normalised q, k, log_alpha = -softplus(a), sigmoid b, w. Checked
through the C ABI against the oracle's prologue (fp64) followed by the oracle."""
import numpy as np
import pytest
import torch

import oracle
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


def _raw(T, h_qk, h_v, seed, dtype=torch.bfloat16):
    """Raw projections: q, k scaled away from unit norm, pre-activations ~ N(0, 1)."""
    gen = torch.Generator(device="cuda").manual_seed(seed)
    n = lambda *s: torch.randn(*s, generator=gen, device="cuda")
    return dict(q=(3.0 * n(T, h_qk, D)).to(dtype), k=(0.5 * n(T, h_qk, D)).to(dtype), v=n(T, h_v, D).to(dtype),
                a=n(T, h_v, D).to(dtype), b=n(T, h_v, D).to(dtype), w=n(T, h_v, D).to(dtype))


def _oracle(d, S0, cu):
    """prologue_ref, then the oracle on the activated inputs (fp32 element type)."""
    q, k, la, b, w = oracle.prologue_ref(d["q"], d["k"], d["a"], d["b"], d["w"])
    f32 = lambda x: np.asarray(x, dtype=np.float32)
    return oracle.fwd_ref(f32(q), f32(k), d["v"].float().cpu().numpy(), f32(la), f32(b), f32(w),
                          S0=None if S0 is None else S0.cpu(), cu_seqlens=cu, bf16=False)


def test_chunk_prologue_matches_oracle(g):
    lens = [200, 64, 131, 0, 65]
    T = sum(lens)
    d = _raw(T, 2, 4, seed=41)
    S0 = W.state_input(len(lens), 4, D, D, 0.05, "cuda", seed=41)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device="cuda")
    o, st = g.gdn2_chunk_fwd(d["q"], d["k"], d["v"], d["a"], d["b"], d["w"], S0=S0, cu_seqlens=cu, prologue=True)
    torch.cuda.synchronize()
    o_ref, st_ref = _oracle(d, S0, cu.cpu())
    eo, es = rel_err(o, o_ref), rel_err(st, st_ref)
    tol = TOL[torch.bfloat16]
    print(f"chunk prologue: o err {eo:.3e}, S_T err {es:.3e} (tol {tol})")
    assert eo <= tol and es <= tol
    torch.testing.assert_close(st[3], S0[3], rtol=0, atol=0)  # the empty sequence


def test_chunk_prologue_decay_beyond_range_is_recomputed(g):
    """A decay pre-activation of +6 on eight channels of one (sequence, head) gives
    log_alpha = -softplus(6) ~ -6 per token, ~380 nats across a chunk: past the tensor-core
    kernel's range, so that pair is recomputed token by token in fp32 (the pre-processing
    included) and matches the oracle to the fp32 bound; the rest keep the bf16 bound."""
    lens = [200, 64, 131]
    T = sum(lens)
    d = _raw(T, 2, 4, seed=44)
    a = d["a"].clone()
    a[264:395, 3, 40:48] = 6.0  # sequence 2, value head 3
    d["a"] = a
    S0 = W.state_input(len(lens), 4, D, D, 0.05, "cuda", seed=44)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device="cuda")
    g.gdn2_device_status()
    o, st = g.gdn2_chunk_fwd(d["q"], d["k"], d["v"], d["a"], d["b"], d["w"], S0=S0, cu_seqlens=cu, prologue=True)
    torch.cuda.synchronize()
    assert g.gdn2_device_status() & g.GDN2_DEVICE_DECAY_RANGE
    o_ref, st_ref = _oracle(d, S0, cu.cpu())
    eo, es = rel_err(o[264:, 3], o_ref[264:, 3]), rel_err(st[2, 3], st_ref[2, 3])
    print(f"recomputed pair: o err {eo:.3e}, S_T err {es:.3e} (tol {TOL[torch.float32]})")
    assert eo <= TOL[torch.float32] and es <= TOL[torch.float32]
    assert rel_err(o, o_ref) <= TOL[torch.bfloat16] and rel_err(st, st_ref) <= TOL[torch.bfloat16]


def test_decode_prologue_matches_oracle(g):
    N, n_tok, H, n_slots = 4, 3, 2, 6
    slots = [5, 0, 3, 1]
    d = _raw(N * n_tok, H, H, seed=42)
    pool = W.state_input(n_slots, H, D, D, 0.05, "cuda", seed=42)
    before = pool.clone()
    dm = {k_: t.view(N, n_tok, *t.shape[1:]) for k_, t in d.items()}
    slots_t = torch.tensor(slots, dtype=torch.int32, device="cuda")
    o, _ = g.gdn2_decode_multi(dm["q"], dm["k"], dm["v"], dm["a"], dm["b"], dm["w"], pool, slots=slots_t,
                               prologue=True)
    torch.cuda.synchronize()
    S0 = torch.stack([before[s] for s in slots])
    o_ref, st_ref = _oracle(d, S0, np.arange(0, N * n_tok + 1, n_tok, dtype=np.int32))
    eo = rel_err(o.reshape(N * n_tok, H, D), o_ref)
    es = rel_err(torch.stack([pool[s] for s in slots]), st_ref)
    tol = TOL[torch.float32]  # fp32 arithmetic in the decode kernel
    print(f"decode prologue: o err {eo:.3e}, S err {es:.3e} (tol {tol})")
    assert eo <= tol and es <= tol


def test_prologue_rejects_what_the_tensor_core_kernel_does_not_take(g):
    d = _raw(70, 1, 1, seed=43, dtype=torch.float32)
    with pytest.raises(g.Gdn2Error) as e:
        g.gdn2_chunk_fwd(d["q"], d["k"], d["v"], d["a"], d["b"], d["w"], n_seq=1, prologue=True)
    assert e.value.status == 2  # GDN2_ERR_UNSUPPORTED
