"""Device-side errors reach the caller through gdn2_device_status (read and clear).

- A bounded wait of the tensor-core prefill that runs out: the testing hook shortens the
  waits to 2 ms and makes the producer withhold the first loads, so no MMA and no copy is
  ever issued; every wait of the CTA gives up, the CTA releases its tensor memory and
  returns, and the status reports GDN2_DEVICE_WAIT_TIMEOUT. Nothing faults or hangs, and
  the next prefill on the same context is correct. The same for the multi-token decode,
  whose first state load is withheld.
- Malformed cu_seqlens (decreasing, or not ending at T_total): the kernels clamp every
  range, and the status reports GDN2_DEVICE_BAD_SEQLENS, for the prefill (both kernels) and
  the backward.
"""
import numpy as np
import pytest
import torch

from gated_delta_rule_160_b200 import workloads as W
from tests.parity import TOL, rel_err, oracle_on

pytestmark = pytest.mark.gpu

NAMES = ("q", "k", "v", "log_alpha", "b", "w")


@pytest.fixture(scope="module")
def g():
    import gated_delta_rule_160_b200 as g
    g.load_library()
    assert torch.cuda.is_available()
    g.gdn2_device_status()  # start from a clear word
    return g


def _inputs(lens, dtype, d=128, seed=41):
    T = int(sum(lens))
    x = W.token_inputs(T, 2, 2, d, d, dtype, "cuda", seed=seed)
    x["lengths"] = list(lens)
    x["cu"] = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device="cuda")
    return x


def test_good_calls_leave_the_status_clear(g):
    x = _inputs([70, 130], torch.bfloat16)
    g.gdn2_chunk_fwd(*(x[k] for k in NAMES), cu_seqlens=x["cu"])
    assert g.gdn2_device_status() == 0


def test_wait_timeout_is_reported_and_the_context_stays_usable(g, oracle_mod):
    lib = g.load_library()
    x = _inputs([200, 150], torch.bfloat16)
    o = torch.full((350, 2, 128), float("nan"), device="cuda")
    lib.gdn2_testing_set_wait_limit(2_000_000, 1)  # 2 ms, first loads withheld
    try:
        g.gdn2_chunk_fwd(*(x[k] for k in NAMES), cu_seqlens=x["cu"], o=o)
        st = g.gdn2_device_status()
    finally:
        lib.gdn2_testing_set_wait_limit(0, 0)
    assert st & g.GDN2_DEVICE_WAIT_TIMEOUT, st
    assert torch.isnan(o).all(), "a CTA whose waits ran out wrote output"
    # the same context runs the next prefill normally
    o2, s2 = g.gdn2_chunk_fwd(*(x[k] for k in NAMES), cu_seqlens=x["cu"])
    assert g.gdn2_device_status() == 0
    ref = oracle_on(oracle_mod, x, S0=None)
    tol = TOL[torch.bfloat16]
    got_o = np.concatenate([o2[int(x["cu"][n]):int(x["cu"][n + 1]), h].cpu().numpy()
                            for n in range(2) for h in range(2)])
    ref_o = np.concatenate([ref[(n, h)][0] for n in range(2) for h in range(2)])
    assert rel_err(got_o, ref_o) <= tol
    assert rel_err(s2, np.stack([[ref[(n, h)][1] for h in range(2)] for n in range(2)])) <= tol


def test_decode_wait_timeout_is_reported_and_the_context_stays_usable(g, oracle_mod):
    """The multi-token decode's bounded wait for an item's state: with the testing hook the
    first state load is never issued, the 2 ms wait runs out, the CTA returns before it
    touches o or the pool, and the status reports the timeout; the next decode is correct."""
    lib = g.load_library()
    N, n_tok, H, D = 3, 4, 2, 128
    x = W.token_inputs(N * n_tok, H, H, D, D, torch.bfloat16, "cuda", seed=61)
    xm = {k: t.view(N, n_tok, *t.shape[1:]) for k, t in x.items()}
    pool = W.state_input(N, H, D, D, 0.05, "cuda", seed=61)
    before = pool.clone()
    o = torch.full((N, n_tok, H, D), float("nan"), device="cuda")
    lib.gdn2_testing_set_wait_limit(2_000_000, 1)  # 2 ms, first state load withheld
    try:
        g.gdn2_decode_multi(*(xm[k] for k in NAMES), pool, o=o)
        st = g.gdn2_device_status()
    finally:
        lib.gdn2_testing_set_wait_limit(0, 0)
    assert st & g.GDN2_DEVICE_WAIT_TIMEOUT, st
    assert torch.isnan(o).all(), "a CTA whose wait ran out wrote output"
    assert torch.equal(pool, before), "a CTA whose wait ran out wrote its state"
    # the same context runs the next decode normally
    o2, _ = g.gdn2_decode_multi(*(xm[k] for k in NAMES), pool)
    assert g.gdn2_device_status() == 0
    tol = TOL[torch.float32]  # fp32 arithmetic in the decode kernel
    for n in range(N):
        ref_o, ref_s = oracle_mod.fwd_ref(*(xm[k][n].cpu() for k in NAMES), S0=before[n:n + 1].cpu(), n_seq=1)
        assert rel_err(o2[n], ref_o) <= tol and rel_err(pool[n], ref_s[0]) <= tol, n


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64)])
@pytest.mark.parametrize("cu", [[0, 100, 50, 200], [0, 120, 150]])
def test_malformed_cu_seqlens_are_flagged(g, dtype, d, cu):
    x = _inputs([100, 100], dtype, d=d)
    bad = torch.tensor(cu, dtype=torch.int32, device="cuda")
    g.gdn2_chunk_fwd(*(x[k] for k in NAMES), cu_seqlens=bad)
    assert g.gdn2_device_status() & g.GDN2_DEVICE_BAD_SEQLENS
    assert g.gdn2_device_status() == 0  # read and cleared


def test_malformed_cu_seqlens_are_flagged_by_the_backward(g):
    x = _inputs([60, 40], torch.float32, d=64)
    bad = torch.tensor([0, 70, 60], dtype=torch.int32, device="cuda")  # decreasing
    dO = torch.randn(100, 2, 64, device="cuda")
    g.gdn2_chunk_bwd(*(x[k] for k in NAMES), dO, cu_seqlens=bad)
    assert g.gdn2_device_status() & g.GDN2_DEVICE_BAD_SEQLENS
