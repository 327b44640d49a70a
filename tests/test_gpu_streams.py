"""Calls on different CUDA streams share no device state: a packed-batch prefill (with its
own workspace), a serving-decode step and a second prefill, queued on two streams so that
they can run at the same time, give bit for bit the results of the same calls made one
after another on one stream. (Only gdn2_chunk_fwd_noalloc shares a scratch array between
calls, and it is not used here.)"""
import numpy as np
import pytest
import torch

from gated_delta_rule_160_b200 import workloads as W

pytestmark = pytest.mark.gpu

NAMES = ("q", "k", "v", "log_alpha", "b", "w")


@pytest.fixture(scope="module")
def g():
    import gated_delta_rule_160_b200 as g
    g.load_library()
    assert torch.cuda.is_available()
    return g


def _cases():
    lens = [300, 70, 513, 1, 190]
    T = sum(lens)
    a = W.token_inputs(T, 2, 4, 128, 128, torch.bfloat16, "cuda", seed=81)
    a["S0"] = W.state_input(len(lens), 4, 128, 128, 0.05, "cuda", seed=81)
    a["cu"] = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device="cuda")
    b = W.token_inputs(4 * 640, 2, 2, 128, 128, torch.bfloat16, "cuda", seed=82)
    N, n_tok = 48, 4
    c = W.token_inputs(N * n_tok, 4, 4, 128, 128, torch.bfloat16, "cuda", seed=83)
    c = {k_: t.view(N, n_tok, *t.shape[1:]) for k_, t in c.items()}
    pool = W.state_input(2 * N, 4, 128, 128, 0.05, "cuda", seed=83)
    slots = torch.randperm(2 * N, generator=torch.Generator().manual_seed(83))[:N].to(torch.int32).to("cuda")
    return a, b, c, pool, slots


def _run(g, a, b, c, pool, slots, s1, s2):
    o1, st1 = g.gdn2_chunk_fwd(*(a[k_] for k_ in NAMES), S0=a["S0"], cu_seqlens=a["cu"], stream=s1)
    om, _ = g.gdn2_decode_multi(*(c[k_] for k_ in NAMES), pool, slots=slots, stream=s2)
    o2, st2 = g.gdn2_chunk_fwd(*(b[k_] for k_ in NAMES), n_seq=4, stream=s2)
    torch.cuda.synchronize()
    return o1, st1, om, o2, st2


def test_concurrent_streams_match_serial_calls(g):
    a, b, c, pool, slots = _cases()
    pool0 = pool.clone()
    one = torch.cuda.Stream()
    serial = _run(g, a, b, c, pool, slots, one, one)
    pool_serial = pool.clone()
    pool.copy_(pool0)
    torch.cuda.synchronize()
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    concurrent = _run(g, a, b, c, pool, slots, s1, s2)
    for x, y in zip(serial, concurrent):
        assert torch.equal(x, y)
    assert torch.equal(pool, pool_serial)
    assert g.gdn2_device_status() == 0
