"""gdn2_chunk_fwd_noalloc: the prefill entry point for callers that cannot allocate device
memory (it keeps the packed-batch scratch in a static array inside the library). Called
through the C ABI, it must give what gdn2_chunk_fwd gives with a caller-allocated
workspace, within the parity tolerance, on two calls in a row with different batches (the
shared scratch keeps the previous call's contents). Nothing here depends on what ran
before: the tests pass alone in a fresh process and after any others. The file name only
places them last in a full run, so that a run stopping at its first failure has already
run every other test."""
import ctypes

import numpy as np
import pytest
import torch

from gated_delta_rule_160_b200 import workloads as W
from tests.parity import TOL, rel_err

pytestmark = pytest.mark.gpu


def _batch(lens, seed):
    T = int(sum(lens))
    d = W.token_inputs(T, 2, 4, 128, 128, torch.bfloat16, "cuda", seed=seed)
    d["S0"] = W.state_input(len(lens), 4, 128, 128, 0.05, "cuda", seed=seed)
    d["cu"] = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device="cuda")
    return d


def test_noalloc_matches_workspace_entry_point():
    import gated_delta_rule_160_b200 as g
    lib = g.load_library()
    P = lambda t: ctypes.c_void_p(t.data_ptr()) if t is not None else None
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for lens, seed in [([300, 0, 64, 129, 1, 70], 5), ([65, 200, 3], 6)]:
        d = _batch(lens, seed)
        o_ref, st_ref = g.gdn2_chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], S0=d["S0"],
                                         cu_seqlens=d["cu"])
        o = torch.full_like(o_ref, float("nan"))
        st = torch.full_like(st_ref, float("nan"))
        shape = g.make_shape(d["q"], d["v"], len(lens), torch.float32)
        status = lib.gdn2_chunk_fwd_noalloc(ctypes.byref(shape), P(d["q"]), P(d["k"]), P(d["v"]),
                                            P(d["log_alpha"]), P(d["b"]), P(d["w"]), P(d["S0"]), P(d["cu"]),
                                            P(o), P(st), stream)
        assert status == 0, lib.gdn2_last_error_string()
        torch.cuda.synchronize()
        tol = TOL[torch.bfloat16]
        assert rel_err(o, o_ref.double().cpu().numpy()) <= tol
        assert rel_err(st, st_ref.double().cpu().numpy()) <= tol


def test_noalloc_rejects_batches_beyond_its_scratch():
    import gated_delta_rule_160_b200 as g
    lib = g.load_library()
    lens = [1] * 16385
    d = _batch([1, 1], 7)
    cu = torch.arange(len(lens) + 1, dtype=torch.int32, device="cuda")
    shape = g.Shape(len(lens), len(lens), 2, 4, 128, 128, g.GDN2_BF16, g.GDN2_F32)
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    status = lib.gdn2_chunk_fwd_noalloc(ctypes.byref(shape), P(d["q"]), P(d["k"]), P(d["v"]), P(d["log_alpha"]),
                                        P(d["b"]), P(d["w"]), None, P(cu), P(d["v"]), None, None)
    assert status == 1  # GDN2_ERR_INVALID_ARG, nothing queued
    assert b"16384" in lib.gdn2_last_error_string()
