"""Host-side checks of the C ABI (no GPU needed): both libraries load, every function the
headers in include/ declare is exported, and argument checks that run before any device
work reject bad calls with the documented status."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared(header):
    text = open(os.path.join(ROOT, "include", header)).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gdn2_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from gated_delta_rule_160_b200 import build
    build.build()
    import gated_delta_rule_160_b200 as g
    return g.load_library()


def test_product_library_exports_every_declared_function(lib):
    names = _declared("gdn2.h")
    assert {"gdn2_chunk_fwd", "gdn2_decode_step", "gdn2_chunk_fwd_workspace_size"} <= set(names)
    for n in names:
        assert hasattr(lib, n), f"libgdn2.so does not export {n}"


def test_oracle_library_exports_every_declared_function(oracle_mod):
    lib = oracle_mod.load()
    for n in _declared("gdn2_ref.h"):
        assert hasattr(lib, n), f"libgdn2_ref.so does not export {n}"


def test_libraries_share_no_symbols(lib, oracle_mod):
    """The oracle and the CUDA library are separate: neither exports the other's entry points."""
    assert not hasattr(lib, "gdn2_fwd_ref")
    assert not hasattr(oracle_mod.load(), "gdn2_chunk_fwd")


def _shape(g, **kw):
    d = dict(n_seq=1, T_total=64, h_qk=1, h_v=1, dk=64, dv=64, dtype=g.GDN2_BF16, o_dtype=g.GDN2_F32)
    d.update(kw)
    return g.Shape(**d)


def _call_chunk(g, lib, shape, ptr=None):
    p = ctypes.c_void_p(ptr) if ptr else None
    return lib.gdn2_chunk_fwd(ctypes.byref(shape) if shape is not None else None,
                              p, p, p, p, p, p, None, None, p, None, None, 0, None)


def test_rejects_before_device_work(lib):
    import gated_delta_rule_160_b200 as g
    assert lib.gdn2_chunk_fwd(None, *([None] * 10), None, 0, None) == 1
    assert b"shape is NULL" in lib.gdn2_last_error_string()
    assert _call_chunk(g, lib, _shape(g, dk=96)) == 2
    assert b"dk = 96" in lib.gdn2_last_error_string()
    assert _call_chunk(g, lib, _shape(g, h_qk=3, h_v=4)) == 1
    assert _call_chunk(g, lib, _shape(g, n_seq=0)) == 1
    assert _call_chunk(g, lib, _shape(g, n_seq=65535, h_qk=65535, h_v=65535)) == 2
    assert b"pairs above 2^31 - 1" in lib.gdn2_last_error_string()
    assert _call_chunk(g, lib, _shape(g, dtype=7)) == 1
    assert _call_chunk(g, lib, _shape(g, o_dtype=5)) == 1
    assert _call_chunk(g, lib, _shape(g)) == 1  # NULL tensors with T_total > 0
    assert b"q is NULL" in lib.gdn2_last_error_string()
    assert _call_chunk(g, lib, _shape(g), ptr=0x1008) == 1  # misaligned
    assert b"16-byte aligned" in lib.gdn2_last_error_string()
    # decode: exactly one token per sequence
    sh = _shape(g, n_seq=4, T_total=5)
    assert lib.gdn2_decode_step(ctypes.byref(sh), *([None] * 9)) == 1
    assert b"one token per sequence" in lib.gdn2_last_error_string()


def test_workspace_size(lib):
    import gated_delta_rule_160_b200 as g
    sh = _shape(g, n_seq=64)
    assert lib.gdn2_chunk_fwd_workspace_size(ctypes.byref(sh), 0) == 0
    ws = lib.gdn2_chunk_fwd_workspace_size(ctypes.byref(sh), 1)
    assert ws >= 64 * 4 and ws % 256 == 0


def test_version(lib):
    assert lib.gdn2_version() >= 100


def test_decode_multi_rejects_before_device_work(lib):
    import gated_delta_rule_160_b200 as g
    nul = [None] * 8

    def call(sh, n_tok, n_slots, slots=None):
        return lib.gdn2_decode_multi(ctypes.byref(sh), n_tok, slots, *nul[:7], n_slots, None, None, None)

    sh = _shape(g, n_seq=4, T_total=12)
    assert call(sh, 0, 4) == 1 and b"n_tok = 0" in lib.gdn2_last_error_string()
    assert call(sh, g.GDN2_DECODE_MAX_TOKENS + 1, 4) == 1
    assert call(sh, 2, 4) == 1 and b"not n_seq * n_tok" in lib.gdn2_last_error_string()
    assert call(sh, 3, 3) == 1 and b"n_slots = 3 too small" in lib.gdn2_last_error_string()
    assert call(sh, 3, 4) == 1 and b"q is NULL" in lib.gdn2_last_error_string()
    # the pool's state rows (n_slots * h_v * dk) are TMA coordinates: int32
    wide = _shape(g, n_seq=4, T_total=12, h_qk=32, h_v=32, dk=128, dv=128)
    assert call(wide, 3, 1 << 20) == 2 and b"state rows" in lib.gdn2_last_error_string()


def test_chunk_bwd_rejects_before_device_work(lib):
    import gated_delta_rule_160_b200 as g

    def call(sh, ptr=None, ws=None, ws_bytes=0):
        p = ctypes.c_void_p(ptr) if ptr else None
        return lib.gdn2_chunk_bwd(ctypes.byref(sh) if sh is not None else None, *([p] * 6), None, None, p, None,
                                  *([p] * 6), None, ws, ws_bytes, None)

    assert call(None) == 1 and b"shape is NULL" in lib.gdn2_last_error_string()
    assert call(_shape(g, dk=96)) == 2 and b"dk = 96" in lib.gdn2_last_error_string()
    assert call(_shape(g, h_qk=2, h_v=3)) == 1
    assert call(_shape(g)) == 1 and b"q is NULL" in lib.gdn2_last_error_string()
    assert call(_shape(g), ptr=0x1008) == 1 and b"16-byte aligned" in lib.gdn2_last_error_string()


def test_chunk_bwd_workspace_size(lib):
    """Checkpoints every 8 tokens (slots n + t0 / 8 + sub-chunk, at most ceil(T / 8) + N) and a
    7-state scratch per (sequence, value head), fp32 states, rounded up to 256 bytes."""
    import gated_delta_rule_160_b200 as g
    assert lib.gdn2_chunk_bwd_workspace_size(None) == 0
    sh = _shape(g, n_seq=2, T_total=100, h_qk=1, h_v=2, dk=64, dv=64)
    state = 64 * 64 * 4
    expect = (-(-100 // 8) + 2) * 2 * state + 2 * 2 * 7 * state
    assert lib.gdn2_chunk_bwd_workspace_size(ctypes.byref(sh)) == -(-expect // 256) * 256


def test_cuda_failure_is_reported_as_cuda_error(lib):
    """On a machine without a usable GPU a call that passes the host checks fails at its
    launch: the status is GDN2_ERR_CUDA and the message carries the CUDA runtime's reason.
    (A zero-token prefill needs no tensors, so it reaches the launch.)"""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present: the launch would succeed")
    import gated_delta_rule_160_b200 as g
    sh = _shape(g, n_seq=1, T_total=0, dk=128, dv=128)
    assert lib.gdn2_chunk_fwd(ctypes.byref(sh), *([None] * 10), None, 0, None) == 3
    msg = lib.gdn2_last_error_string()
    assert msg.startswith(b"chunk kernel launch: ") and len(msg) > len(b"chunk kernel launch: ")
    # the binding raises it as Gdn2Error with the same status
    with pytest.raises(g.Gdn2Error) as e:
        g._check(3)
    assert e.value.status == 3


def test_device_status_rejects_null_flags(lib):
    assert lib.gdn2_device_status(None, None) == 1
    assert b"flags is NULL" in lib.gdn2_last_error_string()


def test_binding_rejects_host_tensors(lib):
    """The binding's argument checks run before any launch and need no GPU: host tensors are
    refused with a ValueError."""
    import torch
    import gated_delta_rule_160_b200 as g
    x = torch.zeros(4, 1, 64)
    with pytest.raises(ValueError, match="CUDA tensor"):
        g.gdn2_chunk_fwd(x, x, x, x, x, x)
    with pytest.raises(ValueError, match="CUDA tensor"):
        g.gdn2_decode_step(x, x, x, x, x, x, torch.zeros(4, 1, 64, 64))
