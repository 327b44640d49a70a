"""The benchmark's roofline accounting, checked on the CPU against hand-computed counts.

The algorithmic bytes (and, for the backward, flops) per launch are the numerators of every
roofline fraction bench.py reports; a slip there would inflate or deflate a fraction
silently, so each formula is pinned to its count written out by hand here.
"""
import importlib.util
import os

import pytest

from gated_delta_rule_160_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_prefill_bytes_headline(bench):
    wl = W.WORKLOADS["prefill_b8_h16_t4096"]
    tokens = 8 * 4096
    # the algorithmic count: per token, q, k bf16 on 16 query/key heads; v, w, b bf16, log_alpha
    # fp32 and o at the input dtype (bf16) on 16 value heads -- 2048 B per token and head;
    # plus S_T written once (S0 is zero and not read)
    per_token = 16 * (128 * 2 + 128 * 2) + 16 * (128 * 2 + 128 * 2 + 128 * 2 + 128 * 4 + 128 * 2)
    assert per_token == 16 * 2048
    expect = tokens * per_token + 8 * 16 * 128 * 128 * 4
    assert bench.prefill_bytes(wl, [4096] * 8) == expect == 1082130432
    # the same with o counted as the fp32 the kernel writes: 2304 B per token and head
    per_token32 = per_token + 16 * 128 * 2
    assert bench.prefill_bytes(wl, [4096] * 8, 4) == tokens * per_token32 + 8 * 16 * 128 * 128 * 4 == 1216348160


def test_prefill_bytes_grouped_counts_qk_once_per_query_key_head(bench):
    wl = W.WORKLOADS["grouped_b2_qk16_v32_t32768"]
    tokens = 2 * 32768
    per_token = 16 * 512 + 32 * 1536           # q, k per query/key head; the rest per value head
    state = 2 * 32 * 128 * 128 * 4
    assert bench.prefill_bytes(wl, [32768] * 2) == tokens * per_token + 2 * state  # S0 read, S_T written
    # 1792 B per token and value head (q and k shared by two value heads)
    assert per_token == 32 * 1792


def test_hbm_roofline_fraction(bench):
    r = bench.hbm_roofline(1_000_000_000, 1_100_000_000, 0.5, 6500.0, "measured", None)
    assert r["achieved"] == pytest.approx(2000.0) and r["frac"] == pytest.approx(2000.0 / 6500.0)
    assert r["fp32_o"]["achieved"] == pytest.approx(2200.0)


def test_prologue_bytes(bench):
    wl = W.WORKLOADS["prefill_b8_h16_t4096"]
    # raw q, k (bf16) per query/key head; v, w, b and the decay pre-activation (bf16) and o
    # (fp32) per value head
    per_token = 16 * 512 + 16 * (256 * 4 + 512)
    assert bench.prologue_bytes(wl, [4096] * 8) == 8 * 4096 * per_token + 8 * 16 * 65536


def test_backward_bytes_and_flops(bench):
    wl = W.WORKLOADS["prefill_b8_h16_t4096"]
    tokens = 8 * 4096
    reads = 16 * 512 + 16 * (256 * 3 + 512 + 512)  # inputs, and dO (fp32)
    writes = 16 * 2 * 512 + 16 * (2 * 512 + 2 * 512)  # dq, dk; dv, dw, dlog_alpha, db (all fp32)
    assert bench.backward_bytes(wl, [4096] * 8) == tokens * (reads + writes) + 2 * 8 * 16 * 65536
    # 7 flops per state element to regenerate S_prev, 21 for the adjoint
    assert bench.backward_flops(wl, [4096] * 8) == tokens * 16 * 128 * 128 * 28 == 240518168576


def test_decode_and_serving_bytes(bench):
    wl = W.WORKLOADS["decode_256seq_h32"]
    io_token = 32 * 512 + 32 * 1792  # one token of one sequence, all 32 heads
    state = 256 * 32 * 65536
    assert bench.decode_bytes(wl) == 256 * io_token + 2 * state
    assert bench.serving_bytes(wl, 4) == 256 * 4 * io_token + 2 * state


def test_fp32_alu_peak(bench):
    assert bench.FP32_SIMT_TFLOPS == pytest.approx(148 * 128 * 2 * 1.965e9 / 1e12)


def test_recorded_traffic_follows_the_kernel_source(bench, monkeypatch, tmp_path):
    """A capture's traffic counts only while the kernel source still has the sha256 prefix
    recorded beside it in profiles/traffic.json; every record names its source and summary."""
    import hashlib
    import json
    rec = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    for key, r in rec.items():
        assert os.path.exists(os.path.join(ROOT, r["source"])), key
        assert os.path.exists(os.path.join(ROOT, r["summary"])), key
        assert len(r["source_sha256_16"]) == 16, key
        assert r["dram_bytes_per_launch"] is None or int(r["dram_bytes_per_launch"]) > 0, key
        sha = hashlib.sha256(open(os.path.join(ROOT, r["source"]), "rb").read()).hexdigest()[:16]
        got = bench.recorded_traffic(key)
        assert got == (r["dram_bytes_per_launch"] if sha == r["source_sha256_16"] else None), key
    # a mismatching prefix, or an unknown key, reads as unknown
    fake_root = tmp_path
    (fake_root / "profiles").mkdir()
    src = "gated_delta_rule_160_b200/csrc/chunk_tc.cu"
    (fake_root / "gated_delta_rule_160_b200" / "csrc").mkdir(parents=True)
    (fake_root / src).write_bytes(open(os.path.join(ROOT, src), "rb").read())
    (fake_root / "profiles" / "traffic.json").write_text(json.dumps(
        {"k": {"source": src, "source_sha256_16": "0" * 16, "dram_bytes_per_launch": 123}}))
    monkeypatch.setattr(bench, "ROOT", str(fake_root))
    assert bench.recorded_traffic("k") is None
    assert bench.recorded_traffic("missing") is None
