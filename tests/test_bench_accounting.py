"""The bench's roofline numerators against the tensors the workloads actually move (CPU).

Every HBM-roofline line of ``bench.py`` divides an algorithmic byte count by a measured time;
these tests rebuild the same workloads (at small sizes, with the bench's own formulas) and
check that the formulas equal the bytes of the input and output tensors, read or written once.
They also check that the committed ncu summaries parse for the machine-read traffic field.
"""
import hashlib
import os
import re

import pytest
import torch

import bench
import kda_inputs as KI

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def nbytes(*ts):
    return sum(t.numel() * t.element_size() for t in ts if t is not None)


@pytest.mark.parametrize("lengths,H,d,dtype", [([96, 33], 4, 128, torch.bfloat16), ([50], 2, 64, torch.float32)])
def test_prefill_bytes_are_the_tensors(lengths, H, d, dtype):
    name = "prefill_8k" if dtype == torch.bfloat16 else "tiny_f32"
    inp = KI.prefill_workload(name, "cpu", lengths=lengths, heads=H)
    assert inp["q"].shape[-1] == d
    o = torch.empty_like(inp["v"])
    S_T = torch.empty_like(inp["S0"])
    moved = nbytes(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["S0"], o, S_T)
    assert bench.prefill_bytes(sum(lengths), len(lengths), H, d, inp["q"].element_size()) == moved


def test_gdn_bytes_are_the_tensors():
    inp = KI.prefill_workload("gdn_8k", "cpu", lengths=[70], heads=bench.H)
    assert inp["log_alpha"].dim() == 2  # one gate per (token, head)
    per_token = bench.GDN_BYTES_PER_TOKEN
    moved = nbytes(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"]) + nbytes(inp["v"])  # + o
    assert 70 * per_token == moved
    assert bench.prefill_bytes(70, 1, bench.H, bench.D, 2, gate_per_channel=False) == moved + 2 * nbytes(inp["S0"])


def test_main_line_constants():
    # 49,280 B per token at H = 32, d = 128, bf16: the figure the design notes and profiles use
    assert bench.PREFILL_BYTES_PER_TOKEN == 49280
    assert bench.T8K * bench.PREFILL_BYTES_PER_TOKEN + bench.PREFILL_STATE_BYTES == 407896064
    assert bench.prefill_bytes(bench.T8K, 1, bench.H, bench.D, 2) == 407896064


def test_decode_bytes_are_the_tensors():
    N, H, d = 3, bench.H, bench.D
    w = KI.decode_workload(N, H, d, 1, torch.bfloat16, "cpu")
    o = torch.empty_like(w["v"][0])
    moved = nbytes(w["q"][0], w["k"][0], w["v"][0], w["log_alpha"][0], w["beta"][0], o) + 2 * nbytes(w["S0"])
    assert bench.DECODE_BYTES // bench.DEC_N * N == moved


def test_conv_bytes_are_the_tensors():
    W = bench.CONV_W
    x, w, st = KI.conv_inputs(bench.T8K, bench.H * bench.D, W, 1, torch.bfloat16, "cpu")
    moved = nbytes(x) + nbytes(x) + nbytes(w) + 2 * nbytes(st)  # x read, y written, taps, state in and out
    assert bench.CONV_BYTES == moved


def test_committed_profiles_carry_the_machine_read_fields():
    for name, sources in (("fused_kernel_prefill_8k.md", bench.PREFILL_SOURCES),
                          ("decode_kernel_decode_256.md", bench.DECODE_SOURCES)):
        txt = open(os.path.join(ROOT, "profiles", name)).read()
        assert re.search(r"traffic_bytes_per_launch:\s*\d+", txt), name
        assert re.search(r"source_sha256:\s*[0-9a-f]{64}", txt), name
        for f in sources:
            assert os.path.exists(os.path.join(ROOT, f)), f


def test_profiled_traffic_follows_the_source_hash(tmp_path, monkeypatch):
    src = tmp_path / "k.cu"
    src.write_text("kernel source")
    (tmp_path / "profiles").mkdir()
    h = hashlib.sha256(b"kernel source").hexdigest()
    (tmp_path / "profiles" / "p.md").write_text("traffic_bytes_per_launch: 1234\nsource_sha256: %s\n" % h)
    monkeypatch.setattr(bench.os.path, "abspath", lambda p: str(tmp_path / "bench.py"))
    assert bench.profiled_traffic("p.md", ["k.cu"]) == 1234
    src.write_text("kernel source, edited")
    assert bench.profiled_traffic("p.md", ["k.cu"]) is None
