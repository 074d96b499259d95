"""Host-side bookkeeping of bench.py: the digest that ties a committed DRAM-traffic
capture to the kernel source it was taken on, and the kernel count per step that
the bench reports as its launch figure."""
import json
import os
from types import SimpleNamespace

import pytest
import torch

import bench


@pytest.fixture(scope="module", autouse=True)
def _library():
    """segment_params and launches_per_step take the route from the library's
    host-only lora_segment_plan."""
    from lora_adapter_application_b200 import build
    build.build()
    import lora_adapter_application_b200 as lora
    lora.load()

CODE = """// fused kernel
__global__ void k(float* y) {   /* body */
    y[threadIdx.x] += 1.0f;     // one add
}
"""


def _write(path, text):
    with open(path, "w") as f:
        f.write(text)


def test_code_digest_ignores_comments_and_spacing(tmp_path):
    a, b = tmp_path / "a.cu", tmp_path / "b.cu"
    _write(a, CODE)
    _write(b, "/* a different\n   header */\n__global__ void k(float* y)\n{\n"
              "  y[threadIdx.x]  +=  1.0f;  // another comment\n}\n")
    assert bench.code_digest(a) == bench.code_digest(b)


def test_code_digest_changes_with_code(tmp_path):
    a, b = tmp_path / "a.cu", tmp_path / "b.cu"
    _write(a, CODE)
    _write(b, CODE.replace("1.0f", "2.0f"))
    assert bench.code_digest(a) != bench.code_digest(b)


def _fake_root(tmp_path, src_text, recorded_text):
    csrc = tmp_path / "lora_adapter_application_b200" / "csrc"
    csrc.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    _write(csrc / "bgmv.cu", src_text)
    rec_src = tmp_path / "recorded.cu"
    _write(rec_src, recorded_text)
    rec = {"bgmv_kernel": {"code_sha256": bench.code_digest(rec_src),
                           "decode_qproj": {"dram_bytes_per_launch": [123456.0]},
                           "multislice_8b": {"dram_bytes_per_launch": [1.0, 2.0, 3.0, 4.0]}}}
    _write(tmp_path / "profiles" / "traffic.json", json.dumps(rec))


def test_traffic_kept_while_code_unchanged(tmp_path, monkeypatch):
    _fake_root(tmp_path, CODE + "// a note added after the capture\n", CODE)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_traffic("decode_qproj", 1) == (123456.0, [123456.0])
    # a layer set: one figure per layer, summed over the step
    assert bench.measured_traffic("multislice_8b", 4) == (10.0, [1.0, 2.0, 3.0, 4.0])
    assert bench.measured_traffic("multislice_8b", 3) == (None, None)   # layers missing
    assert bench.measured_traffic("prefill", 1) == (None, None)         # no capture for it


def test_traffic_dropped_once_code_changes(tmp_path, monkeypatch):
    _fake_root(tmp_path, CODE.replace("+=", "-="), CODE)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_traffic("decode_qproj", 1) == (None, None)


def test_traffic_missing_record(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_traffic("decode_qproj", 1) == (None, None)


def _w(name, T, N, r_max, slices_per_layer, dtype=torch.bfloat16, d_out=64):
    widths = d_out if isinstance(d_out, list) else [d_out] * len(slices_per_layer)
    layers = [SimpleNamespace(d_out=[c] * s) for s, c in zip(slices_per_layer, widths)]
    return SimpleNamespace(name=name, T=T, N=N, r_max=r_max, dtype=dtype, layers=layers)


def test_launches_per_step_hand_counted():
    # decode-only batch: one-block grouping + one gathered-tile kernel per layer
    assert bench.launches_per_step(_w("decode_qproj", 256, 32, 16, [1])) == 2
    assert bench.launches_per_step(_w("multislice_8b", 1024, 100, 64, [3, 1, 2, 1])) == 5
    # prompts: the tensor-core kernel joins each layer it can take
    assert bench.launches_per_step(_w("prefill", 77000, 8, 16, [1])) == 7 + 1 + 1
    # 70B MLP batch (up and down projections, r 16): both layers take both kernels
    assert bench.launches_per_step(_w("mixed_70b", 8192, 16, 16, [1, 1])) == 1 + 2 + 2
    # two slices of 64 ranks stack to 128: still the tensor-core kernel
    assert bench.launches_per_step(_w("prefill", 4096, 8, 64, [2])) == 1 + 2
    # more than 128 stacked ranks, r_max not a multiple of 16, or fp32: no tensor-core kernel
    assert bench.launches_per_step(_w("prefill", 2048, 8, 64, [3])) == 1 + 1
    assert bench.launches_per_step(_w("prefill", 2048, 8, 24, [1])) == 1 + 1
    assert bench.launches_per_step(_w("prefill", 2048, 8, 16, [1], torch.float32)) == 1 + 1
    # a batch with fewer 128-row tiles than SMs and a layer 8192+ columns wide: the
    # gathered-tile kernel takes every row of that layer (the 70B MLP's two layers)
    assert bench.launches_per_step(_w("mixed_70b", 8192, 16, 16, [1, 1], d_out=[28672, 8192]), sms=148) == 1 + 1 + 1
    assert bench.launches_per_step(_w("mixed_70b", 8192, 16, 16, [1, 1], d_out=[28672, 4096]), sms=148) == 1 + 1 + 2
    assert bench.launches_per_step(_w("mixed_70b", 8192, 16, 16, [1, 1], d_out=[28672, 8192]), sms=40) == 1 + 2 + 2
    assert bench.launches_per_step(_w("prefill", 77000, 8, 16, [1], d_out=[28672]), sms=148) == 7 + 2


def test_segment_params_follow_the_route(monkeypatch):
    monkeypatch.delenv("LORA_TC_ROUTE", raising=False)
    # decode-only and narrow prompt batches: the table's runs, 16-row tiles
    assert bench.segment_params(_w("decode_qproj", 256, 32, 16, [1]), sms=148) == (16, 0)
    assert bench.segment_params(_w("prefill", 77000, 8, 16, [1], d_out=4096), sms=148) == (16, 64)
    # every layer 8192+ wide with fewer 128-row tiles than SMs: no runs, 32-row tiles
    wide = _w("mixed_70b", 8192, 16, 16, [1, 1], d_out=[28672, 8192])
    assert bench.segment_params(wide, sms=148) == (32, 0)
    assert bench.segment_params(wide, sms=40) == (16, 64)
    # one narrow layer keeps the runs for the tensor-core kernel
    assert bench.segment_params(_w("mixed_70b", 8192, 16, 16, [1, 1], d_out=[28672, 4096]), sms=148) == (16, 64)
    # a long prefill batch fills the SMs with 128-row tiles: runs kept
    assert bench.segment_params(_w("prefill", 77000, 8, 16, [1], d_out=[28672]), sms=148) == (16, 64)
    monkeypatch.setenv("LORA_TC_ROUTE", "1")
    assert bench.segment_params(wide, sms=148) == (16, 64)
    assert bench.launches_per_step(wide, sms=148) == 1 + 2 + 2
    monkeypatch.setenv("LORA_TC_ROUTE", "2")
    assert bench.segment_params(wide, sms=148) == (32, 0)


def test_launches_per_step_grouping_boundaries():
    assert bench.launches_per_step(_w("decode_qproj", 2048, 5000, 16, [1])) == 2
    assert bench.launches_per_step(_w("decode_qproj", 2049, 5000, 16, [1])) == 8
    assert bench.launches_per_step(_w("decode_qproj", 8192, 1023, 16, [1])) == 2
    assert bench.launches_per_step(_w("decode_qproj", 8192, 1024, 16, [1])) == 8
    assert bench.launches_per_step(_w("decode_qproj", 8193, 8, 16, [1])) == 8


def test_reference_arm_under_torchrun_two_ranks():
    """`bench.py --impl reference` launched the way a 2-GPU run is: rank 0 alone
    times the oracle and prints one JSON line; the other rank exits 0 without work."""
    import socket
    import subprocess
    import sys
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py",
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3",
           "--ref-seconds", "1", "--cpu-budget", "1"]
    r = subprocess.run(cmd, cwd=bench.ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2 and rec["steps"] == 1
    assert rec["cpu_baseline"]["kind"] == "oracle" and rec["value"] > 0
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["e2e"]["d2h_bytes_per_step"] == 0
