"""The boundary as a C caller sees it: include/lora_delta.h compiles as strict
C99 and as C++17, and a C program linked against the built library calls the
host-only entry points (sizes, status strings, the segment plan, the slot
cache) with the results their declarations state.  Runs without a GPU."""
import os
import shutil
import subprocess

import pytest

import lora_adapter_application_b200 as lora

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")
PKG = os.path.dirname(os.path.abspath(lora.__file__))
SRC = os.path.join(ROOT, "tests", "c", "abi_host.c")

pytestmark = pytest.mark.skipif(shutil.which("gcc") is None or shutil.which("g++") is None,
                                reason="needs gcc and g++")


@pytest.fixture(scope="module")
def built():
    from lora_adapter_application_b200 import build
    build.build()
    lora.load()


def test_header_compiles_as_c99_and_cxx17():
    for cmd in (["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-fsyntax-only"],
                ["g++", "-std=c++17", "-Wall", "-Wextra", "-Werror", "-pedantic", "-fsyntax-only",
                 "-x", "c++"]):
        r = subprocess.run(cmd + ["-I", INCLUDE, SRC], capture_output=True, text=True)
        assert r.returncode == 0, r.stderr


def test_c_program_calls_host_entry_points(built, tmp_path, monkeypatch):
    monkeypatch.delenv("LORA_TC_ROUTE", raising=False)
    exe = str(tmp_path / "abi_host")
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", INCLUDE, SRC, "-L", PKG,
                        "-llora_delta", f"-Wl,-rpath,{PKG}", "-o", exe],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, (r.stdout, r.stderr)
    out = dict(line.split(" ", 1) for line in r.stdout.strip().splitlines())
    assert int(out["version"]) == lora.lora_version()
    assert out["status"] == "LORA_ERR_SHAPE"
    # 64 tiles of 16 rows + up to 100 partial ones; no contiguous tiles with min_run 0
    assert out["capacity"] == "164 0"
    assert int(out["scratch"]) == lora.lora_segments_scratch_bytes(77431, 8)
    # 8192 rows (64 long tiles < 148 SMs), both layers 8192+ wide: 32-row tiles, no runs
    assert out["plan"] == "32 0 1 1"
    assert out["plan_null"] == "-1"                       # LORA_ERR_NULL
    assert out["acquire"] == "0 0 42"                     # a free slot, to be loaded
    assert out["again"] == "0 1"                          # resident, second pin
    assert out["evict_pinned"] == "-7"                    # LORA_ERR_CAPACITY while pinned
    assert out["evict"] == "0 -1"                         # freed once unpinned
