"""Host check (no GPU) that the library's cached set-up -- kernel attributes,
SM counts, the no-alloc scratch address -- is keyed by device index: compiles
tests/native/device_once_check.cpp against the library's device_once.h with the
host C++ compiler and runs it."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "boolean_weight_matmul_b200", "csrc")
SRC = os.path.join(ROOT, "tests", "native", "device_once_check.cpp")


def test_per_device_setup_caches(tmp_path):
    cxx = shutil.which("g++") or shutil.which("c++")
    if cxx is None:
        pytest.skip("no host C++ compiler")
    exe = str(tmp_path / "device_once_check")
    subprocess.run([cxx, "-std=c++17", "-O1", "-pthread", "-I", CSRC, SRC, "-o", exe], check=True)
    r = subprocess.run([exe], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr


def test_every_attribute_cache_is_per_device():
    """No kernel launcher keeps a process-wide 'attribute already set' flag."""
    for name in os.listdir(CSRC):
        if not name.endswith((".cu", ".cuh")):
            continue
        with open(os.path.join(CSRC, name)) as f:
            text = f.read()
        assert "static bool attr_set" not in text, name
        if "cudaFuncSetAttribute" in text:
            assert name == "mbok_common.cuh", f"{name} sets kernel attributes outside set_smem_attr_once"
