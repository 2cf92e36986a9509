"""Host check of the packed-sequence work mapping (`packed_unit` in
csrc/attn_internal.h): the grid row of floor(total / U) + num_seqs items
reaches every unit of every sequence exactly once and leaves at most one empty
item per sequence, over thousands of random length mixes (empty and one-row
sequences included). The C++ check is compiled with nvcc for the host; no GPU
is needed."""
import os
import shutil
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_packed_unit_reaches_every_unit_once():
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    with tempfile.TemporaryDirectory() as tmp:
        exe = os.path.join(tmp, "packed_unit_check")
        subprocess.run([nvcc, "-O2", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
                        "-I", os.path.join(ROOT, "include"), "-o", exe,
                        os.path.join(ROOT, "tests", "native", "packed_unit_check.cu")],
                       check=True, capture_output=True, text=True, timeout=300)
        r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.startswith("ok"), r.stdout + r.stderr
