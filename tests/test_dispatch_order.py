"""Host logic of the attention kernels' CTA dispatch order: compiles a small
host program against the kernels' own header with nvcc and runs it (no GPU
needed)."""
import os
import shutil
import subprocess
import tempfile

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "..", "block_sparse_long_key_b200", "csrc")


@pytest.mark.skipif(shutil.which("nvcc") is None, reason="needs nvcc")
def test_bucket_order_and_lead():
    with tempfile.TemporaryDirectory() as td:
        exe = os.path.join(td, "dispatch_order")
        subprocess.run(["nvcc", "-std=c++17", "-O1", "-I" + CSRC, os.path.join(HERE, "host", "dispatch_order.cu"),
                        "-o", exe], check=True, capture_output=True)
        out = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0 and out.stdout.strip() == "ok", out.stdout + out.stderr
