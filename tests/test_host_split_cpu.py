"""Host-side logic of the gated decode split, compiled and run on the CPU:
``tests/host/gated_split_check.cu`` includes the library's internal header
and checks ``gated_cold_split`` (CTA limit, exact cover, partial slots per
unit) over a grid of sizes.  Needs nvcc only (no GPU, no CUDA call)."""
import os
import shutil
import subprocess
import tempfile

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


def _nvcc():
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    return None


@pytest.mark.skipif(_nvcc() is None, reason="nvcc not available")
def test_gated_cold_split_invariants():
    with tempfile.TemporaryDirectory() as tmp:
        exe = os.path.join(tmp, "gated_split_check")
        subprocess.run([_nvcc(), "-std=c++17", "-O1",
                        "-I", os.path.join(ROOT, "compressed_decode_attention_encode_b200", "csrc"),
                        "-I", os.path.join(ROOT, "include"),
                        os.path.join(HERE, "host", "gated_split_check.cu"), "-o", exe],
                       check=True, capture_output=True)
        out = subprocess.run([exe], capture_output=True, text=True)
        assert out.returncode == 0, out.stdout + out.stderr
        assert out.stdout.startswith("ok")
