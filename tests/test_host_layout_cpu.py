"""Host-side check of the record layout helpers the encoders' word-parallel
merge relies on, compiled and run on the CPU: ``tests/host/layout_check.cu``
includes the library's internal header and checks ``sign_chunk_bit`` (one
to one; the per-half word / nibble identities the merge's compile-time sign
permutation assumes), ``lane_word_offset`` (distinct aligned words inside a
plane) and the code-word counts.  Needs nvcc only (no GPU, no CUDA call)."""
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
def test_record_layout_helpers():
    with tempfile.TemporaryDirectory() as tmp:
        exe = os.path.join(tmp, "layout_check")
        subprocess.run([_nvcc(), "-std=c++17", "-O1",
                        "-I", os.path.join(ROOT, "compressed_decode_attention_encode_b200", "csrc"),
                        "-I", os.path.join(ROOT, "include"),
                        os.path.join(HERE, "host", "layout_check.cu"), "-o", exe],
                       check=True, capture_output=True)
        out = subprocess.run([exe], capture_output=True, text=True)
        assert out.returncode == 0, out.stdout + out.stderr
        assert out.stdout.startswith("ok")
