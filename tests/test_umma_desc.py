"""The tcgen05 descriptor encodings of the dense refresh-edge kernel, checked on the host.

gm_umma.cuh builds the tensor-core instruction descriptor (bf16 x bf16 -> fp32, K-major) and
the shared-memory matrix descriptor (128-byte swizzle, K-major) by hand. This test compiles a
host-only program (tests/umma/check_desc.cu) that sets the same fields through CUTLASS's bit
field definitions of those descriptors and compares the bits. No GPU is needed.
"""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


def cutlass_include():
    """CUTLASS/CuTe headers vendored with an installed package (found without importing it)."""
    import importlib.util
    spec = importlib.util.find_spec("flashinfer")
    if spec is None or spec.origin is None:
        return None
    inc = os.path.join(os.path.dirname(spec.origin), "data", "cutlass", "include")
    return inc if os.path.isdir(os.path.join(inc, "cute")) else None


@pytest.mark.skipif(shutil.which("nvcc") is None and not os.path.exists("/usr/local/cuda/bin/nvcc"),
                    reason="needs nvcc")
def test_descriptors_match_cutlass_bit_fields(tmp_path):
    inc = cutlass_include()
    if inc is None:
        pytest.skip("CUTLASS headers not found")
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    exe = tmp_path / "check_desc"
    subprocess.run([nvcc, "-std=c++17", "-I", inc, os.path.join(HERE, "umma", "check_desc.cu"), "-o",
                    str(exe)], check=True, capture_output=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0 and out.stdout.strip().endswith("ok"), out.stdout + out.stderr
