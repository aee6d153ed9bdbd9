"""The split-K W4A16 work partition on the host: tests/native/w4_partition_check.cu
includes the kernel header and checks its partition functions (every unit in one
run, runs contiguous and non-empty, unique partial slots, tiles inside a run
whole) for the CTA counts the library launches. Needs nvcc, no GPU."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
NVCC = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"


@pytest.mark.skipif(not os.path.exists(NVCC), reason="nvcc not found")
def test_w4a16_splitk_partition(tmp_path):
    exe = tmp_path / "w4_partition_check"
    subprocess.run([NVCC, "-std=c++17", "-O1", "-gencode", "arch=compute_100a,code=sm_100a",
                    f"-I{ROOT}/include", f"-I{ROOT}/exact_attention_forward_11_b200/csrc",
                    "-o", str(exe), os.path.join(HERE, "native", "w4_partition_check.cu")],
                   check=True, capture_output=True, text=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stdout + out.stderr
    assert out.stdout.startswith("ok")
