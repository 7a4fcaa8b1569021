"""CPU check of the short-batch forward kernel's shared-memory plan, compiled
from the header the kernel uses (no GPU needed)."""
import os
import subprocess

from invariant_lm_head_gemm_b200 import build

HERE = os.path.dirname(os.path.abspath(__file__))
EXE = os.path.join(HERE, "..", "_build", "decode_config_check")


def test_decode_shared_memory_plan():
    os.makedirs(os.path.dirname(EXE), exist_ok=True)
    subprocess.check_call([build.NVCC] + build.ARCH + ["-std=c++17", "-O1", "-I" + build.CSRC,
                           "-I" + build.INCLUDE, os.path.join(HERE, "decode_config_check.cu"),
                           "-o", EXE])
    out = subprocess.run([EXE], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0 and out.stdout.strip().endswith("OK"), out.stdout + out.stderr
    print(out.stdout)
