"""CPU check of the fused backward's unit schedule, compiled from the same
header the kernel uses (no GPU needed)."""
import os
import subprocess

import pytest

from invariant_lm_head_gemm_b200 import build

HERE = os.path.dirname(os.path.abspath(__file__))
EXE = os.path.join(HERE, "..", "_build", "bwd_schedule_check")


@pytest.fixture(scope="module")
def exe():
    os.makedirs(os.path.dirname(EXE), exist_ok=True)
    subprocess.check_call([build.NVCC] + build.ARCH + ["-std=c++17", "-O1", "-I" + build.CSRC,
                           "-I" + build.INCLUDE,
                           os.path.join(HERE, "bwd_schedule_check.cu"), "-o", EXE])
    return EXE


def _vchunk(V):
    return min(8192, (V + 255) // 256 * 256)


@pytest.mark.parametrize("T,H,V", [
    (1, 64, 1), (7, 64, 129), (130, 128, 1000), (257, 192, 8193), (300, 256, 20000),
    (512, 1024, 32768), (5980, 4096, 151936), (64, 256, 1024), (8192, 4096, 151936),
    (129, 4096, 3 * 8192), (200, 320, 4 * 8192 + 5),
])
def test_schedule(exe, T, H, V):
    out = subprocess.run([exe, str(T), str(H), str(V), str(_vchunk(V))], capture_output=True,
                         text=True, timeout=600)
    assert out.returncode == 0 and out.stdout.startswith("OK"), out.stdout + out.stderr
