import os
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")


def _compile_host_tool(src_name: str, tmp_dir: str) -> str:
    src = os.path.join(ROOT, "tests", "native", src_name)
    exe = os.path.join(tmp_dir, os.path.splitext(src_name)[0])
    subprocess.check_call(["nvcc", "-O0", "-Wno-deprecated-gpu-targets", "-o", exe, src])
    return exe


@pytest.fixture(scope="session")
def curand_philox(tmp_path_factory):
    """Callable: (counters [n,4], keys [n,2]) -> words [n,4] from curand's
    host-side Philox4x32-10."""
    exe = _compile_host_tool("curand_philox_ref.cu", str(tmp_path_factory.mktemp("curand")))

    def run(ctr: np.ndarray, key: np.ndarray) -> np.ndarray:
        lines = "\n".join("%x %x %x %x %x %x" % (*map(int, c), *map(int, k)) for c, k in zip(ctr, key))
        out = subprocess.run([exe], input=lines + "\n", capture_output=True, text=True, check=True).stdout
        return np.array([[int(w, 16) for w in ln.split()] for ln in out.strip().splitlines()], dtype=np.uint32)

    return run


@pytest.fixture(scope="session")
def cuda_fp4_rn(tmp_path_factory):
    """Callable: float32 array -> E2M1 codes from cuda_fp4.h's host
    round-to-nearest conversion."""
    exe = _compile_host_tool("cuda_fp4_ref.cu", str(tmp_path_factory.mktemp("cudafp4")))

    def run(x: np.ndarray) -> np.ndarray:
        bits = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
        out = subprocess.run([exe], input="\n".join("%x" % int(b) for b in bits) + "\n", capture_output=True,
                             text=True, check=True).stdout
        return np.array([int(t, 16) for t in out.split()], dtype=np.uint8)

    return run
