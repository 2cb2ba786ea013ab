"""The small parity and canary cases once more, under libfa_checks.so: the same
ABI compiled with FA_CHECKS, whose kernels check each direct memory access
against its tensor's size and record FA_ERR_BOUNDS in the device status word
(skipping the access) instead of making it.  Every test below ends by asserting
a clean status word, so an out-of-range index anywhere in these cases fails.

Run in a child process, because the library is chosen when it is first
loaded (FA_LIBRARY names the file).  The full-size workloads are left to the
normal build; these cases span every kernel, ragged tails, single rows, GQA,
d = 64 and 128, fp16 and bf16, dropout, block-sparse empty tiles, FP8 and the
fp32 accumulator paths.
"""
import os
import subprocess
import sys

import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CHECKS = os.path.join(ROOT, "exact_io_aware_80_b200", "libfa_checks.so")


def test_small_cases_pass_under_the_index_checking_build():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    assert os.path.exists(CHECKS), "libfa_checks.so is not built (python -m exact_io_aware_80_b200.build --checks)"
    env = dict(os.environ, FA_LIBRARY="libfa_checks.so")
    probe = subprocess.run([sys.executable, "-c", "from exact_io_aware_80_b200 import _lib; _lib.load(); "
                            "print(_lib.LIB_PATH)"], env=env, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert probe.returncode == 0 and probe.stdout.strip().endswith("libfa_checks.so"), probe.stderr
    files = ["tests/test_gpu_parity.py", "tests/test_gpu_canaries.py", "tests/test_gpu_blocksparse.py",
             "tests/test_gpu_dropout.py", "tests/test_gpu_fp8.py", "tests/test_gpu_ring.py"]
    sel = ("not full and not training and not long and not workload_sampled and not eight_ranks "
           "and not persistent and not process_group and not 8192")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu and not slow", "-k", sel] + files,
                       env=env, cwd=ROOT, capture_output=True, text=True, timeout=1500)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
    assert " passed" in r.stdout
