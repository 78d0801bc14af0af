"""The parity suites of the quantize family, the GEMM, the routed-expert
layer and the top-k KL loss, re-run on the bounds-checking build of the
library (libnvfp4_debug.so, built with -DNVFP4_DEBUG_BOUNDS): every kernel
checks its computed global indices against the extents of its buffers and
records NVFP4_ERR_BOUNDS on a violation, skipping that access. The suites
run in a subprocess with NVFP4_LIBRARY=debug; every test there must pass
and leave no bounds status (tests/conftest.py). The full-size file is left
out to keep the run short; its launch shapes are the same kernels."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_parity_suites_on_the_bounds_checking_build():
    lib = os.path.join(ROOT, "qad_nvfp4_quantize_b200", "libnvfp4_debug.so")
    if not os.path.exists(lib):
        pytest.fail(f"{lib} is missing; build it with `python -m qad_nvfp4_quantize_b200.build --debug`")
    env = dict(os.environ, NVFP4_LIBRARY="debug")
    files = ["tests/test_gpu_quantize.py", "tests/test_gpu_gemm.py", "tests/test_gpu_moe.py",
             "tests/test_gpu_kd_loss.py"]
    res = subprocess.run([sys.executable, "-m", "pytest", *files, "-m", "gpu", "-q", "-x", "-p", "no:cacheprovider",
                          "-k", "not long_rows"],
                         cwd=ROOT, env=env, capture_output=True, text=True, timeout=1500)
    tail = "\n".join((res.stdout + res.stderr).strip().splitlines()[-25:])
    assert res.returncode == 0, tail
    assert " passed" in res.stdout, tail
