"""The parity suites again, on the bounds-guard build libsq_debug.so (the same kernels with
device-side guards on their data-dependent indices: gathered positions, outlier indices,
tail stores). Every test there ends its GPU work with sq_sync_status(), which raises if a
guard fired, so a green run means no guarded access left its buffer on those shapes.
Runs in a child process, because the binding loads one library per process."""
import os
import subprocess
import sys

import pytest

from w8a8_quantized_gemm_b200 import build as _b

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SUITES = ["tests/test_gpu_gemm.py", "tests/test_gpu_quant.py", "tests/test_gpu_llmint8.py",
          "tests/test_gpu_variants.py"]


def test_parity_suites_on_the_guarded_build():
    assert os.path.exists(_b.LIB_DEBUG), "libsq_debug.so is not built"
    env = dict(os.environ, SQ_LIB_PATH=_b.LIB_DEBUG)
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider", *SUITES],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=1800)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
    assert " passed" in r.stdout
