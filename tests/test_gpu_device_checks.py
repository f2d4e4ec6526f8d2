"""The checked build (libdsaidx_checked.so, compiled with -DDSA_DEVICE_CHECKS=1) on the exact parity
cases.

Its kernels verify the indices they compute on the device - every gathered key row of the
tensor-core producers, the candidate positions and output slots of the PIVOT Reuse selection, the
bitmap words and output slots of the selects - and record a violation (code 4, with the site) in
the workspace status word instead of touching memory outside a buffer.  With DSA_LIBRARY=checked
the package loads that build and raises after any call whose status word holds such a record, so
the exact integer suites passing through it show that no index left its buffer.  A malformed
caller-supplied candidate list is still reported with its own code (2).
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CASES = "exact or refine_on_supplied or misleads or layer or k_larger or all_equal or k_is_one"


def checked_env():
    return dict(os.environ, DSA_LIBRARY="checked")


def test_checked_build_is_loaded():
    out = subprocess.run([sys.executable, "-c", "import sparse_attention_indexer_04_b200 as d; print(d.LIB_PATH)"],
                         cwd=ROOT, env=checked_env(), capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    assert out.stdout.strip().endswith("libdsaidx_checked.so")


def test_exact_suites_record_no_index_error():
    files = ["tests/test_gpu_dense.py", "tests/test_gpu_variants.py", "tests/test_gpu_layers.py",
             "tests/test_gpu_limits.py"]
    r = subprocess.run([sys.executable, "-m", "pytest", *files, "-q", "-x", "-m", "gpu", "-k", CASES, "-p",
                        "no:cacheprovider"], cwd=ROOT, env=checked_env(), capture_output=True, text=True,
                       timeout=1500)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
    assert " passed" in r.stdout and "failed" not in r.stdout
