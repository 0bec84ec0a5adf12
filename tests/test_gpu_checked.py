"""The bounds-checked build (libattamba_checked.so) on small valid inputs (GPU).

That build compiles the same kernels with ATTAMBA_CHECKED: the attention's item
tiles and per-row key ranges, the decode step's ring position, boundary rows and
split ranges, and the scan's chunk-table offsets are each tested against the
arrays they address, and a failure sets ATTAMBA_DEV_BOUNDS in the status word
instead of making the access.  It stands in for a memory checker.  Here a set of
the parity tests runs in a child process against that library: every one of them
requires a clean status word, so each check held on every access, and the
outputs still match the oracle.
"""

import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SELECTION = [
    "tests/test_gpu_index.py::test_random_sweep",
    "tests/test_gpu_scan.py::test_scan_small",
    "tests/test_gpu_attn.py::test_attention_small",
    "tests/test_gpu_attn.py::test_attention_wide_score_range",
    "tests/test_gpu_decode.py::test_decode_many_splits",
    "tests/test_gpu_decode.py::test_decode_after_short_handoff_into_long_capacity",
    "tests/test_gpu_decode.py::test_full_cache_raises_status_bit",
    "tests/test_gpu_handoff.py",
    "tests/test_gpu_layer.py",
]
RUNNER = """
import sys
import pytest
from ssm_compressed_chunked_b200 import attamba as A
assert "checked" in A.version(), A.version()
sys.exit(pytest.main(["-q", "-x", "-m", "gpu", "-p", "no:cacheprovider"] + sys.argv[1:]))
"""


def test_parity_cases_pass_with_every_index_checked():
    env = dict(os.environ, ATTAMBA_LIBRARY="checked", PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, "-c", RUNNER] + SELECTION, cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=1200)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
    assert " passed" in r.stdout and "failed" not in r.stdout, r.stdout[-2000:]
