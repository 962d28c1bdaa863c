"""The range-checking build (libala_debug.so, ALA_DEBUG_BOUNDS=1) on the GPU.

Its kernels check every block-table entry they read against [0, numBlocks).
A bad entry does not fault: the kernel records code 0x10B in the status word and
reads the zero-filled row past the cache instead (the same bounds-checked TMA
load a pointer past the last page uses).  The cases run in a child process
(tests/debug_bounds_run.py) so that the main test process keeps libala.so.
"""
import json
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BAD_BLOCK_INDEX = 0x10B


@pytest.fixture(scope="module")
def results():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from paged_attention_varlen_b200 import build
    build.build(debug_bounds=True)
    env = dict(os.environ, ALA_LIBRARY="debug")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "debug_bounds_run.py")], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    return json.loads(r.stdout.strip().splitlines()[-1])


def test_debug_build_valid_tables_pass_with_status_clean(results):
    for case in ("prefill_ok", "mla_ok"):
        assert results[case]["status"] == 0, case
        assert results[case]["max_err"] <= 2e-2, case


def test_debug_build_reports_a_block_index_outside_the_cache(results):
    assert results["prefill_bad_entry"]["status"] == BAD_BLOCK_INDEX
    assert results["mla_bad_entry"]["status"] == BAD_BLOCK_INDEX
