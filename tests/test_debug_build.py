"""The debug build libfa_debug.so (the library's sources compiled with FA_DEBUG): device-side
index checks and per-kernel tile-visit counters, the stand-in for a memory checker.

On the host: the debug library exists, reports itself as the debug build and exports every
function that include/fa.h declares; the release library refuses the visit-counter call.
On a GPU: tests/_debug_visits.py, in a fresh process bound to the debug library, checks that
every kernel kind visits each visible (query tile, key tile) pair exactly once and no other, at
ragged lengths, both masks and both head dimensions, with no index check failing.
"""
import ctypes
import os
import subprocess
import sys

import numpy as np
import pytest

from io_aware_exact_22_b200 import fa
from tests.test_abi import declared_functions

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
DEBUG_LIB = os.path.join(ROOT, "io_aware_exact_22_b200", "libfa_debug.so")


def test_debug_library_exports_the_abi():
    assert os.path.exists(DEBUG_LIB), "build it with `python -m io_aware_exact_22_b200.build --all`"
    D = ctypes.CDLL(DEBUG_LIB)
    for name in declared_functions():
        assert hasattr(D, name), name
    D.fa_debug_build.restype = ctypes.c_int
    assert D.fa_debug_build() == 1


def test_release_library_has_no_visit_counters():
    assert fa.fa_debug_build() == 0
    assert fa.fa_debug_visits(np.zeros(4, dtype=np.int32), 4, True, 0) == 2  # FA_ERR_UNSUPPORTED
    assert fa.fa_status_string(5) == "FA_ERR_DEVICE_CHECK"


@pytest.mark.gpu
def test_debug_build_visits_exactly_the_visible_tiles(cuda_ok):
    env = dict(os.environ, FA_LIB_PATH=DEBUG_LIB)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "_debug_visits.py")], cwd=ROOT,
                       env=env, capture_output=True, text=True, timeout=900)
    print(r.stdout[-2000:])
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert "visited exactly once" in r.stdout
