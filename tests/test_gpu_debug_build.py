"""The debug build (libfa_debug.so, compiled with FA_DEBUG_CHECKS): its kernels check the
bounds of every global-memory index they compute by hand and report a failure through the
error word instead of touching memory outside a buffer.  On the GPU, every path run through
the debug build must match the oracle with no check firing, and the bounds self-test must
make the check fire (and skip the stores) without disturbing the outputs it does write.  On
the CPU, the builds report their flags and the release build refuses the self-test."""
import ctypes
import os
import subprocess
import sys

import pytest

from exact_io_aware_81_b200 import build, ops

HERE = os.path.dirname(os.path.abspath(__file__))


def test_build_flags_and_release_refuses_the_bounds_selftest():
    build.build()
    build.build(debug=True)
    rel = ctypes.CDLL(build.LIB)
    dbg = ctypes.CDLL(build.LIB_DEBUG)
    assert rel.fa_build_flags() == 0 and dbg.fa_build_flags() == 1
    fake = 0x10000  # never dereferenced: the release build returns before any launch
    rc = rel.fa_debug_selftest_bounds(fake, fake, fake, fake, fake, 1, 4, 4, 256, 256, 128, ctypes.c_float(0.1), 1,
                                      None)
    assert rc == ops.FA_ERR_UNSUPPORTED


@pytest.mark.gpu
def test_debug_build_paths_and_bounds_selftest():
    build.build(debug=True)
    env = dict(os.environ, FA_LIBRARY=build.LIB_DEBUG)
    r = subprocess.run([sys.executable, os.path.join(HERE, "debug_worker.py")], env=env, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-3000:]
    assert "debug build ok" in r.stdout
