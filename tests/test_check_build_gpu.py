"""The bounds-checked debug build (libwf_check.so, -DWF_CHECK) on the GPU.

Every kernel family runs on ragged seeded shapes (ring wrap, partial tiles, N
not a multiple of 256, ragged K) once with the debug build, in a subprocess,
and once with the normal build in this process.  No check may fire (every
status WF_OK), and the outputs must be bit-identical: the checks skip nothing
on valid shapes and change no arithmetic."""
import os
import subprocess
import sys

import numpy as np
import pytest

from chunk_causal_dit_b200 import build as wf_build

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_debug_build_passes_every_check_and_matches(tmp_path):
    wf_build.build()
    wf_build.build(check=True)
    out = tmp_path / "check.npz"
    env = dict(os.environ, WF_LIB_VARIANT="check")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "check_build_driver.py"),
                        str(out)], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    dbg = np.load(out)
    from chunk_causal_dit_b200 import wf
    from tests.check_build_driver import run_all
    ref, st = run_all(wf)
    for name, s in st.items():
        assert s == wf.WF_OK, "normal build: %s status %d" % (name, s)
        assert int(dbg["status_" + name]) == wf.WF_OK, \
            "debug build: a bounds check fired in %s (status %d)" % (name, int(dbg["status_" + name]))
    for name, a in ref.items():
        assert np.array_equal(dbg[name], a), name
