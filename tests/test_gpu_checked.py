"""The index-checked build (libh3b_check.so, compiled with -DH3B_CHECK=1):
every hand-indexed global load and store checks its element range against
its buffer's extent and records a violation in the device error word instead
of performing it.  The same calls (tests/checked_run.py: every kernel family,
ragged tails, split-K and key-split tails, folded norms, reduction windows,
condition rows, the loop) must record nothing and give the default build's
results bit for bit."""
import os
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "audio_diffusion_transformer_dit_b200")


def _run(tmp_path, lib):
    out = os.path.join(tmp_path, os.path.basename(lib) + ".npz")
    env = dict(os.environ, H3B_LIBRARY=lib)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "checked_run.py"), out], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
    return np.load(out)


@pytest.mark.gpu
def test_index_checked_build_records_nothing_and_matches(tmp_path):
    lib_check = os.path.join(PKG, "libh3b_check.so")
    assert os.path.exists(lib_check), "libh3b_check.so not built (python -m audio_diffusion_transformer_dit_b200.build)"
    ref = _run(str(tmp_path), os.path.join(PKG, "libh3b.so"))
    chk = _run(str(tmp_path), lib_check)
    assert int(ref["device_error"][0]) == 0
    assert int(chk["device_error"][0]) == 0, f"index check fired: code {int(chk['device_error'][0]):#x}"
    # the check records an out-of-range index in the checked build only, and
    # nothing for an index inside its extent
    assert int(ref["index_checked"][0]) == 0 and int(chk["index_checked"][0]) == 1
    assert int(ref["selftest_error"][0]) == 0 and int(chk["selftest_error"][0]) == (4 << 8) | 99
    assert int(ref["selftest_in_range_error"][0]) == 0 and int(chk["selftest_in_range_error"][0]) == 0
    assert sorted(ref.files) == sorted(chk.files)
    skip = {"index_checked", "selftest_error"}
    for k in ref.files:
        if k not in skip:
            assert np.array_equal(ref[k], chk[k], equal_nan=True), k
