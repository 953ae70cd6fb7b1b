"""The debug-check build (libsamba_debug.so, SAMBA_DEBUG_CHECKS=1): its two
self-tests report SAMBA_ERR_BOUNDS with the failing site and leave the context
usable, and the library's entry points run under it with no device check
failing, no workspace guard band and no margin around a user buffer
overwritten, and the same oracle parity as the release build.  The workload
runs in a child process (tests/debug_checks_child.py) because the binding
chooses the library when it is first imported."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def run():
    lib = os.path.join(ROOT, "sliding_window_attention_samba_b200", "libsamba_debug.so")
    if not os.path.exists(lib):
        from sliding_window_attention_samba_b200 import build
        build.build(debug_checks=True)
    env = dict(os.environ, SAMBA_DEBUG_CHECKS="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "debug_checks_child.py")], env=env,
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    return json.loads(r.stdout.strip().splitlines()[-1])


def test_debug_library_is_loaded(run):
    assert run["enabled"] == 1 and run["lib"] == "libsamba_debug.so"


def test_device_check_selftest_reports_site(run):
    from sliding_window_attention_samba_b200._lib import SAMBA_ERR_BOUNDS, SAMBA_OK
    assert run["kind0_rc"] == SAMBA_OK
    assert run["kind0_err"] == SAMBA_ERR_BOUNDS
    assert run["kind0_site"].startswith("elementwise.cu:")


def test_guard_band_selftest_reports_band(run):
    from sliding_window_attention_samba_b200._lib import SAMBA_ERR_BOUNDS, SAMBA_OK
    assert run["kind1_rc"] == SAMBA_OK
    assert run["kind1_err"] == SAMBA_ERR_BOUNDS
    assert run["kind1_site"] == "workspace guard band 0 overwritten"
    assert run["after_err"] == SAMBA_OK  # read and cleared; the context stays usable


def test_entry_points_clean_under_checks(run):
    for k in ("scan", "swa", "block"):
        assert run[f"{k}_err"] == 0, (k, run)
        assert run[f"{k}_margins"], (k, run)
    assert run["block_pos"] == [160 + 96 + 3] * 2
    assert run["smoke"] == "ok"
