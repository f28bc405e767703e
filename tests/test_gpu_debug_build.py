"""The FM_DEBUG build of the library (device-side checks on list lengths and entries that record
the bad value and skip the access, and shared-memory canary words checked at kernel exit; a
failed check comes back as FM_ERR_DEVICE_CHECK from fm_get_device_status) runs the small GPU
parity cases: tiny, ragged, grouped-query, fixed-order, varlen and head dimension 256.  Each of
those tests compares against the oracle and asserts a clean status word after its calls, so any
check that fires fails them; test_gpu_debug_checks then shows that a check does fire on a bad
list entry.  Run in a subprocess with FM_DEBUG=1, which makes the binding load
libfm_b200_debug.so instead of the release library."""
import os
import subprocess
import sys

import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CASES = "tiny or ragged or grouped or fixed_order or varlen or head_dim_256 or fully_masked"


def test_debug_build_runs_small_parity_cases():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mask_aware_flash_b200 import _build
    _build.build(debug=True)
    env = dict(os.environ, FM_DEBUG="1")
    chk = subprocess.run([sys.executable, "-c", "import mask_aware_flash_b200 as m; m.lib(); print(m.LIB_PATH)"],
                         cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert chk.returncode == 0 and chk.stdout.strip().endswith("libfm_b200_debug.so"), chk.stdout + chk.stderr
    r = subprocess.run([sys.executable, "-m", "pytest", os.path.join(ROOT, "tests", "test_gpu_parity.py"),
                        os.path.join(ROOT, "tests", "test_gpu_debug_checks.py"), "-q", "-m", "gpu",
                        "-k", CASES + " or bad_list_entry", "-p", "no:cacheprovider"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    tail = (r.stdout + r.stderr)[-3000:]
    assert r.returncode == 0, tail
    assert " passed" in r.stdout, tail
