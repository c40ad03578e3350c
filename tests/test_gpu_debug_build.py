"""The checked build (libws_debug.so, device index checks on every computed cache row,
output row, partial slot and merge counter; a failed check skips the access and ws_sync
reports WS_ERR_DEVICE_CHECK) on the tiny workload, ragged key runs at both head sizes,
a readback, a two-session call and a prefill stretch: every status is WS_OK and every
output is bit for bit that of the normal build.  Each library runs in a process of its
own (WS_LIBRARY is read when the binding loads)."""
import os
import subprocess
import sys

import numpy as np
import pytest

from gpu_util import require_gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


def _run(lib, path):
    env = dict(os.environ)
    env.pop("WS_LIBRARY", None)
    if lib == "debug":
        env["WS_LIBRARY"] = "debug"
    r = subprocess.run([sys.executable, os.path.join(HERE, "debug_build_cases.py"), path], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    return np.load(path)


@pytest.mark.gpu
def test_checked_build_passes_its_checks_with_identical_outputs(tmp_path):
    require_gpu()
    if not os.path.exists(os.path.join(ROOT, "kv_cache_serving_ws_b200", "libws_debug.so")):
        from kv_cache_serving_ws_b200 import build
        build.build(debug=True)
    normal = _run("normal", str(tmp_path / "normal.npz"))
    checked = _run("debug", str(tmp_path / "checked.npz"))
    assert sorted(normal.files) == sorted(checked.files)
    for k in normal.files:
        if k.endswith("_status"):
            assert int(checked[k]) == 0 and int(normal[k]) == 0, (k, int(normal[k]), int(checked[k]))
        else:
            assert np.array_equal(normal[k], checked[k]), k
