"""The attention kernel on pairs of SMs (tcgen05.mma.cta_group::2), selected with
WS_ATTENTION_KERNEL=pair, against the fp64 oracle: several items per pair, ragged key
runs, forced splits, a stressed query, in-kernel merges of cut items and non-finite
values in rows past a run's end.  The cases run in a child process, because the
kernel choice is read once per process."""
import os
import subprocess
import sys

import pytest

from gpu_util import require_gpu

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.gpu
def test_pair_kernel_matches_the_oracle():
    require_gpu()
    env = dict(os.environ, WS_ATTENTION_KERNEL="pair")
    r = subprocess.run([sys.executable, os.path.join(HERE, "pair_kernel_cases.py")], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "all ok" in r.stdout, r.stdout
