"""Parity cases for the attention kernel on pairs of SMs, run in a process of their own
with WS_ATTENTION_KERNEL=pair (the kernel choice is read once per process).  Each case
compares the GPU output with the fp64 oracle at the stated tolerance and checks that the
paired kernel ran.  Prints one line per case; exits non-zero on the first failure."""
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(HERE))
sys.path.insert(0, HERE)

import numpy as np  # noqa: E402

from gpu_util import ATOL_MAX, ATOL_MEAN, STRESSED_MAX, STRESSED_MEAN, half_ulp_bf16  # noqa: E402
from kv_cache_serving_ws_b200 import native as ws  # noqa: E402
from oracle import ws_oracle as orc  # noqa: E402
from test_gpu_attention import Pair, _times4  # noqa: E402
from test_gpu_masking import Pair as PoisonPair  # noqa: E402


def run(name, cfg, units, commit_skip=(), splits=0, layer=0, qs=None, tol=(ATOL_MAX, ATOL_MEAN)):
    p = Pair(cfg, seed=7)
    for u in units[:-1]:
        p.cond(u)
        if u not in commit_skip:
            p.commit(u)
    p.cond(units[-1])
    got, want = p.attend(layer, units[-1], q_scale=qs, splits=splits)
    kernel = ws.ws_profile_read(p.h)["last_kernel"]
    p.close()
    d = np.abs(got - want)
    bound = tol[0] + (half_ulp_bf16(want) if tol[0] > ATOL_MAX else 0.0)   # stressed: plus the output's rounding
    ok = kernel == 2 and np.all(np.isfinite(got)) and np.all(d <= bound) and d.mean() <= tol[1]
    print(f"{name}: kernel={kernel} max={d.max():.2e} mean={d.mean():.2e} {'ok' if ok else 'FAIL'}", flush=True)
    if not ok:
        sys.exit(1)


def poisoned_neighbour_rows():
    cfg = orc.Config(n_layers=1, n_heads=2, head_dim=128, n_video=120, n_audio=4, n_cond=40, history_units=3)
    p = PoisonPair(cfg, seed=131)
    for u in range(5):
        p.cond(u)
        p.commit(u, poison=(u == 1))
    p.cond(5)
    p.cond(6)
    got, want = p.attend(0, 6, 0)
    kernel = ws.ws_profile_read(p.h)["last_kernel"]
    p.close()
    d = np.abs(got - want)
    ok = kernel == 2 and np.all(np.isfinite(got)) and d.max() <= ATOL_MAX and d.mean() <= ATOL_MEAN
    print(f"stale poisoned rows after a run: kernel={kernel} max={d.max():.2e} {'ok' if ok else 'FAIL'}", flush=True)
    if not ok:
        sys.exit(1)


if __name__ == "__main__":
    assert os.environ.get("WS_ATTENTION_KERNEL") == "pair"
    C = orc.Config
    run("one pair, one item, 3 key tiles", C(1, 1, 128, 100, 4, 16, 2), list(range(3)), splits=1)
    run("one pair, 4 items in a row", C(1, 4, 128, 100, 4, 16, 2), list(range(3)), splits=1)
    run("ragged runs, a gap, an uncommitted unit", C(2, 3, 128, 130, 3, 5, 4), [0, 1, 2, 4, 5, 6],
        commit_skip=(5,), layer=1)
    run("same, 4 pairs per lane", C(2, 3, 128, 130, 3, 5, 4), [0, 1, 2, 4, 5, 6], commit_skip=(5,), splits=4,
        layer=1)
    run("stressed query (x4)", C(2, 3, 128, 130, 3, 5, 4), [0, 1, 2, 4, 5, 6], commit_skip=(5,), splits=1,
        qs=_times4, tol=(STRESSED_MAX, STRESSED_MEAN))
    run("two query blocks, 8 heads, all pairs", C(1, 8, 128, 300, 4, 32, 6), list(range(7)))
    run("long items merged inside the kernel", C(1, 1, 128, 250, 6, 0, 511), list(range(512)), splits=12)
    poisoned_neighbour_rows()
    print("all ok")
