"""The decode router's launch modes at model scale, each against the oracle: 16-CTA clusters
with one token each (the default while the device holds a cluster per token), two tokens per
cluster (MOE_ROUTE_CLUSTER=2, the layout used when the tokens outnumber the resident clusters)
and the plain grid router (MOE_ROUTE_CLUSTER=0).  The library reads the variable once per
process, so every mode runs in a child process (route_mode_case.py)."""
import os
import subprocess
import sys
from pathlib import Path

import numpy as np
import pytest

pytestmark = pytest.mark.gpu
HERE = Path(__file__).resolve().parent


def _run(mode, out):
    env = dict(os.environ)
    env.pop("MOE_ROUTE_CLUSTER", None)
    if mode is not None:
        env["MOE_ROUTE_CLUSTER"] = mode
    r = subprocess.run([sys.executable, str(HERE / "route_mode_case.py"), str(out)], env=env, capture_output=True,
                       text=True, timeout=1200)
    assert r.returncode == 0, f"mode {mode}:\n{r.stdout[-3000:]}\n{r.stderr[-3000:]}"
    print(f"mode {mode}:\n{r.stdout}")
    return dict(np.load(out))


def test_router_modes(tmp_path):
    res = {m: _run(m, tmp_path / f"route_{m}.npz") for m in (None, "2", "0")}
    one, two, plain = res[None], res["2"], res["0"]
    for k in one:
        # one or two tokens per cluster: the same sums in the same order, bit for bit
        assert np.array_equal(one[k], two[k]), k
    for n in (1, 3, 8):
        assert np.array_equal(one[f"idx{n}"], plain[f"idx{n}"])
