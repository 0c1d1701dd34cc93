"""Child process of test_gpu_route_modes.py: one model-scale decode layer (512 experts, d_model
2,048, top-10 + a shared expert, Q2 blocks) for 1, 3 and 8 tokens, each checked against the
oracle, and a two-layer stack call, under the router mode that MOE_ROUTE_CLUSTER selects (the
library reads it once per process).  Saves the outputs and the selections to the .npz named on
the command line."""
import sys
from pathlib import Path

HERE = Path(__file__).resolve().parent
sys.path[:0] = [str(HERE), str(HERE.parent)]

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synth  # noqa: E402
from helpers import load_layer_device, moe_for, x_device  # noqa: E402
from test_gpu_decode import _check_layer, _run_layer  # noqa: E402


def main(out: str) -> None:
    wl, seed = synth.VERIFY, 11
    moe = moe_for(wl, 2, 8, seed=seed)
    for layer in range(2):
        load_layer_device(moe, layer, wl, seed, layer)
    res = {}
    for n in (1, 3, 8):
        x, y, rb = _run_layer(torch, moe, wl, seed, n)
        err, excl = _check_layer(wl, seed, 0, x, y, rb)
        print(f"n={n}: max rel L2 {err:.3e} (excluded near ties {excl})")
        res[f"y{n}"], res[f"idx{n}"], res[f"w{n}"] = y, rb["idx"], rb["w"]
    # the second layer's router reads the first layer's fp32 output (the other x type)
    x = x_device(wl, seed, 8, 1)
    y = torch.empty((8, wl.d_model), dtype=torch.float32, device="cuda")
    moe.forward_stack(0, 2, x, y)
    torch.cuda.synchronize()
    res["stack"] = y.cpu().numpy()
    moe.close()
    np.savez(out, **res)


if __name__ == "__main__":
    main(sys.argv[1])
