"""GPU parity of the two variants of the routed-MoE layer against the fp64 oracle:

  * selection-only router bias (the top-k of logit + bias, weighted by the softmax of the
    unbiased logits of the selected experts);
  * sigmoid-gated shared expert (o_shared scaled by sigmoid(g . x), g a d_model vector stored
    like a router row).

Both paths: the dequant-fused GEMV path (1-8 tokens, max relative L2 <= 1e-3) and the grouped
tensor-core path (more tokens, <= 2e-2); expert sets exact with near ties excluded and counted."""
import dataclasses

import numpy as np
import pytest

import synth
from helpers import (TIE_EPS, TOL_DECODE, TOL_PREFILL, compare_routing, load_layer_device, moe_for, oracle_layer,
                     rel_l2, route_buffers, supply_from_generator, x_device, x_f64)

pytestmark = pytest.mark.gpu

VARIANTS = [(True, False), (False, True), (True, True)]


def _ids(v):
    return {(True, False): "select_bias", (False, True): "gated_shared", (True, True): "both"}[v]


def _run_and_check(torch, wl, seed, n, tol, pass_idx=0, L=None, sample=None):
    moe = moe_for(wl, 1, max(n, 8), seed=seed)
    load_layer_device(moe, 0, wl, seed, 0)
    x = x_device(wl, seed, n, pass_idx)
    y = torch.empty((n, wl.d_model), dtype=torch.float32, device="cuda")
    rb = route_buffers(n, wl.top_k, wl.n_experts)
    moe.forward(0, x, y, route=rb)
    torch.cuda.synchronize()
    moe.close()
    y = y.cpu().numpy()
    rb = {k: v.cpu().numpy() for k, v in rb.items()}
    xs = x_f64(wl, x.view(torch.int16).cpu().numpy().view(np.uint16))
    if L is None:
        L = oracle_layer(wl, seed, 0)
    idx_all, w_all, margin = L.route(xs)
    bad, excl = compare_routing(rb["idx"], idx_all, margin, wl.n_experts, rb["counts"])
    assert bad == 0, f"routing mismatches on {bad} checks (excluded {excl})"
    keep = margin >= TIE_EPS
    for t in np.nonzero(keep)[0]:
        order = {e: j for j, e in enumerate(idx_all[t])}
        assert np.allclose(rb["w"][t], [w_all[t][order[e]] for e in rb["idx"][t]], rtol=1e-5, atol=1e-6)
    rows = np.nonzero(keep)[0] if sample is None else np.asarray([r for r in sample if keep[r]])
    if not L._experts:
        supply_from_generator(wl, seed)(0, L, sorted(set(idx_all[rows].reshape(-1).tolist())))
    ref = L.forward(xs[rows])
    err = rel_l2(y[rows], ref["y"])
    assert err <= tol, f"max rel L2 {err:.3e}"
    return err, excl


@pytest.mark.parametrize("variant", VARIANTS, ids=_ids)
@pytest.mark.parametrize("n", [1, 5, 8, 40, 300])
def test_variant_small_layer(variant, n):
    import torch

    bias_select, gate = variant
    wl = synth.small_workload(d_model=512, d_ff=256, n_experts=32, top_k=4, n_shared=1, shared_d_ff=256,
                              bias_select=bias_select, shared_gate=gate)
    _run_and_check(torch, wl, 21, n, TOL_DECODE if n <= 8 else TOL_PREFILL)


@pytest.mark.parametrize("fmt", [synth.FMT_Q2, synth.FMT_CB35, synth.FMT_NVFP4])
def test_variants_model_scale(fmt):
    """Both variants on one model-scale layer (d_model 2048, d_ff 768, 512 experts top-10 +
    shared, Zipf bias): an 8-token verify batch and a 1,180-token chunk (96 sampled tokens)."""
    import torch

    base = {synth.FMT_Q2: synth.VERIFY, synth.FMT_CB35: synth.CODEBOOK, synth.FMT_NVFP4: synth.NVFP4}[fmt]
    wl = dataclasses.replace(base, bias_select=True, shared_gate=True)
    err8, ex8 = _run_and_check(torch, wl, 0, 8, TOL_DECODE, pass_idx=8, L=oracle_layer(wl, 0, 0, full=False))
    sample = np.random.default_rng(4).choice(1180, 96, replace=False)
    errp, exp = _run_and_check(torch, wl, 0, 1180, TOL_PREFILL, pass_idx=9, L=oracle_layer(wl, 0, 0, full=False),
                               sample=sample)
    print(f"variants fmt={fmt}: 8 tokens max rel L2 {err8:.2e} (excluded {ex8}); 1,180-token chunk {errp:.2e} "
          f"(excluded {exp})")
