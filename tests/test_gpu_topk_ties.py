"""GPU parity of the decode router's top-k on exact ties, where the selection rule (descending
logit, equal logits in ascending expert index) decides every slot and no near-tie exclusion
applies.  A zero router makes every token's logits equal to the bias:

  * all_equal  -- every logit ties: more candidates than the rank-count pass takes, so the
                  round-based pass (warp argmax per selection) runs;
  * few_values -- four distinct bias values: the rank-count pass runs with ties among the
                  candidates.
Both at 128 experts (warp per token) and 1,000 (more than 512: the one-row pass).

Indices are compared in order, the softmax weights and the outputs against the oracle."""
import numpy as np
import pytest

import oracle
import synth
from helpers import TOL_DECODE, moe_for, rel_l2, route_buffers, x_device, x_f64

pytestmark = pytest.mark.gpu


def _bias(pattern: str, e: int) -> np.ndarray:
    if pattern == "all_equal":
        return np.zeros(e, dtype=np.float32)
    return (np.random.default_rng(3).integers(0, 4, e) * 0.25).astype(np.float32)


@pytest.mark.parametrize("pattern", ["all_equal", "few_values"])
@pytest.mark.parametrize("n", [1, 8])
@pytest.mark.parametrize("n_experts", [128, 1000])
def test_topk_exact_ties(pattern, n, n_experts):
    import torch

    assert torch.cuda.is_available()
    wl = synth.small_workload(d_model=256, d_ff=128, n_experts=n_experts, top_k=8, n_shared=1, shared_d_ff=128)
    seed = 11
    experts = synth.gen_layer_experts(wl, seed, 0)
    shared = synth.gen_shared(wl, seed, 0)
    router = np.zeros((wl.n_experts, wl.d_model), dtype=synth.gen_router(wl, seed, 0).dtype)
    bias = _bias(pattern, wl.n_experts)
    moe = moe_for(wl, 1, 8, seed=seed)
    moe.load_layer(0, router, bias, experts, shared)
    x = x_device(wl, seed, n)
    y = torch.empty((n, wl.d_model), dtype=torch.float32, device="cuda")
    rb = route_buffers(n, wl.top_k, wl.n_experts)
    moe.forward(0, x, y, route=rb)
    torch.cuda.synchronize()
    L = oracle.Layer(fmt=wl.fmt, d_model=wl.d_model, d_ff=wl.d_ff, n_experts=wl.n_experts, top_k=wl.top_k,
                     n_shared=wl.n_shared, shared_d_ff=wl.shared_d_ff, router_w=router,
                     router_dtype=wl.router_dtype, bias=bias, experts=experts, shared=shared)
    xs = x_f64(wl, x.view(torch.int16).cpu().numpy().view(np.uint16)
               if wl.act_dtype == synth.DT_BF16 else x.cpu().numpy())
    ref = L.forward(xs)
    idx = rb["idx"].cpu().numpy()
    assert np.array_equal(idx, ref["idx"]), (idx[0], ref["idx"][0])
    # the selection itself: the K largest biases, equal ones in ascending expert index
    order = np.lexsort((np.arange(wl.n_experts), -bias.astype(np.float64)))[:wl.top_k]
    assert np.array_equal(idx[0], order)
    assert np.allclose(rb["w"].cpu().numpy(), ref["w"], rtol=1e-5, atol=1e-6)
    assert np.array_equal(rb["counts"].cpu().numpy(), ref["counts"])
    assert rel_l2(y.cpu().numpy(), ref["y"]) <= TOL_DECODE
    moe.close()
