"""moe_route_noalloc: routing for callers that cannot allocate device memory where they route
(inside CUDA stream capture, under a runtime that plans all device memory itself, or in a loop
that must not take cudaMalloc's implicit synchronisation).  Its scratch is a static device array,
so this test checks, through the C ABI, that two calls in a row give the same experts and weights
as the routing step of moe_forward on the same inputs.  This file is collected last on purpose:
if it fails, a run that stops at the first failure has already run every other test."""
import ctypes as C

import numpy as np
import pytest

import synth
from helpers import load_layer_device, moe_for, route_buffers, x_device

pytestmark = pytest.mark.gpu


def _route_via_forward(torch, moe, wl, x):
    n = x.shape[0]
    y = torch.empty((n, wl.d_model), dtype=torch.float32, device="cuda")
    rb = route_buffers(n, wl.top_k, wl.n_experts)
    moe.forward(0, x, y, route=rb)
    torch.cuda.synchronize()
    return rb["idx"].cpu().numpy(), rb["w"].cpu().numpy()


def test_route_noalloc_matches_forward_routing_twice():
    import torch

    import expert_ffn_gemv_b200 as P

    wl = synth.small_workload(d_model=512, d_ff=128, n_experts=512, top_k=10, n_shared=1, shared_d_ff=128)
    seed = 11
    moe = moe_for(wl, 1, 8, seed=seed)
    load_layer_device(moe, 0, wl, seed, 0)
    dev = torch.device("cuda")
    router = synth.gen_router_torch(wl, seed, 0, dev).contiguous()
    bias = torch.from_numpy(synth.gen_bias(wl, seed, 0)).to(dev)
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call, (n, pass_idx) in enumerate(((8, 1), (5, 2))):  # two calls in a row, different inputs
        x = x_device(wl, seed, n, pass_idx)
        idx = torch.full((n, wl.top_k), -1, dtype=torch.int32, device=dev)
        w = torch.zeros((n, wl.top_k), dtype=torch.float32, device=dev)
        st = P.moe_route_noalloc(router.data_ptr(), P.MOE_BF16, bias.data_ptr(), wl.n_experts, wl.d_model,
                                 wl.top_k, x.data_ptr(), P.MOE_BF16, n, idx.data_ptr(), w.data_ptr(), stream)
        assert st == P.MOE_OK, f"call {call}: status {st}"
        torch.cuda.synchronize()
        ref_idx, ref_w = _route_via_forward(torch, moe, wl, x)
        got_idx, got_w = idx.cpu().numpy(), w.cpu().numpy()
        assert np.array_equal(got_idx, ref_idx), f"call {call}: experts differ"
        assert np.allclose(got_w, ref_w, rtol=1e-5, atol=1e-6), f"call {call}: weights differ"
        assert np.allclose(got_w.sum(1), 1.0, atol=1e-5)
    moe.close()


def test_route_noalloc_rejects_sizes_beyond_its_scratch():
    import torch

    import expert_ffn_gemv_b200 as P

    dev = torch.device("cuda")
    router = torch.zeros((2048, 512), dtype=torch.bfloat16, device=dev)
    x = torch.zeros((9, 512), dtype=torch.bfloat16, device=dev)
    idx = torch.zeros((9, 32), dtype=torch.int32, device=dev)
    w = torch.zeros((9, 32), dtype=torch.float32, device=dev)
    s = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    args = lambda e, d, k, n: (router.data_ptr(), P.MOE_BF16, None, e, d, k, x.data_ptr(), P.MOE_BF16, n,
                               idx.data_ptr(), w.data_ptr(), s)
    assert P.moe_route_noalloc(*args(512, 512, 10, 9)) == P.MOE_ERR_UNSUPPORTED   # > 8 tokens
    assert P.moe_route_noalloc(*args(2048, 512, 10, 8)) == P.MOE_ERR_UNSUPPORTED  # > 1024 experts
    assert P.moe_route_noalloc(*args(512, 512, 40, 8)) == P.MOE_ERR_UNSUPPORTED   # top_k > 32
    assert P.moe_route_noalloc(*args(512, 500, 10, 8)) == P.MOE_ERR_INVALID_ARGUMENT  # d_model % 128
    assert P.moe_route_noalloc(*args(512, 512, 0, 8)) == P.MOE_ERR_INVALID_ARGUMENT
