"""moe_route_noalloc: routing without a handle and without any device allocation, for callers
that cannot allocate device memory at the point where they route -- runtimes that plan every
byte of device memory up front and hand kernels only the buffers they planned, or loops that must
not take the device-wide synchronisation that cudaMalloc / cudaFree can imply.  Its only scratch
is a static device array of fixed size, so this file checks, through the C ABI:

  * two calls in a row give the same experts and weights as the routing step of moe_forward on
    the same inputs (and as the oracle), over router / input dtypes, with and without a bias, and
    with an expert count whose last router CTA is partly empty;
  * exact ties resolve to the lower expert index, and experts masked by a -inf bias are taken
    only after every finite logit, with weight 0, in the same way as moe_forward;
  * sizes beyond the static array and a misaligned router pointer are rejected.

This file is collected last on purpose: if it fails, a run that stops at the first failure has
already run every other test."""
import ctypes as C

import numpy as np
import pytest

import oracle
import synth
from helpers import TIE_EPS, compare_routing, moe_for, route_buffers, x_device, x_f64

pytestmark = pytest.mark.gpu


def _stream(torch):
    return C.c_void_p(torch.cuda.current_stream().cuda_stream)


def _noalloc(torch, P, router, router_dtype, bias, wl, x, x_dtype):
    n = x.shape[0]
    dev = torch.device("cuda")
    idx = torch.full((n, wl.top_k), -1, dtype=torch.int32, device=dev)
    w = torch.zeros((n, wl.top_k), dtype=torch.float32, device=dev)
    st = P.moe_route_noalloc(router.data_ptr(), router_dtype, None if bias is None else bias.data_ptr(),
                             wl.n_experts, wl.d_model, wl.top_k, x.data_ptr(), x_dtype, n, idx.data_ptr(),
                             w.data_ptr(), _stream(torch))
    torch.cuda.synchronize()
    return st, idx.cpu().numpy(), w.cpu().numpy()


def _forward_routing(torch, moe, wl, x):
    n = x.shape[0]
    y = torch.empty((n, wl.d_model), dtype=torch.float32, device="cuda")
    rb = route_buffers(n, wl.top_k, wl.n_experts)
    moe.forward(0, x, y, route=rb)
    torch.cuda.synchronize()
    return rb["idx"].cpu().numpy(), rb["w"].cpu().numpy()


def _layer(torch, wl, seed, router_np, bias_np):
    """A handle whose layer 0 has the given router and bias (small experts; only routing is
    compared), plus the same router / bias on the device for the no-alloc call."""
    moe = moe_for(wl, 1, 8, seed=seed)
    moe.load_layer(0, router_np, bias_np, synth.gen_layer_experts(wl, seed, 0), synth.gen_shared(wl, seed, 0))
    dev = torch.device("cuda")
    if wl.router_dtype == synth.DT_BF16:
        router = torch.from_numpy(np.ascontiguousarray(router_np).view(np.int16)).to(dev).view(torch.bfloat16)
    else:
        router = torch.from_numpy(np.ascontiguousarray(router_np)).to(dev)
    bias = None if bias_np is None else torch.from_numpy(bias_np).to(dev)
    return moe, router.contiguous(), bias


@pytest.mark.parametrize("router_dtype", [synth.DT_BF16, synth.DT_F32])
@pytest.mark.parametrize("x_dtype", [synth.DT_BF16, synth.DT_F32])
@pytest.mark.parametrize("with_bias", [True, False])
@pytest.mark.parametrize("n_experts", [512, 500])
def test_route_noalloc_matches_forward_and_oracle_twice(router_dtype, x_dtype, with_bias, n_experts):
    import torch

    import expert_ffn_gemv_b200 as P

    wl = synth.small_workload(d_model=512, d_ff=128, n_experts=n_experts, top_k=10, n_shared=1, shared_d_ff=128,
                              router_dtype=router_dtype, act_dtype=x_dtype, zipf_bias=with_bias)
    seed = 11
    router_np = synth.gen_router(wl, seed, 0)
    bias_np = synth.gen_bias(wl, seed, 0)
    moe, router, bias = _layer(torch, wl, seed, router_np, bias_np)
    L = oracle.Layer(fmt=wl.fmt, d_model=wl.d_model, d_ff=wl.d_ff, n_experts=wl.n_experts, top_k=wl.top_k,
                     n_shared=0, shared_d_ff=wl.shared_d_ff, router_w=router_np, router_dtype=wl.router_dtype,
                     bias=bias_np)
    for call, (n, pass_idx) in enumerate(((8, 1), (5, 2))):  # two calls in a row, different inputs
        x = x_device(wl, seed, n, pass_idx)
        st, got_idx, got_w = _noalloc(torch, P, router, router_dtype, bias, wl, x, x_dtype)
        assert st == P.MOE_OK, f"call {call}: status {st}"
        ref_idx, ref_w = _forward_routing(torch, moe, wl, x)
        assert np.array_equal(got_idx, ref_idx), f"call {call}: experts differ from moe_forward"
        assert np.allclose(got_w, ref_w, rtol=1e-5, atol=1e-6), f"call {call}: weights differ from moe_forward"
        assert np.allclose(got_w.sum(1), 1.0, atol=1e-5)
        xs = x_f64(wl, x.view(torch.int16).cpu().numpy().view(np.uint16) if x_dtype == synth.DT_BF16
                   else x.cpu().numpy())
        o_idx, o_w, margin = L.route(xs)
        bad, _ = compare_routing(got_idx, o_idx, margin, wl.n_experts)
        assert bad == 0, f"call {call}: experts differ from the oracle"
        for t in np.nonzero(margin >= TIE_EPS)[0]:
            order = {e: j for j, e in enumerate(o_idx[t])}
            assert np.allclose(got_w[t], [o_w[t][order[e]] for e in got_idx[t]], rtol=1e-5, atol=1e-6)
    moe.close()


@pytest.mark.parametrize("pattern", ["all_equal", "few_values", "masked"])
def test_route_noalloc_ties_and_masked_experts(pattern):
    """A zero router makes every logit equal to the bias.  all_equal / few_values: exact ties,
    resolved to the lower expert index (indices compared in order with the oracle and with
    moe_forward).  masked: a -inf bias on all but five experts with top-8, so three masked
    experts are taken after the finite ones, lowest index first, with weight 0."""
    import torch

    import expert_ffn_gemv_b200 as P

    wl = synth.small_workload(d_model=256, d_ff=128, n_experts=128, top_k=8, n_shared=1, shared_d_ff=128)
    seed = 11
    router_np = np.zeros((wl.n_experts, wl.d_model), dtype=np.uint16)
    rng = np.random.default_rng(3)
    if pattern == "all_equal":
        bias_np = np.zeros(wl.n_experts, dtype=np.float32)
    elif pattern == "few_values":
        bias_np = (rng.integers(0, 4, wl.n_experts) * 0.25).astype(np.float32)
    else:
        bias_np = np.full(wl.n_experts, -np.inf, dtype=np.float32)
        live = np.sort(rng.choice(wl.n_experts, 5, replace=False))
        bias_np[live] = np.array([0.5, -0.25, 1.0, 0.0, 0.75], dtype=np.float32)
    moe, router, bias = _layer(torch, wl, seed, router_np, bias_np)
    x = x_device(wl, seed, 8)
    for _ in range(2):
        st, got_idx, got_w = _noalloc(torch, P, router, P.MOE_BF16, bias, wl, x, P.MOE_BF16)
        assert st == P.MOE_OK
        ref_idx, ref_w = _forward_routing(torch, moe, wl, x)
        assert np.array_equal(got_idx, ref_idx)
        assert np.allclose(got_w, ref_w, rtol=1e-6, atol=0)
        order = np.lexsort((np.arange(wl.n_experts), -bias_np.astype(np.float64)))[:wl.top_k]
        assert all(np.array_equal(row, order) for row in got_idx)
        if pattern == "masked":
            assert np.all(got_w[:, 5:] == 0.0) and np.allclose(got_w.sum(1), 1.0, atol=1e-6)
            assert set(order[:5].tolist()) == set(live.tolist())
        else:
            L = oracle.Layer(fmt=wl.fmt, d_model=wl.d_model, d_ff=wl.d_ff, n_experts=wl.n_experts,
                             top_k=wl.top_k, n_shared=0, shared_d_ff=wl.shared_d_ff, router_w=router_np,
                             router_dtype=wl.router_dtype, bias=bias_np)
            xs = x_f64(wl, x.view(torch.int16).cpu().numpy().view(np.uint16))
            o_idx, o_w, _ = L.route(xs)
            assert np.array_equal(got_idx, o_idx)
            assert np.allclose(got_w, o_w, rtol=1e-5, atol=1e-6)
    moe.close()


def test_route_noalloc_rejects_sizes_beyond_its_scratch():
    import torch

    import expert_ffn_gemv_b200 as P

    dev = torch.device("cuda")
    router = torch.zeros((2048 * 512 + 64,), dtype=torch.bfloat16, device=dev)
    x = torch.zeros((9, 512), dtype=torch.bfloat16, device=dev)
    idx = torch.zeros((9, 32), dtype=torch.int32, device=dev)
    w = torch.zeros((9, 32), dtype=torch.float32, device=dev)
    s = _stream(torch)
    args = lambda e, d, k, n, r=router.data_ptr(): (r, P.MOE_BF16, None, e, d, k, x.data_ptr(), P.MOE_BF16, n,
                                                     idx.data_ptr(), w.data_ptr(), s)
    assert P.moe_route_noalloc(*args(512, 512, 10, 9)) == P.MOE_ERR_UNSUPPORTED   # > 8 tokens
    assert P.moe_route_noalloc(*args(2048, 512, 10, 8)) == P.MOE_ERR_UNSUPPORTED  # > 1024 experts
    assert P.moe_route_noalloc(*args(512, 512, 40, 8)) == P.MOE_ERR_UNSUPPORTED   # top_k > 32
    assert P.moe_route_noalloc(*args(512, 500, 10, 8)) == P.MOE_ERR_INVALID_ARGUMENT  # d_model % 128
    assert P.moe_route_noalloc(*args(512, 512, 0, 8)) == P.MOE_ERR_INVALID_ARGUMENT
    # the router rows are read 16 bytes at a time: a router pointer off a 16-byte boundary
    # (a view starting at an odd element) is rejected instead of faulting
    assert P.moe_route_noalloc(*args(512, 512, 10, 8, router.data_ptr() + 2)) == P.MOE_ERR_INVALID_ARGUMENT
    assert P.moe_route_noalloc(*args(512, 512, 10, 8, router.data_ptr() + 16)) == P.MOE_OK
    torch.cuda.synchronize()
