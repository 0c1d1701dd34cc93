"""The C ABI's error behaviour on the GPU: argument checks, unloaded layers, the allocation cap,
the bounded device wait (a flag nothing sets) and recovery afterwards."""
import ctypes as C

import numpy as np
import pytest

import synth
from helpers import load_layer_device, moe_for, x_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def P():
    import torch

    assert torch.cuda.is_available()
    import expert_ffn_gemv_b200 as P

    return P


def _cfg(P, **kw):
    base = dict(n_layers=1, d_model=256, d_ff=128, n_experts=16, top_k=2, n_shared=0, shared_d_ff=128,
                fmt=P.MOE_FMT_Q2_32, act_dtype=P.MOE_BF16, router_dtype=P.MOE_BF16, out_dtype=P.MOE_F32,
                max_tokens=8, codebook_grid=None, device=0, bias_mode=0, shared_gate=0)
    base.update(kw)
    return P.moe_config(C.sizeof(P.moe_config), *[base[k] for k in (
        "n_layers", "d_model", "d_ff", "n_experts", "top_k", "n_shared", "shared_d_ff", "fmt", "act_dtype",
        "router_dtype", "out_dtype", "max_tokens", "codebook_grid", "device", "bias_mode", "shared_gate")])


@pytest.mark.parametrize("bad", [dict(d_model=200), dict(d_ff=96), dict(top_k=0), dict(top_k=17),
                                 dict(n_shared=2), dict(fmt=7), dict(max_tokens=0), dict(max_tokens=9000),
                                 dict(fmt=1), dict(device=999), dict(n_experts=0), dict(bias_mode=2),
                                 dict(shared_gate=1), dict(shared_gate=2, n_shared=1)])
def test_create_rejects_bad_config(P, bad):
    h = C.c_void_p()
    assert P.lib().moe_create(C.byref(_cfg(P, **bad)), C.byref(h)) == P.MOE_ERR_INVALID_ARGUMENT
    assert not h.value


def test_create_rejects_wrong_struct_size(P):
    cfg = _cfg(P)
    cfg.struct_size = 12
    h = C.c_void_p()
    assert P.lib().moe_create(C.byref(cfg), C.byref(h)) == P.MOE_ERR_INVALID_ARGUMENT


def test_forward_errors_and_destroy_null(P):
    import torch

    assert P.moe_destroy(None) == P.MOE_OK
    h = P.moe_create(_cfg(P))
    x = torch.zeros((2, 256), dtype=torch.bfloat16, device="cuda")
    y = torch.zeros((2, 256), dtype=torch.float32, device="cuda")
    s = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert P.moe_forward(h, 0, x.data_ptr(), y.data_ptr(), 2, s) == P.MOE_ERR_NOT_LOADED
    assert P.moe_forward(h, 1, x.data_ptr(), y.data_ptr(), 2, s) == P.MOE_ERR_INVALID_ARGUMENT
    assert P.moe_forward(h, 0, x.data_ptr(), y.data_ptr(), 0, s) == P.MOE_ERR_INVALID_ARGUMENT
    assert P.moe_forward(h, 0, x.data_ptr(), y.data_ptr(), 9, s) == P.MOE_ERR_INVALID_ARGUMENT
    assert P.moe_forward(h, 0, None, y.data_ptr(), 2, s) == P.MOE_ERR_INVALID_ARGUMENT
    assert P.moe_forward_stack(h, 0, 2, x.data_ptr(), y.data_ptr(), 2, s) == P.MOE_ERR_INVALID_ARGUMENT
    assert P.moe_forward_stack(h, 0, 1, x.data_ptr(), x.data_ptr(), 2, s) == P.MOE_ERR_INVALID_ARGUMENT
    w = P.moe_layer_weights(None, None, None, None)
    assert P.moe_load_layer(h, 0, w, s) == P.MOE_ERR_INVALID_ARGUMENT
    assert "layer" in P.moe_last_error(h) or "weight" in P.moe_last_error(h)
    assert P.moe_destroy(h) == P.MOE_OK


def test_allocation_cap_gives_out_of_memory(P):
    wl = synth.small_workload(d_model=256, d_ff=128, n_experts=16, top_k=2, n_shared=0)
    moe = moe_for(wl, 1, 8)
    P.moe_debug_set_alloc_cap(moe.h, moe.device_bytes() + 1024)
    with pytest.raises(P.MoeError) as ei:
        load_layer_device(moe, 0, wl, 0, 0)
    assert ei.value.status == P.MOE_ERR_OUT_OF_MEMORY
    P.moe_debug_set_alloc_cap(moe.h, 0)
    load_layer_device(moe, 0, wl, 0, 0)  # works again without the cap
    moe.close()


def test_bounded_wait_times_out_and_context_survives(P):
    import torch

    wl = synth.small_workload(d_model=256, d_ff=128, n_experts=16, top_k=2, n_shared=0)
    moe = moe_for(wl, 1, 8)
    load_layer_device(moe, 0, wl, 0, 0)
    x = x_device(wl, 0, 3)
    y0 = torch.empty((3, 256), dtype=torch.float32, device="cuda")
    moe.forward(0, x, y0)
    P.moe_debug_set_spin_limit(moe.h, 20000)  # ~10 us
    s = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert P.moe_debug_wait_test(moe.h, s) == P.MOE_OK
    torch.cuda.synchronize()
    assert moe.check() == P.MOE_ERR_TIMEOUT
    assert moe.check() == P.MOE_OK  # cleared
    P.moe_debug_set_spin_limit(moe.h, 0)
    y1 = torch.empty_like(y0)
    moe.forward(0, x, y1)
    torch.cuda.synchronize()
    assert torch.equal(y0, y1)
    moe.close()


def test_reload_layer_replaces_weights(P):
    import torch

    wl = synth.small_workload(d_model=256, d_ff=128, n_experts=16, top_k=2)
    moe = moe_for(wl, 1, 8)
    x = x_device(wl, 1, 2)
    ya = torch.empty((2, 256), dtype=torch.float32, device="cuda")
    yb = torch.empty_like(ya)
    load_layer_device(moe, 0, wl, 1, 0)
    moe.forward(0, x, ya)
    load_layer_device(moe, 0, wl, 1, 1)
    moe.forward(0, x, yb)
    load_layer_device(moe, 0, wl, 1, 0)
    yc = torch.empty_like(ya)
    moe.forward(0, x, yc)
    torch.cuda.synchronize()
    assert not torch.equal(ya, yb) and torch.equal(ya, yc)
    moe.close()


def test_bf16_output(P):
    import torch

    wl = synth.small_workload(d_model=256, d_ff=128, n_experts=16, top_k=2)
    a = moe_for(wl, 1, 8)
    b = moe_for(wl, 1, 8, out_dtype=P.MOE_BF16)
    load_layer_device(a, 0, wl, 2, 0)
    load_layer_device(b, 0, wl, 2, 0)
    x = x_device(wl, 2, 4)
    yf = torch.empty((4, 256), dtype=torch.float32, device="cuda")
    yb = torch.empty((4, 256), dtype=torch.bfloat16, device="cuda")
    a.forward(0, x, yf)
    b.forward(0, x, yb)
    torch.cuda.synchronize()
    assert torch.equal(yf.to(torch.bfloat16), yb)
    a.close()
    b.close()
