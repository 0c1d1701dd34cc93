"""Model-scale stacks on the GPU against the fp64 oracle.

* The 48-layer verify stack (2-bit blocks, d_model 2048, d_ff 768, 512 experts top-10 + shared,
  Zipf router bias, 8 tokens = 1 + 7 verify batch, ~36 GB resident), and the same stack in NVFP4
  blocks (~65 GB resident): every layer teacher-forced
  (the GPU's own input of the layer, captured through x_trace, fed to the oracle layer: expert
  sets, counts, max relative L2 <= 1e-3), and end to end from the same x over the first layers.
* The codebook (3.5-bit) configuration: independent model-scale layers applied to the same x, at
  1 and 8 tokens.
Near ties (oracle margin below 1e-4) are excluded from index parity and counted."""
import numpy as np
import pytest

import oracle
import synth
from helpers import (TOL_DECODE, TIE_EPS, compare_routing, moe_for, oracle_layer, rel_l2, route_buffers,
                     supply_from_generator, x_device, x_f64)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    import torch

    assert torch.cuda.is_available()
    return torch


def _load_stack(moe, wl, seed, layers):
    """Generate model-scale layers on the device (byte-identical to the CPU generator)."""
    import torch

    dev = torch.device("cuda")
    buf = torch.empty((wl.n_experts, wl.expert_bytes()), dtype=torch.uint8, device=dev)
    sh = torch.empty((1, wl.expert_bytes(shared=True)), dtype=torch.uint8, device=dev)
    for slot, l in enumerate(layers):
        for e0 in range(0, wl.n_experts, 128):
            ids = range(e0, min(wl.n_experts, e0 + 128))
            synth.gen_experts_torch(wl, seed, l, ids, buf[e0:e0 + len(ids)])
        synth.gen_experts_torch(wl, seed, l, [wl.n_experts], sh)
        router = synth.gen_router_torch(wl, seed, l, dev).contiguous()
        bias = torch.from_numpy(synth.gen_bias(wl, seed, l)).to(dev)
        moe.load_layer(slot, router, bias, buf, sh)
    torch.cuda.synchronize()
    del buf, sh


def _oracle_layer_for(wl, seed, l, x):
    L = oracle_layer(wl, seed, l, full=False)
    idx, _, _ = L.route(x)
    supply_from_generator(wl, seed)(l, L, sorted(set(idx.reshape(-1).tolist())))
    return L


@pytest.mark.parametrize("wl", [synth.VERIFY, synth.NVFP4], ids=lambda w: w.name)
def test_verify_stack_48_layers_model_scale(torch_cuda, wl):
    torch = torch_cuda
    nl, n, seed = wl.n_layers, wl.n_tokens, 0
    moe = moe_for(wl, nl, 8)
    _load_stack(moe, wl, seed, range(nl))
    x = x_device(wl, seed, n, pass_idx=3)
    out = torch.empty((n, wl.d_model), dtype=torch.float32, device="cuda")
    trace = torch.empty((nl, n, wl.d_model), dtype=torch.float32, device="cuda")
    routes = [route_buffers(n, wl.top_k, wl.n_experts) for _ in range(nl)]
    moe.forward_stack(0, nl, x, out, routes=routes, x_trace=trace)
    torch.cuda.synchronize()
    tr = trace.cpu().numpy().astype(np.float64)
    fin = out.cpu().numpy().astype(np.float64)
    x0 = x_f64(wl, x.view(torch.int16).cpu().numpy().view(np.uint16))
    assert np.array_equal(tr[0], x0)
    worst, excluded = 0.0, 0
    any_excl = np.zeros(n, dtype=bool)
    for l in range(nl):
        L = _oracle_layer_for(wl, seed, l, tr[l])
        ref = L.forward(tr[l])
        rb = {k: v.cpu().numpy() for k, v in routes[l].items()}
        bad, excl = compare_routing(rb["idx"], ref["idx"], ref["margin"], wl.n_experts, rb["counts"])
        assert bad == 0, f"layer {l}: routing mismatches on {bad} checks"
        keep = ref["margin"] >= TIE_EPS
        any_excl |= ~keep
        y_gpu = (tr[l + 1] if l + 1 < nl else fin) - tr[l]
        err = rel_l2(y_gpu, ref["y"], keep)
        assert err <= TOL_DECODE, f"layer {l}: teacher-forced max rel L2 {err:.3e}"
        worst, excluded = max(worst, err), excluded + excl
    # end to end from the same x: the oracle's own fp64 stack over the first layers
    n_e2e = 4
    ref_x, recs = oracle.stack_forward([(lambda l: oracle_layer(wl, seed, l, full=False))] * n_e2e, x0,
                                       supply=supply_from_generator(wl, seed))
    e2e_excl = np.zeros(n, dtype=bool)
    for r in recs:
        e2e_excl |= r["margin"] < TIE_EPS
    err_e2e = rel_l2(tr[n_e2e], ref_x, ~e2e_excl)
    print(f"{wl.name} 48 layers x 8 tokens: teacher-forced max rel L2 {worst:.3e}, excluded near "
          f"ties {excluded} (token-layers); end to end over {n_e2e} layers {err_e2e:.3e}")
    assert err_e2e <= TOL_DECODE
    moe.close()


def test_codebook_layers_model_scale(torch_cuda):
    """The codebook configuration: independent model-scale layers y_l = MoE_l(x) on the same x
    (layers 0, 1, 23 and 47 of the 48), at 1 and 8 tokens."""
    torch = torch_cuda
    wl = synth.CODEBOOK
    seed, layers = 0, (0, 1, 23, 47)
    moe = moe_for(wl, len(layers), 8)
    _load_stack(moe, wl, seed, layers)
    worst, excluded = 0.0, 0
    for n in (1, 8):
        x = x_device(wl, seed, n, pass_idx=n)
        xs = x_f64(wl, x.view(torch.int16).cpu().numpy().view(np.uint16))
        for slot, l in enumerate(layers):
            y = torch.empty((n, wl.d_model), dtype=torch.float32, device="cuda")
            rb = route_buffers(n, wl.top_k, wl.n_experts)
            moe.forward(slot, x, y, route=rb)
            torch.cuda.synchronize()
            L = _oracle_layer_for(wl, seed, l, xs)
            ref = L.forward(xs)
            rbn = {k: v.cpu().numpy() for k, v in rb.items()}
            bad, excl = compare_routing(rbn["idx"], ref["idx"], ref["margin"], wl.n_experts, rbn["counts"])
            assert bad == 0, f"layer {l}, {n} tokens: routing mismatches on {bad} checks"
            err = rel_l2(y.cpu().numpy(), ref["y"], ref["margin"] >= TIE_EPS)
            assert err <= TOL_DECODE, f"layer {l}, {n} tokens: max rel L2 {err:.3e}"
            worst, excluded = max(worst, err), excluded + excl
    print(f"codebook layers {layers} at 1 and 8 tokens: max rel L2 {worst:.3e}, excluded near ties {excluded}")
    moe.close()
