"""GPU parity of the grouped tensor-core path (more than 8 tokens per call) against the fp64
oracle.  bf16 operands: max relative L2 error per token <= 2e-2; expert indices exact (near ties
excluded and counted)."""
import numpy as np
import pytest

import oracle
import synth
from helpers import (TOL_PREFILL, compare_routing, load_layer_device, moe_for, oracle_layer, rel_l2, route_buffers,
                     supply_from_generator, x_device, x_f64)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    import torch

    assert torch.cuda.is_available()
    return torch


def _forward(torch, moe, wl, seed, n, pass_idx=0):
    x = x_device(wl, seed, n, pass_idx)
    y = torch.empty((n, wl.d_model), dtype=torch.float32, device="cuda")
    rb = route_buffers(n, wl.top_k, wl.n_experts)
    moe.forward(0, x, y, route=rb)
    torch.cuda.synchronize()
    return x, y.cpu().numpy(), {k: v.cpu().numpy() for k, v in rb.items()}


def _check(torch, wl, seed, x, y, rb, L, sample=None, tol=TOL_PREFILL):
    xs = x_f64(wl, x.view(torch.int16).cpu().numpy().view(np.uint16)
               if wl.act_dtype == synth.DT_BF16 else x.cpu().numpy())
    rows = np.arange(xs.shape[0]) if sample is None else np.asarray(sample)
    if not L._experts:
        idx, _, _ = L.route(xs[rows])
        supply_from_generator(wl, seed)(0, L, sorted(set(idx.reshape(-1).tolist())))
    ref = L.forward(xs[rows])
    counts = rb["counts"] if sample is None else None
    bad, excl = compare_routing(rb["idx"][rows], ref["idx"], ref["margin"], wl.n_experts, counts)
    assert bad == 0, f"routing mismatches on {bad} tokens (excluded {excl})"
    keep = ref["margin"] >= 1e-4
    err = rel_l2(y[rows], ref["y"], keep)
    print(f"prefill n={xs.shape[0]} fmt={wl.fmt}: max rel L2 {err:.3e} over {keep.sum()} tokens, excluded {excl}")
    assert err <= tol
    return err


@pytest.mark.parametrize("fmt", [synth.FMT_Q2, synth.FMT_CB35, synth.FMT_NVFP4])
@pytest.mark.parametrize("n", [9, 37, 300])
def test_small_prefill(torch_cuda, fmt, n):
    """Ragged token counts: tiles of 128 rows, partial tiles, empty experts, the shared expert."""
    torch = torch_cuda
    wl = synth.small_workload(fmt=fmt, d_model=256, d_ff=256, n_experts=16, top_k=4, n_shared=1, shared_d_ff=128)
    moe = moe_for(wl, 1, 512, seed=2)
    load_layer_device(moe, 0, wl, 2, 0)
    x, y, rb = _forward(torch, moe, wl, 2, n)
    _check(torch, wl, 2, x, y, rb, oracle_layer(wl, 2, 0))
    moe.close()


def test_prefill_matches_decode_within_tolerance(torch_cuda):
    """The same tokens through both paths (8-token decode calls vs one 40-token call)."""
    torch = torch_cuda
    wl = synth.small_workload(d_model=512, d_ff=256, n_experts=32, top_k=4, n_shared=1, shared_d_ff=256)
    moe = moe_for(wl, 1, 64, seed=3)
    load_layer_device(moe, 0, wl, 3, 0)
    x = x_device(wl, 3, 40)
    yp = torch.empty((40, wl.d_model), dtype=torch.float32, device="cuda")
    moe.forward(0, x, yp)
    yd = torch.empty_like(yp)
    for i in range(0, 40, 8):
        moe.forward(0, x[i:i + 8].contiguous(), yd[i:i + 8])
    torch.cuda.synchronize()
    assert rel_l2(yp.cpu().numpy(), yd.cpu().numpy()) <= TOL_PREFILL
    # bit-reproducible
    yp2 = torch.empty_like(yp)
    moe.forward(0, x, yp2)
    torch.cuda.synchronize()
    assert torch.equal(yp, yp2)
    moe.close()


def _sample_tokens(idx_ref, keep, n_experts, rng, n_random):
    """Tokens to check against the oracle one by one: some of the largest expert group, some of
    experts holding 1-15 tokens (partial tiles), and a random draw."""
    n = idx_ref.shape[0]
    counts = np.bincount(idx_ref.reshape(-1), minlength=n_experts)
    big = int(np.argmax(counts))
    rows_big = np.nonzero((idx_ref == big).any(1))[0]
    small = np.nonzero((counts >= 1) & (counts <= 15))[0]
    rows_small = np.nonzero(np.isin(idx_ref, small).any(1))[0]
    pick = [rng.choice(rows_big, min(48, rows_big.size), replace=False)]
    if rows_small.size:
        pick.append(rng.choice(rows_small, min(64, rows_small.size), replace=False))
    pick.append(rng.choice(n, n_random, replace=False))
    rows = np.unique(np.concatenate(pick))
    return rows[keep[rows]], int(counts[big]), int(small.size)


@pytest.mark.parametrize("fmt,n", [(synth.FMT_Q2, 1180), (synth.FMT_Q2, 8192), (synth.FMT_CB35, 1180),
                                   (synth.FMT_NVFP4, 1180)])
def test_prefill_chunk_model_scale(torch_cuda, fmt, n):
    """A prompt chunk (1,180 or 8,192 tokens) through one model-scale layer (d_model 2048, d_ff
    768, 512 experts top-10 + shared, Zipf router bias): expert sets of every token and the
    per-expert counts of every non-excluded token against the oracle's routing, the GPU's counts
    against its own index rows, and the outputs of sampled tokens (the largest expert group,
    experts with 1-15 tokens, a random draw) against the oracle token by token."""
    torch = torch_cuda
    wl = {synth.FMT_Q2: synth.PREFILL, synth.FMT_CB35: synth.CODEBOOK, synth.FMT_NVFP4: synth.NVFP4}[fmt]
    moe = moe_for(wl, 1, 8192)
    load_layer_device(moe, 0, wl, 0, 0)
    x, y, rb = _forward(torch, moe, wl, 0, n, pass_idx=5)
    L = oracle_layer(wl, 0, 0, full=False)
    xs = x_f64(wl, x.view(torch.int16).cpu().numpy().view(np.uint16))
    idx_all, _, margin_all = L.route(xs)
    bad, excl = compare_routing(rb["idx"], idx_all, margin_all, wl.n_experts, rb["counts"])
    assert bad == 0, f"routing mismatches on {bad} checks (excluded near ties {excl})"
    keep = margin_all >= 1e-4
    rows, big, n_small = _sample_tokens(idx_all, keep, wl.n_experts, np.random.default_rng(n), 96)
    supply_from_generator(wl, 0)(0, L, sorted(set(idx_all[rows].reshape(-1).tolist())))
    ref = L.forward(xs[rows])
    err = rel_l2(y[rows], ref["y"])
    print(f"prefill chunk n={n} fmt={fmt}: routing of all tokens exact, excluded near ties {excl}; "
          f"max rel L2 {err:.3e} over {rows.size} sampled tokens (largest group {big} tokens, "
          f"{n_small} experts with 1-15 tokens)")
    assert err <= TOL_PREFILL
    moe.close()


@pytest.mark.parametrize("fmt", [synth.FMT_Q2, synth.FMT_CB35, synth.FMT_NVFP4])
def test_prefill_stack_teacher_forced(torch_cuda, fmt):
    torch = torch_cuda
    wl = synth.small_workload(fmt=fmt, d_model=256, d_ff=256, n_experts=16, top_k=4, n_shared=1, shared_d_ff=256)
    nl, n, seed = 2, 100, 6
    moe = moe_for(wl, nl, 128, seed=seed)
    for l in range(nl):
        load_layer_device(moe, l, wl, seed, l)
    x = x_device(wl, seed, n)
    out = torch.empty((n, wl.d_model), dtype=torch.float32, device="cuda")
    trace = torch.empty((nl, n, wl.d_model), dtype=torch.float32, device="cuda")
    routes = [route_buffers(n, wl.top_k, wl.n_experts) for _ in range(nl)]
    moe.forward_stack(0, nl, x, out, routes=routes, x_trace=trace)
    torch.cuda.synchronize()
    tr = trace.cpu().numpy().astype(np.float64)
    for l in range(nl):
        ref = oracle_layer(wl, seed, l).forward(tr[l])
        rb = {k: v.cpu().numpy() for k, v in routes[l].items()}
        bad, _ = compare_routing(rb["idx"], ref["idx"], ref["margin"], wl.n_experts)
        assert bad == 0
        y_gpu = (tr[l + 1] if l + 1 < nl else out.cpu().numpy().astype(np.float64)) - tr[l]
        assert rel_l2(y_gpu, ref["y"], ref["margin"] >= 1e-4) <= TOL_PREFILL
    moe.close()
