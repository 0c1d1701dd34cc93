"""Helpers shared by the parity tests: build layers from the seeded generators, run the fp64
oracle on the same bytes, and compare with the tolerance rules of the method.

Comparison rules
  * expert indices are compared as sets per token, bit-exactly, except for tokens whose
    oracle margin l_(k) - l_(k+1) is below 1e-4 (near ties, counted and reported);
  * per-expert token counts are compared over the non-excluded tokens;
  * outputs: per token ||y - y_ref|| / ||y_ref||, max over tokens, at most 1e-3 on the
    decode / verify (fp32-accumulate) path and 2e-2 on the bf16-operand prefill path.
"""
from __future__ import annotations

import numpy as np

import oracle
import synth

TIE_EPS = 1e-4
TOL_DECODE = 1e-3
TOL_PREFILL = 2e-2


def oracle_layer(wl: synth.Workload, seed: int, layer: int, full: bool = True, grid=None) -> oracle.Layer:
    """The oracle's view of one generated layer (all experts, or none for lazy supply)."""
    if grid is None and wl.fmt == synth.FMT_CB35:
        grid = synth.gen_grid(wl, seed)
    return oracle.Layer(
        fmt=wl.fmt, d_model=wl.d_model, d_ff=wl.d_ff, n_experts=wl.n_experts, top_k=wl.top_k,
        n_shared=wl.n_shared, shared_d_ff=wl.shared_d_ff, router_w=synth.gen_router(wl, seed, layer),
        router_dtype=wl.router_dtype, bias=synth.gen_bias(wl, seed, layer),
        experts=synth.gen_layer_experts(wl, seed, layer) if full else None,
        shared=synth.gen_shared(wl, seed, layer), grid=grid, shared_gate=synth.gen_shared_gate(wl, seed, layer),
        bias_mode=oracle.BIAS_SELECT if wl.bias_select else oracle.BIAS_LOGIT)


def supply_from_generator(wl: synth.Workload, seed: int, layer_of=lambda l: l):
    """Hook for oracle.stack_forward: generate the needed experts of layer l on the CPU."""

    def supply(l, L, need):
        for e in need:
            if e not in L._experts:
                L.set_expert(e, synth.gen_expert(wl, seed, layer_of(l), e))

    return supply


def x_f64(wl: synth.Workload, x_bits) -> np.ndarray:
    return oracle.to_f64(x_bits, wl.act_dtype)


def rel_l2(y, y_ref, mask=None) -> float:
    y = np.asarray(y, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    num = np.linalg.norm(y - y_ref, axis=-1)
    den = np.maximum(np.linalg.norm(y_ref, axis=-1), 1e-30)
    r = num / den
    if mask is not None:
        r = r[mask]
    return float(r.max()) if r.size else 0.0


def compare_routing(idx_gpu, idx_ref, margin, n_experts, counts_gpu=None, eps=TIE_EPS):
    """Returns (n_mismatch, n_excluded).

    * expert sets are compared per non-excluded token (oracle margin >= eps);
    * per-expert token counts are compared over the non-excluded tokens (the GPU's rows of
      those tokens against the oracle's), whatever the number of excluded tokens;
    * ``counts_gpu`` (the GPU's expert_counts output over all tokens of the call) must equal
      the histogram of the GPU's own index rows.
    Every failed check adds one to n_mismatch."""
    idx_gpu = np.asarray(idx_gpu)
    idx_ref = np.asarray(idx_ref)
    keep = np.asarray(margin) >= eps
    bad = 0
    for t in range(idx_ref.shape[0]):
        if keep[t] and set(idx_gpu[t].tolist()) != set(idx_ref[t].tolist()):
            bad += 1
    kept_gpu = np.bincount(idx_gpu[keep].reshape(-1), minlength=n_experts)
    kept_ref = np.bincount(idx_ref[keep].reshape(-1), minlength=n_experts)
    if not np.array_equal(kept_gpu, kept_ref):
        bad += 1
    if counts_gpu is not None:
        own = np.bincount(idx_gpu.reshape(-1), minlength=n_experts)
        if not np.array_equal(np.asarray(counts_gpu), own):
            bad += 1
    return bad, int((~keep).sum())


def moe_for(wl: synth.Workload, n_layers: int, max_tokens: int, seed: int = 0, out_dtype=None):
    import expert_ffn_gemv_b200 as P

    grid = synth.gen_grid(wl, seed) if wl.fmt == synth.FMT_CB35 else None
    return P.MoE(n_layers=n_layers, d_model=wl.d_model, d_ff=wl.d_ff, n_experts=wl.n_experts, top_k=wl.top_k,
                 n_shared=wl.n_shared, shared_d_ff=wl.shared_d_ff, fmt=wl.fmt, act_dtype=wl.act_dtype,
                 router_dtype=wl.router_dtype, out_dtype=P.MOE_F32 if out_dtype is None else out_dtype,
                 max_tokens=max_tokens, codebook_grid=grid, device=0,
                 bias_mode=P.MOE_BIAS_SELECT if wl.bias_select else P.MOE_BIAS_LOGIT, shared_gate=int(wl.shared_gate))


def load_layer_host(moe, slot: int, wl: synth.Workload, seed: int, layer: int):
    """Load a generated layer from host (numpy) buffers."""
    experts = synth.gen_layer_experts(wl, seed, layer)
    router = np.ascontiguousarray(synth.gen_router(wl, seed, layer))
    bias = synth.gen_bias(wl, seed, layer)
    shared = synth.gen_shared(wl, seed, layer)
    moe.load_layer(slot, router, bias, experts, shared, synth.gen_shared_gate(wl, seed, layer))


def load_layer_device(moe, slot: int, wl: synth.Workload, seed: int, layer: int, chunk: int = 64):
    """Generate a layer on the device (torch, byte-identical to numpy) and load it from there."""
    import torch

    dev = torch.device("cuda")
    eb = wl.expert_bytes()
    blocks = torch.empty((wl.n_experts, eb), dtype=torch.uint8, device=dev)
    for e0 in range(0, wl.n_experts, chunk):
        ids = list(range(e0, min(wl.n_experts, e0 + chunk)))
        synth.gen_experts_torch(wl, seed, layer, ids, blocks[e0:e0 + len(ids)])
    shared = None
    if wl.n_shared:
        shared = torch.empty((1, wl.expert_bytes(shared=True)), dtype=torch.uint8, device=dev)
        synth.gen_experts_torch(wl, seed, layer, [wl.n_experts], shared)
    router = synth.gen_router_torch(wl, seed, layer, dev).contiguous()
    b = synth.gen_bias(wl, seed, layer)
    bias = None if b is None else torch.from_numpy(b).to(dev)
    gate = synth.gen_shared_gate_torch(wl, seed, layer, dev)
    moe.load_layer(slot, router, bias, blocks, shared, gate)
    torch.cuda.synchronize()
    del blocks, shared


def x_device(wl: synth.Workload, seed: int, n: int, pass_idx: int = 0):
    import torch

    return synth.gen_x_torch(wl, seed, n, pass_idx, torch.device("cuda")).contiguous()


def route_buffers(n: int, k: int, e: int):
    import torch

    return dict(idx=torch.full((n, k), -1, dtype=torch.int32, device="cuda"),
                w=torch.zeros((n, k), dtype=torch.float32, device="cuda"),
                counts=torch.full((e,), -1, dtype=torch.int32, device="cuda"))
