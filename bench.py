#!/usr/bin/env python
"""Benchmark of the routed mixture-of-experts FFN from low-bit blocks on B200.

Default workload (one JSON line on stdout, rank 0):
  verify-stack-48L-8tok-q2 -- 1 + 7 token verify batches through a 48-layer MoE-only stack
  (d_model 2048, expert d_ff 768, 512 routed experts top-10 + 1 shared expert, 2-bit Q2 blocks,
  ~36 GB resident in HBM), residual add between layers, no norm, fresh seeded x per pass.
  A step is one pass: 8 tokens through all 48 layers.  Every pass reads ~3.6 GB of distinct
  expert blocks, far more than the 126 MB L2, so no flush is needed between steps.

Also: --workload decode (1 token through 16 model-scale layers of seeds 0-15, one step = the 16
layers), --workload codebook (3.5-bit codebook blocks, 48 independent layers on the same x),
--workload prefill (1,180 / 8,192-token chunks through the stack, grouped GEMM path),
--workload nvfp4 (the verify stack with NVFP4 blocks: E2M1 weights, E4M3 block scales, fp32
tensor scale per matrix).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload verify|nvfp4|decode|codebook|prefill]
  python bench.py --impl reference ...   # the fp64 CPU oracle on a bounded sample, same metric

Multi-GPU: replicas only (each rank holds the full stack and its own token stream; no
collective on the data path); time = max over ranks, value = all ranks' tokens / that time.
"""
from __future__ import annotations

import argparse
import ctypes as C
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time
from pathlib import Path

import numpy as np

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

import synth  # noqa: E402

METRIC = "routed-MoE tokens/s (48-layer stack); decode HBM GB/s; prefill TFLOP/s"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------------------------------ utilities
def peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = Path(os.environ.get("TMPDIR", "/tmp")) / f"clocks_{os.getpid()}.csv"

    def __enter__(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None or not self.path.exists():
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.path.read_text().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "samples": len(sm), "reasons": sorted(reasons)}


def source_hash(*files) -> str:
    h = hashlib.sha256()
    for f in files:
        h.update((ROOT / f).read_bytes())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str, src_hash: str, algorithmic_bytes: float):
    """DRAM bytes per launch of `kernel`: the committed ncu summary's measured ratio of DRAM bytes
    (read + write) to the captured launch's algorithmic bytes, times this run's algorithmic bytes
    per launch -- if the summary was taken on the current kernel source (else None)."""
    p = ROOT / "profiles" / f"{kernel}_{workload}.md"
    if not p.exists():
        return None
    t = p.read_text()
    m = re.search(r"source_hash:\s*([0-9a-f]+)", t)
    r = re.search(r"dram_over_algorithmic:\s*([0-9.eE+]+)", t)
    if not m or not r or m.group(1) != src_hash:
        return None
    return float(r.group(1)) * algorithmic_bytes


# ------------------------------------------------------------------------------------ distributed
def dist_setup(n_gpus, backend="nccl"):
    """One process per GPU: RANK / LOCAL_RANK / WORLD_SIZE come from the launcher, and WORLD_SIZE
    must equal --gpus (a mismatch is an error, not a silent 1-GPU run)."""
    import torch

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus:
        raise SystemExit(f"bench.py: --gpus {n_gpus} but WORLD_SIZE={world}")
    if world > 1:
        import datetime

        import torch.distributed as dist

        kw = dict(device_id=torch.device("cuda", local)) if backend == "nccl" else {}
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=600), **kw)
    if backend == "nccl":
        torch.cuda.set_device(local)
    return rank, world, local


def relaunch(n_gpus) -> int:
    """--gpus N > 1 without a launcher: run this command again under torch.distributed.run with
    N processes on this node (rendezvous on 127.0.0.1); rank 0 prints the JSON line."""
    import socket

    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        port = so.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n_gpus}",
           "--master-addr", "127.0.0.1", "--master-port", str(port), str(Path(__file__).resolve()), *sys.argv[1:]]
    return subprocess.run(cmd).returncode


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def _reduce_device():
    import torch
    import torch.distributed as dist

    return torch.device("cuda") if dist.get_backend() == "nccl" else torch.device("cpu")


def max_over_ranks(v: float, world: int) -> float:
    """Max of a per-rank value (the job's time is the slowest rank's)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist

    t = torch.tensor([v], dtype=torch.float64, device=_reduce_device())
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(v: float, world: int) -> float:
    """Sum of a per-rank value (tokens processed by all replicas)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist

    t = torch.tensor([v], dtype=torch.float64, device=_reduce_device())
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# ------------------------------------------------------------------------------------ model setup
def load_stack(moe, wl, seed, layers, layer_of=lambda i: i, chunk=128):
    """Generate each layer on the device (seeded hash, byte-identical to the CPU generator) and
    load it through moe_load_layer from device memory."""
    import torch

    dev = torch.device("cuda")
    buf = torch.empty((wl.n_experts, wl.expert_bytes()), dtype=torch.uint8, device=dev)
    sh = torch.empty((1, wl.expert_bytes(shared=True)), dtype=torch.uint8, device=dev) if wl.n_shared else None
    for i in range(layers):
        l = layer_of(i)
        s = seed if not isinstance(seed, (list, tuple)) else seed[i]
        for e0 in range(0, wl.n_experts, chunk):
            ids = range(e0, min(wl.n_experts, e0 + chunk))
            synth.gen_experts_torch(wl, s, l, ids, buf[e0:e0 + len(ids)])
        if sh is not None:
            synth.gen_experts_torch(wl, s, l, [wl.n_experts], sh)
        router = synth.gen_router_torch(wl, s, l, dev).contiguous()
        b = synth.gen_bias(wl, s, l)
        bias = None if b is None else torch.from_numpy(b).to(dev)
        moe.load_layer(i, router, bias, buf, sh)
    torch.cuda.synchronize()
    del buf, sh


def make_moe(wl, n_layers, max_tokens, seed=0):
    import expert_ffn_gemv_b200 as P

    grid = synth.gen_grid(wl, seed) if wl.fmt == synth.FMT_CB35 else None
    return P.MoE(n_layers=n_layers, d_model=wl.d_model, d_ff=wl.d_ff, n_experts=wl.n_experts, top_k=wl.top_k,
                 n_shared=wl.n_shared, shared_d_ff=wl.shared_d_ff, fmt=wl.fmt, act_dtype=wl.act_dtype,
                 router_dtype=wl.router_dtype, out_dtype=P.MOE_F32, max_tokens=max_tokens, codebook_grid=grid,
                 device=0 if "LOCAL_RANK" not in os.environ else int(os.environ["LOCAL_RANK"]))


# ------------------------------------------------------------------------------------ CPU oracle
def oracle_sample_stack(wl, seed, n_tokens, n_layers_sample, pass_idx=0, threads=0):
    """Time the fp64 oracle on n_tokens through the first n_layers_sample layers (generation of
    the sampled layers' bytes is outside the timed part).  Returns (seconds, threads used)."""
    import oracle

    sys.path.insert(0, str(ROOT / "tests"))
    from helpers import oracle_layer, supply_from_generator

    x = oracle.to_f64(synth.gen_x(wl, seed, n_tokens, pass_idx), wl.act_dtype)
    total = 0.0
    for l in range(n_layers_sample):
        L = oracle_layer(wl, seed, l, full=False)
        idx, _, _ = L.route(x)
        supply_from_generator(wl, seed)(l, L, sorted(set(idx.reshape(-1).tolist())))
        t0 = time.perf_counter()
        r = L.forward(x, n_threads=threads)
        total += time.perf_counter() - t0
        x = x + r["y"]
    used = min(n_tokens, threads if threads > 0 else oracle.max_threads())
    return total, used


# ------------------------------------------------------------------------------------ verify stack
WEIGHTS_DESC = {synth.FMT_Q2: "Q2 2-bit blocks, 10 B / 32 weights",
                synth.FMT_CB35: "CB35 3.5-bit codebook blocks, 14 B / 32 weights",
                synth.FMT_NVFP4: "NVFP4 blocks (E2M1 x E4M3 scale, 9 B / 16 weights, fp32 tensor scale per matrix)"}
GEMV_DTYPE = {synth.FMT_Q2: "q2 blocks x int16 acts (dp2a, i32) -> f32 accumulate",
              synth.FMT_CB35: "cb35 blocks x int16 acts (dp2a, i32) -> f32 accumulate",
              synth.FMT_NVFP4: "nvfp4 (2 x e2m1 int8) x int16 acts (dp2a, i32) -> f32 accumulate"}


def verify_config(wl, L):
    """The workload description both arms print (static: identical in the reference arm)."""
    return {"workload": wl.name, "d_model": wl.d_model, "d_ff": wl.d_ff, "n_experts": wl.n_experts,
            "top_k": wl.top_k, "n_shared": wl.n_shared, "layers": L, "tokens_per_pass": wl.n_tokens,
            "weights": WEIGHTS_DESC[wl.fmt], "router_bias": "Zipf(1.1), beta 0.5",
            "l2": "inputs larger than L2: each pass reads several GB of distinct expert blocks (126 MB L2)",
            "parallelism": "replicas (one process per GPU, no data-path collective)"}


def near_ties(wl, seed, trace):
    """Near ties of one pass, counted as the parity rule counts them: for each layer, the oracle's
    router margin l_(k) - l_(k+1) on the GPU's own input of that layer (teacher-forced); a token
    whose margin is below 1e-4 would be excluded from index parity."""
    sys.path.insert(0, str(ROOT / "tests"))
    from helpers import TIE_EPS, oracle_layer

    per_layer = []
    for l in range(trace.shape[0]):
        _, _, m = oracle_layer(wl, seed, l, full=False).route(trace[l])
        per_layer.append(int((m < TIE_EPS).sum()))
    return {"excluded_token_layers": int(sum(per_layer)), "token_layers": int(trace.shape[0] * trace.shape[1]),
            "layers_with_ties": [l for l, c in enumerate(per_layer) if c],
            "rule": "oracle margin l_(k) - l_(k+1) < 1e-4 on the GPU's per-layer input (teacher-forced), "
                    "last timed pass"}


def bench_verify(args, rank, world, local):
    import torch

    import expert_ffn_gemv_b200 as P

    wl = synth.NVFP4 if args.workload == "nvfp4" else synth.VERIFY
    L = args.layers
    n = wl.n_tokens
    K, W = args.steps, args.warmup
    seed = args.seed
    moe = make_moe(wl, L, 8, seed)
    t0 = time.time()
    load_stack(moe, wl, seed, L)
    load_s = time.time() - t0
    dev = torch.device("cuda")
    # fresh x per pass; each rank its own token stream
    xs = torch.stack([synth.gen_x_torch(wl, seed, n, 1000 * rank + p, dev) for p in range(W + K)]).contiguous()
    x_in = torch.empty((n, wl.d_model), dtype=torch.bfloat16, device=dev)
    out = torch.empty((n, wl.d_model), dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream()
    # headline graph: one pass, no event nodes (an event between two kernels would split their
    # programmatic launch overlap)
    with torch.cuda.stream(stream):
        x_in.copy_(xs[0])
        moe.forward_stack(0, L, x_in, out)  # eager warm call
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream, capture_error_mode="thread_local"):
            moe.forward_stack(0, L, x_in, out)
        for p in range(W):
            x_in.copy_(xs[p])
            g.replay()
        stream.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        with torch.cuda.stream(stream):
            ev0.record(stream)
            for p in range(K):
                x_in.copy_(xs[W + p])
                g.replay()
            ev1.record(stream)
        stream.synchronize()
    torch.cuda.synchronize()
    barrier(world)
    ms_local = ev0.elapsed_time(ev1)
    ms = max_over_ranks(ms_local, world)
    # roofline kernel: a second graph of the same pass with event pairs around each expert-GEMV
    # launch (gate/up + down), replayed Kr times over the same inputs; durations of its last replay
    P.moe_profile_enable(moe.h, 1 << P.PROF_GATEUP)
    Kr = min(K, 32)
    with torch.cuda.stream(stream):
        g2 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g2, stream=stream, capture_error_mode="thread_local"):
            moe.forward_stack(0, L, x_in, out)
        for p in range(Kr):
            x_in.copy_(xs[W + p])
            g2.replay()
        stream.synchronize()
    st_, gu_ms, gu_cnt = P.moe_profile_read(moe.h, P.PROF_GATEUP)
    if st_ != P.MOE_OK:
        print(f"profile read: status {st_}: {P.moe_last_error(moe.h)}", file=sys.stderr)
    del g2
    # per-kernel breakdown of one eager (untimed) pass of the same input
    P.moe_profile_enable(moe.h, True)
    with torch.cuda.stream(stream):
        x_in.copy_(xs[W + K - 1])
        moe.forward_stack(0, L, x_in, out)
    stream.synchronize()
    kern = {}
    for kind, name in ((P.PROF_ROUTE, "k_route"), (P.PROF_GATEUP, "k_gemv"), (P.PROF_DOWN, "k_combine")):
        _, tot, cnt = P.moe_profile_read(moe.h, kind)
        kern[name] = (tot, cnt)
    P.moe_profile_enable(moe.h, False)
    # routing of every timed pass (deterministic: re-run eagerly, untimed) -> active experts
    counts = [torch.empty(wl.n_experts, dtype=torch.int32, device=dev) for _ in range(L)]
    routes = [dict(counts=c) for c in counts]
    u_all = np.zeros((K, L), dtype=np.int64)
    with torch.cuda.stream(stream):
        for p in range(K):
            x_in.copy_(xs[W + p])
            moe.forward_stack(0, L, x_in, out, routes=routes)
            u_all[p] = torch.stack([(c > 0).sum() for c in counts]).cpu().numpy()
    stream.synchronize()
    expert_bytes = wl.expert_bytes()
    mat_bytes = expert_bytes // 3
    # algorithmic bytes: every active expert's blocks (gate + up + down) + shared, + router
    router_bytes = wl.n_experts * wl.d_model * 2
    step_bytes = ((u_all + wl.n_shared) * expert_bytes).sum(axis=1) + L * router_bytes  # per pass
    gemv_bytes_last = float(((u_all[Kr - 1] + wl.n_shared) * expert_bytes).sum())  # input of g2's last replay

    tokens = K * n
    total_tokens = sum_over_ranks(tokens, world)
    value = total_tokens / (ms / 1e3)
    pk, pk_kind = peaks()
    hbm_peak = pk["hbm_gbs"]
    achieved = gemv_bytes_last / (gu_ms / 1e3) / 1e9 if gu_ms > 0 else None
    src = source_hash("expert_ffn_gemv_b200/csrc/decode.cu", "expert_ffn_gemv_b200/csrc/moe_internal.cuh")
    traffic = profiled_traffic("k_gemv", args.workload, src, gemv_bytes_last / max(gu_cnt, 1))
    res = {
        "metric": METRIC,
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": K,
        "warmup": W,
        "ms_per_step": ms / K,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": GEMV_DTYPE[wl.fmt],
        "data": "synthetic (seeded integer-hash generator, random-init weights)",
        "config": verify_config(wl, L),
        "resident_weight_gb": round(moe.device_bytes() / 1e9, 2),
        "distinct_block_gb_per_pass": round(float(step_bytes.mean()) / 1e9, 2),
        "launch": "one CUDA graph per pass (48 x 3 kernels, programmatic dependent launches)",
        "hbm": {"active_expert_and_router_bytes_per_step": float(step_bytes.mean()),
                "gbs": float(step_bytes.sum() / (ms_local / 1e3) / 1e9),
                "frac_of_measured_peak": float(step_bytes.sum() / (ms_local / 1e3) / 1e9 / hbm_peak),
                "mean_active_experts_per_layer": float(u_all.mean() + wl.n_shared)},
        "roofline": {"kernel": "k_gemv (gate/up + down)", "bound": "hbm", "achieved": achieved, "peak": hbm_peak,
                     "peak_kind": pk_kind, "unit": "GB/s",
                     "frac": achieved / hbm_peak if achieved else None, "traffic": traffic,
                     "algorithmic_bytes_per_launch": gemv_bytes_last / max(gu_cnt, 1),
                     "avg_launch_us": gu_ms / max(gu_cnt, 1) * 1e3},
        "kernels_eager_pass_us": {k: round(v[0] * 1e3, 2) for k, v in kern.items()},
        "gpu_launches": K * L * 3,
        "clocks": clk.summary(),
        "load_seconds": round(load_s, 1),
    }
    # ---- end to end through the C ABI with host buffers (pinned), copies inside the timed region
    if not args.no_e2e:
        xh = xs[W:W + K].cpu().pin_memory()
        oh = torch.empty((n, wl.d_model), dtype=torch.float32).pin_memory()
        Ke = min(K, args.e2e_steps)
        for p in range(2):
            moe.forward_stack(0, L, xh[p], oh)
        barrier(world)
        t0 = time.perf_counter()
        for p in range(Ke):
            moe.forward_stack(0, L, xh[p], oh)  # library stages H2D, runs, copies D2H, syncs
        el = time.perf_counter() - t0
        el = max_over_ranks(el, world)
        res["e2e"] = {"value": sum_over_ranks(Ke * n, world) / el, "unit": "tokens/s",
                      "h2d_bytes_per_step": n * wl.d_model * 2, "d2h_bytes_per_step": n * wl.d_model * 4,
                      "steps": Ke, "api": "moe_forward_stack(host x, host x_out)"}
    # ---- CPU baseline: the oracle on a bounded sample (rank 0, one GPU only)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        trace = torch.empty((L, n, wl.d_model), dtype=torch.float32, device=dev)
        with torch.cuda.stream(stream):
            x_in.copy_(xs[W + K - 1])
            moe.forward_stack(0, L, x_in, out, x_trace=trace)
        stream.synchronize()
        res["near_ties"] = near_ties(wl, seed, trace.cpu().numpy().astype(np.float64))
        nl = args.cpu_layers
        sec, used = oracle_sample_stack(wl, seed, n, nl, pass_idx=0)
        res["cpu_baseline"] = {"value": n * nl / sec / L, "unit": "tokens/s", "cores": used, "kind": "oracle",
                               "sample": f"{n} tokens through the first {nl} of {L} layers, fp64 C oracle "
                                         f"(OpenMP over tokens); tokens/s scaled to the {L}-layer stack"}
    moe.close()
    return res


# ------------------------------------------------------------------------------------ other workloads
def _graph_time(moe, step, prep, W, K, world, local, prof_kind):
    """Capture step() into a CUDA graph (with event pairs around kernel class prof_kind), replay W
    warm-up and K timed steps (prep(p) before each), return (ms total max over ranks, kernel ms,
    kernel launches of the last replay, clocks)."""
    import torch

    import expert_ffn_gemv_b200 as P

    stream = torch.cuda.Stream()
    P.moe_profile_enable(moe.h, 1 << prof_kind)
    with torch.cuda.stream(stream):
        prep(0)
        step()
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream, capture_error_mode="thread_local"):
            step()
        for p in range(W):
            prep(p)
            g.replay()
        stream.synchronize()
    barrier(world)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        with torch.cuda.stream(stream):
            ev0.record(stream)
            for p in range(K):
                prep(W + p)
                g.replay()
            ev1.record(stream)
        stream.synchronize()
    barrier(world)
    ms = max_over_ranks(ev0.elapsed_time(ev1), world)
    _, kms, kcnt = P.moe_profile_read(moe.h, prof_kind)
    P.moe_profile_enable(moe.h, False)
    del g
    return ms, kms, kcnt, clk.summary()


def _base_result(wl, world, K, W, ms, metric_unit, value):
    return {"metric": METRIC, "value": value, "unit": metric_unit, "n_gpus": world, "steps": K, "warmup": W,
            "ms_per_step": ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "data": "synthetic (seeded integer-hash generator, random-init weights)"}


def bench_decode_layers(args, rank, world, local):
    """1 token through 16 model-scale layers built from seeds 0-15 (one layer each); a step runs
    the 16 layers (y_i = MoE_i(x_i)); the 16 layers' ~0.27 GB of active blocks defeat the L2."""
    import torch

    import expert_ffn_gemv_b200 as P

    wl = synth.DECODE
    nl = 16
    moe = make_moe(wl, nl, 8)
    load_stack(moe, wl, list(range(nl)), nl, layer_of=lambda i: 0)
    dev = torch.device("cuda")
    xs = [synth.gen_x_torch(wl, s, 1, 0, dev).contiguous() for s in range(nl)]
    ys = torch.empty((nl, 1, wl.d_model), dtype=torch.float32, device=dev)

    def step():
        for i in range(nl):
            moe.forward(i, xs[i], ys[i])

    K, W = args.steps, args.warmup
    ms, kms, kcnt, clocks = _graph_time(moe, step, lambda p: None, W, K, world, local, P.PROF_GATEUP)
    counts = [torch.empty(wl.n_experts, dtype=torch.int32, device=dev) for _ in range(nl)]
    for i in range(nl):
        moe.forward(i, xs[i], ys[i], route=dict(counts=counts[i]))
    u = np.array([int((c > 0).sum()) for c in counts]) + wl.n_shared
    eb = wl.expert_bytes()
    step_bytes = float((u * eb).sum())
    pk, kind = peaks()
    gbs = step_bytes * K / (ms / 1e3) / 1e9
    res = _base_result(wl, world, K, W, ms, "GB/s", sum_over_ranks(gbs, world))
    res.update({"dtype": "q2 blocks x int16 acts (dp2a, i32) -> f32 accumulate",
                "config": {"workload": wl.name, "layers_per_step": nl, "seeds": "0-15", "tokens": 1,
                           "bytes": "active-expert blocks (routed + shared) per layer",
                           "l2": "16 distinct layers per step"},
                "tokens_per_s_one_layer": K * nl / (ms / 1e3),
                "us_per_layer": ms * 1e3 / (K * nl),
                "roofline": {"kernel": "k_gemv (gate/up + down)", "bound": "hbm", "unit": "GB/s", "peak": pk["hbm_gbs"],
                             "peak_kind": kind,
                             "achieved": step_bytes / (kms / 1e3) / 1e9 if kms else None,
                             "frac": step_bytes / (kms / 1e3) / 1e9 / pk["hbm_gbs"] if kms else None,
                             "avg_launch_us": kms / max(kcnt, 1) * 1e3},
                "hbm_frac_whole_layer": gbs / pk["hbm_gbs"], "clocks": clocks, "gpu_launches": K * nl * 3})
    moe.close()
    return res


def bench_codebook(args, rank, world, local):
    """3.5-bit codebook blocks: 1 and 8 tokens through 48 model-scale layers applied to the same x
    (no residual chain: the synthetic codebook weights make a norm-free chain overflow)."""
    import torch

    import expert_ffn_gemv_b200 as P

    wl = synth.CODEBOOK
    nl = args.layers
    moe = make_moe(wl, nl, 8)
    load_stack(moe, wl, args.seed, nl)
    dev = torch.device("cuda")
    K, W = args.steps, args.warmup
    out = {}
    pk, kind = peaks()
    for n in (1, 8):
        x = synth.gen_x_torch(wl, args.seed, n, 0, dev).contiguous()
        ys = torch.empty((nl, n, wl.d_model), dtype=torch.float32, device=dev)

        def step():
            for i in range(nl):
                moe.forward(i, x, ys[i])

        ms, kms, kcnt, clocks = _graph_time(moe, step, lambda p: None, W, K, world, local, P.PROF_GATEUP)
        counts = [torch.empty(wl.n_experts, dtype=torch.int32, device=dev) for _ in range(nl)]
        for i in range(nl):
            moe.forward(i, x, ys[i], route=dict(counts=counts[i]))
        u = np.array([int((c > 0).sum()) for c in counts]) + wl.n_shared
        eb = wl.expert_bytes()
        gbs = float((u * eb).sum()) * K / (ms / 1e3) / 1e9
        gb = float((u * eb).sum())
        out[n] = {"tokens_per_s": sum_over_ranks(n * K / (ms / 1e3), world), "ms_per_step": ms / K, "gbs": gbs,
                  "frac": gbs / pk["hbm_gbs"], "gemv_gbs": gb / (kms / 1e3) / 1e9 if kms else None,
                  "clocks": clocks}
    res = _base_result(wl, world, K, W, out[8]["ms_per_step"] * K, "tokens/s", out[8]["tokens_per_s"])
    res.update({"dtype": "cb35 blocks x int16 acts (dp2a, i32) -> f32 accumulate",
                "config": {"workload": wl.name, "layers": nl, "tokens": [1, 8], "chain": "independent layers"},
                "by_tokens": out, "gpu_launches": K * nl * 3,
                "roofline": {"kernel": "k_gemv (gate/up + down)", "bound": "hbm", "unit": "GB/s", "peak": pk["hbm_gbs"],
                             "peak_kind": kind, "achieved": out[8]["gemv_gbs"],
                             "frac": out[8]["gemv_gbs"] / pk["hbm_gbs"] if out[8]["gemv_gbs"] else None}})
    moe.close()
    return res


def bench_prefill(args, rank, world, local):
    """Prompt chunks (default 8,192 tokens; --chunk 1180 for the short one) through the 48-layer
    stack, grouped tensor-core path."""
    import torch

    import expert_ffn_gemv_b200 as P

    wl = synth.PREFILL
    nl, n = args.layers, args.chunk
    moe = make_moe(wl, nl, max(n, 9))
    load_stack(moe, wl, args.seed, nl)
    dev = torch.device("cuda")
    K, W = args.steps, args.warmup
    xs = torch.stack([synth.gen_x_torch(wl, args.seed, n, 1000 * rank + p, dev) for p in range(2)]).contiguous()
    x_in = torch.empty((n, wl.d_model), dtype=torch.bfloat16, device=dev)
    out = torch.empty((n, wl.d_model), dtype=torch.float32, device=dev)

    def step():
        moe.forward_stack(0, nl, x_in, out)

    ms, kms, kcnt, clocks = _graph_time(moe, step, lambda p: x_in.copy_(xs[p % 2]), W, K, world, local,
                                        P.PROF_GATEUP)
    rows = n * (wl.top_k + wl.n_shared)
    flop_gu = 2.0 * rows * 2 * wl.d_ff * wl.d_model        # per layer, gate + up
    flop_layer = 2.0 * rows * 3 * wl.d_ff * wl.d_model + 2.0 * n * wl.n_experts * wl.d_model
    # active experts of each layer (one eager pass of the last input, untimed)
    counts = [torch.empty(wl.n_experts, dtype=torch.int32, device=dev) for _ in range(nl)]
    x_in.copy_(xs[(W + K - 1) % 2])
    moe.forward_stack(0, nl, x_in, out, routes=[dict(counts=c) for c in counts])
    u = np.array([int((c > 0).sum()) for c in counts]) + wl.n_shared
    eb = wl.expert_bytes()
    # gate/up GEMM bytes per layer: the active experts' gate and up blocks, the grouped bf16 rows
    # in and the bf16 h rows out
    bytes_gu = float(((u * eb * 2) // 3).mean()) + rows * wl.d_model * 2 + rows * wl.d_ff * 2
    pk, kind = peaks()
    peak_burst = pk["bf16_tflops"]
    peak_sus = pk.get("bf16_tflops_sustained", peak_burst)
    tfl = flop_layer * nl * K / (ms / 1e3) / 1e12
    gu_tf = flop_gu * kcnt / (kms / 1e3) / 1e12 if kms else None
    gu_gbs = bytes_gu * kcnt / (kms / 1e3) / 1e9 if kms else None
    # arithmetic intensity of the gate/up GEMM against the ridge of the measured peaks: the
    # 8,192-token chunk is tensor-bound, the 1,180-token chunk HBM-bound
    intensity = flop_gu / bytes_gu
    ridge = peak_burst * 1e12 / (pk["hbm_gbs"] * 1e9)
    if intensity >= ridge:
        roof = {"kernel": "k_pf_gemm<gate/up>", "bound": "tensor", "unit": "TFLOP/s", "peak": peak_burst,
                "peak_kind": kind + " burst bf16", "achieved": gu_tf, "frac": gu_tf / peak_burst if gu_tf else None,
                "frac_of_sustained": gu_tf / peak_sus if gu_tf else None}
    else:
        roof = {"kernel": "k_pf_gemm<gate/up>", "bound": "hbm", "unit": "GB/s", "peak": pk["hbm_gbs"],
                "peak_kind": kind, "achieved": gu_gbs, "frac": gu_gbs / pk["hbm_gbs"] if gu_gbs else None,
                "tflops": gu_tf}
    src = source_hash("expert_ffn_gemv_b200/csrc/prefill.cu", "expert_ffn_gemv_b200/csrc/prefill.cuh",
                      "expert_ffn_gemv_b200/csrc/moe_internal.cuh")
    roof.update({"avg_launch_us": kms / max(kcnt, 1) * 1e3,
                 "traffic": profiled_traffic("k_pf_gemm", f"prefill{n}", src, bytes_gu),
                 "algorithmic_bytes_per_launch": bytes_gu, "flop_per_launch": flop_gu,
                 "intensity_flop_per_byte": intensity, "ridge_flop_per_byte": ridge})
    res = _base_result(wl, world, K, W, ms, "tokens/s", sum_over_ranks(n * K / (ms / 1e3), world))
    res.update({"dtype": "bf16 operands (dequantised q2), f32 accumulate (tcgen05)",
                "config": {"workload": wl.name, "layers": nl, "chunk_tokens": n,
                           "l2": "each chunk reads the whole 36 GB stack"},
                "tflops_whole_step": tfl, "frac_of_burst_peak_whole_step": tfl / peak_burst,
                "mean_active_experts_per_layer": float(u.mean()),
                "roofline": roof, "clocks": clocks, "gpu_launches": K * nl * 7})
    moe.close()
    return res


# ------------------------------------------------------------------------------------ reference arm
def bench_reference(args):
    """The fp64 CPU oracle as the reference arm: each step = 8 tokens through one layer of the
    48-layer verify stack (layer = step mod 48), timed on the host cores."""
    import oracle

    sys.path.insert(0, str(ROOT / "tests"))
    from helpers import oracle_layer, supply_from_generator

    wl = synth.NVFP4 if args.workload == "nvfp4" else synth.VERIFY
    L, n, seed = args.layers, wl.n_tokens, args.seed
    cache = {}

    def layer(l):
        if l not in cache:
            if len(cache) >= 4:
                cache.pop(next(iter(cache)))
            cache[l] = oracle_layer(wl, seed, l, full=False)
        return cache[l]

    x = oracle.to_f64(synth.gen_x(wl, seed, n, 0), wl.act_dtype)
    times = []
    for s in range(args.warmup + args.steps):
        l = s % L
        Ll = layer(l)
        idx, _, _ = Ll.route(x)
        supply_from_generator(wl, seed)(l, Ll, sorted(set(idx.reshape(-1).tolist())))
        t0 = time.perf_counter()
        Ll.forward(x)
        if s >= args.warmup:
            times.append(time.perf_counter() - t0)
    sec = sum(times)
    used = min(n, oracle.max_threads())
    value = n * len(times) / sec / L
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec / len(times) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded integer-hash generator)",
        "config": verify_config(wl, L),
        "step": "8 tokens through one layer (layer = step mod 48), scaled to the 48-layer stack",
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": used, "kind": "oracle",
                         "sample": f"{len(times)} steps of 8 tokens x 1 layer"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ------------------------------------------------------------------------------------ replica plumbing
def bench_plumbing(args, rank, world, local):
    """No GPU (gloo): the replica launch, the barriers and the max / sum over ranks, with a fixed
    host loop standing in for a step.  It checks the multi-process plumbing on a CPU machine and
    reports no GPU figure."""
    barrier(world)
    t0 = time.perf_counter()
    acc = 0
    for _ in range(args.steps):
        acc += sum(range(20000 * (rank + 1)))
    el_ms = (time.perf_counter() - t0) * 1e3
    barrier(world)
    ms = max_over_ranks(el_ms, world)
    tokens = sum_over_ranks(args.steps * 8, world)
    return {"metric": "replica plumbing check (host loop, no GPU)", "value": tokens / (ms / 1e3), "unit": "steps*8/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "rank_ms": el_ms, "total_tokens": tokens}


# ------------------------------------------------------------------------------------ main
def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=256)
    ap.add_argument("--warmup", type=int, default=8)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["verify", "nvfp4", "decode", "codebook", "prefill"], default="verify")
    ap.add_argument("--chunk", type=int, default=8192, help="prefill chunk tokens")
    ap.add_argument("--layers", type=int, default=48)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=64)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-layers", type=int, default=12)
    ap.add_argument("--plumbing-check", action="store_true",
                    help="no GPU: run only the replica launch / barrier / max-over-ranks logic (gloo)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(bench_reference(args)), flush=True)
        return 0
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        return relaunch(args.gpus)
    rank, world, local = dist_setup(args.gpus, "gloo" if args.plumbing_check else "nccl")
    fn = {"verify": bench_verify, "nvfp4": bench_verify, "decode": bench_decode_layers, "codebook": bench_codebook,
          "prefill": bench_prefill}[args.workload]
    if args.plumbing_check:
        fn = bench_plumbing
    res = fn(args, rank, world, local)
    if world > 1:
        import torch.distributed as dist

        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
