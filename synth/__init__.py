"""Seeded synthetic inputs for the routed mixture-of-experts FFN workloads.

This module only draws numbers and packs bytes; it holds none of the method's
arithmetic (no dequantisation, no routing, no expert math).  It serves two
independent consumers: the fp64 CPU oracle (numpy arrays) and the CUDA path
(torch tensors on the device).  Every value is a pure function of
(seed, workload id, layer, tensor id, element index), computed with integer
hashing and table look-ups only, so the numpy and the torch versions produce
identical bytes.

Random stream
-------------
``hash32`` is the "lowbias32" 32-bit integer mixer published by Chris Wellons
(hash-prospector): x ^= x>>16; x *= 0x7feb352d; x ^= x>>15; x *= 0x846ca68b;
x ^= x>>16.  Element i of a stream with 64-bit key (k0, k1) is
hash32((hash32(i ^ k0) + k1) mod 2^32).  Arithmetic is done on int64 arrays
holding values in [0, 2^32); the 32x32-bit products are split in 16-bit halves
so that nothing overflows int64 in either library.

Value recipes (the synthetic workloads of the routed-MoE pages: Qwen3.8-Flash-
Next-style layers of 512 experts, d_model 2048, expert d_ff 768, top-10 plus one
shared expert, 2-bit and 3.5-bit block files):

* block scale s ~ U[0.005, 0.02] as fp16: 16 hash bits index a 65,536-entry
  table of fp16(0.005 + 0.015 (u + 1/2) / 65536);
* 2-bit codes: uniform, the bytes of hash words;
* codebook grid 256x4 int8, entries uniform over {1, 3, ..., 15};
* codebook indices (uint8) and sign bits: uniform, bytes of hash words;
* NVFP4: E2M1 codes uniform (bytes of hash words); E4M3 block scales with exponent field
  5..8 and mantissa 0..7 uniform (0.25 .. 3.75); the matrix's fp32 tensor scale
  2^-9 (1 + u/8), u uniform in 0..7 (weight RMS ~0.014, that of the 2-bit blocks, so
  that a 48-layer residual stack without norms stays bounded);
* N(0, sigma^2) activations / router weights: 16 hash bits index a table of
  the 65,536 mid-quantiles sigma * Phi^-1((u + 1/2) / 65536), rounded to the
  storage dtype (bf16 round-to-nearest-even, or fp32);
* router bias with Zipf(1.1) expert popularity: b[perm[r]] =
  beta * ln(r^-1.1 / H), r = 1..E, H = sum r^-1.1, perm a seeded permutation.

Block interchange layouts (what ``moe_load_layer`` and the oracle consume):

* Q2 (10 bytes / 32 weights): bytes 0-1 fp16 scale (little endian), bytes 2-9
  codes, weight i in byte 2 + (i >> 2) at bits 2*(i & 3) .. +1.
* CB35 (14 bytes / 32 weights): bytes 0-1 fp16 scale, bytes 2-9 grid row
  indices (byte 2+g covers weights 4g .. 4g+3), bytes 10-13 a little-endian
  uint32 of sign bits (bit i set: weight i negated).
* NVFP4 (9 bytes / 16 weights, after a 4-byte little-endian fp32 tensor scale at
  the start of every matrix): byte 0 the E4M3 block scale, bytes 1-8 the E2M1
  codes, weight i in byte 1 + i/2 (low nibble for even i).

Blocks run along a matrix row (the reduction dimension); rows are contiguous.
An expert is [gate (F x D)][up (F x D)][down (D x F)]; experts are contiguous
in index order.
"""
from __future__ import annotations

import math
import statistics
from dataclasses import dataclass, field
from functools import lru_cache

import numpy as np

M32 = 0xFFFFFFFF

FMT_Q2 = 0
FMT_CB35 = 1
FMT_NVFP4 = 2
BLOCK_BYTES = {FMT_Q2: 10, FMT_CB35: 14, FMT_NVFP4: 9}
BLOCK_WEIGHTS = {FMT_Q2: 32, FMT_CB35: 32, FMT_NVFP4: 16}
MATRIX_HEADER = {FMT_Q2: 0, FMT_CB35: 0, FMT_NVFP4: 4}  # NVFP4: the matrix's fp32 tensor scale

DT_F32 = 0
DT_BF16 = 1

# tensor ids of the random streams
T_ROUTER = 1
T_BIAS_PERM = 2
T_X = 3
T_GRID = 4
T_SHARED_GATE = 5
T_EXPERT = 16
F_SCALE = 0
F_CODES = 1
F_IDX = 2
F_SIGN = 3
F_TSCALE = 4


# ----------------------------------------------------------------------------------------------
# integer hashing (works on numpy int64 arrays, torch int64 tensors and python ints)
# ----------------------------------------------------------------------------------------------
def _mul32(x, c: int):
    lo = c & 0xFFFF
    hi = c >> 16
    return (x * lo + (((x * hi) & 0xFFFF) << 16)) & M32


def hash32(x):
    x = x ^ (x >> 16)
    x = _mul32(x, 0x7FEB352D)
    x = x ^ (x >> 15)
    x = _mul32(x, 0x846CA68B)
    x = x ^ (x >> 16)
    return x


def stream_key(*parts: int) -> tuple[int, int]:
    """Fold integer parts into a 64-bit stream key (two 32-bit halves)."""
    a, b = 0x243F6A88, 0x85A308D3
    for p in parts:
        p = int(p) & M32
        a = hash32(a ^ p)
        b = hash32((b + p + 0x9E3779B9) & M32)
    return a, b


def words_np(key: tuple[int, int], start: int, count: int) -> np.ndarray:
    """uint32 values (as int64) of stream ``key`` at indices start .. start+count-1."""
    i = np.arange(start, start + count, dtype=np.int64)
    return hash32((hash32(i ^ key[0]) + key[1]) & M32)


def words_torch(key: tuple[int, int], start: int, count: int, device):
    import torch

    i = torch.arange(start, start + count, dtype=torch.int64, device=device)
    return hash32((hash32(i ^ key[0]) + key[1]) & M32)


# ----------------------------------------------------------------------------------------------
# value tables
# ----------------------------------------------------------------------------------------------
def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even); returns uint16 bit patterns."""
    u = np.asarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounding = ((u >> 16) & 1) + 0x7FFF
    return ((u + rounding) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint32) << 16).view(np.float32)


@lru_cache(maxsize=None)
def scale_table_f16() -> np.ndarray:
    u = np.arange(65536, dtype=np.float64)
    s = 0.005 + 0.015 * (u + 0.5) / 65536.0
    return s.astype(np.float16).view(np.uint16)


@lru_cache(maxsize=None)
def _std_normal_quantiles() -> np.ndarray:
    nd = statistics.NormalDist()
    return np.array([nd.inv_cdf((u + 0.5) / 65536.0) for u in range(65536)], dtype=np.float64)


@lru_cache(maxsize=None)
def normal_table(sigma: float, dtype: int) -> np.ndarray:
    """65,536 N(0, sigma^2) mid-quantiles as bf16 bits (uint16) or fp32."""
    v = (_std_normal_quantiles() * sigma).astype(np.float32)
    if dtype == DT_BF16:
        return f32_to_bf16_bits(v)
    return v


# ----------------------------------------------------------------------------------------------
# workload description
# ----------------------------------------------------------------------------------------------
@dataclass(frozen=True)
class Workload:
    """Shapes and value recipe of one synthetic routed-MoE workload."""

    name: str
    wid: int  # workload id, part of every stream key
    d_model: int
    d_ff: int
    n_experts: int
    top_k: int
    n_shared: int
    shared_d_ff: int
    fmt: int = FMT_Q2
    act_dtype: int = DT_BF16
    router_dtype: int = DT_BF16
    zipf_bias: bool = True
    beta: float = 0.5
    n_layers: int = 1
    n_tokens: int = 1
    bias_select: bool = False   # router bias used for the selection only
    shared_gate: bool = False   # sigmoid-gated shared expert (gate vector like a router row)
    extra: dict = field(default_factory=dict, compare=False, hash=False)

    @property
    def block_bytes(self) -> int:
        return BLOCK_BYTES[self.fmt]

    def matrix_bytes(self, shared: bool = False) -> int:
        f = self.shared_d_ff if shared else self.d_ff
        return MATRIX_HEADER[self.fmt] + f * self.d_model // BLOCK_WEIGHTS[self.fmt] * self.block_bytes

    def expert_bytes(self, shared: bool = False) -> int:
        return 3 * self.matrix_bytes(shared)


# The five synthetic workloads (sizes of the pages' model; see module docstring)
TINY = Workload("tiny-layer-d256-f128-e16-top2", 0, 256, 128, 16, 2, 0, 128,
                act_dtype=DT_F32, router_dtype=DT_F32, zipf_bias=False, n_tokens=4)
DECODE = Workload("decode-layer-d2048-f768-e512-top10+1", 1, 2048, 768, 512, 10, 1, 768, n_tokens=1)
VERIFY = Workload("verify-stack-48L-8tok-q2", 2, 2048, 768, 512, 10, 1, 768, n_layers=48, n_tokens=8)
CODEBOOK = Workload("codebook-stack-48L-cb35", 3, 2048, 768, 512, 10, 1, 768, fmt=FMT_CB35,
                    n_layers=48, n_tokens=8)
PREFILL = Workload("prefill-stack-48L-q2", 4, 2048, 768, 512, 10, 1, 768, n_layers=48, n_tokens=8192)
NVFP4 = Workload("nvfp4-stack-48L", 5, 2048, 768, 512, 10, 1, 768, fmt=FMT_NVFP4, n_layers=48, n_tokens=8)

WORKLOADS = {w.wid: w for w in (TINY, DECODE, VERIFY, CODEBOOK, PREFILL, NVFP4)}


def small_workload(**kw) -> Workload:
    """A reduced-size workload for fast tests (same recipes)."""
    base = dict(name="small", wid=100, d_model=256, d_ff=128, n_experts=16, top_k=4, n_shared=1,
                shared_d_ff=128)
    base.update(kw)
    return Workload(**base)


# ----------------------------------------------------------------------------------------------
# generators (numpy)
# ----------------------------------------------------------------------------------------------
def gen_grid(wl: Workload, seed: int) -> np.ndarray:
    """Codebook grid, 256 x 4 int8, entries uniform over {1,3,...,15}."""
    w = words_np(stream_key(seed, wl.wid, T_GRID), 0, 1024)
    return (1 + 2 * (w & 7)).astype(np.int8).reshape(256, 4)


def gen_router(wl: Workload, seed: int, layer: int) -> np.ndarray:
    """Router weight [E x D]: bf16 bits (uint16) or fp32, N(0, 1/D)."""
    n = wl.n_experts * wl.d_model
    w = words_np(stream_key(seed, wl.wid, layer, T_ROUTER), 0, n)
    tab = normal_table(1.0 / math.sqrt(wl.d_model), wl.router_dtype)
    return tab[w & 0xFFFF].reshape(wl.n_experts, wl.d_model)


def gen_shared_gate(wl: Workload, seed: int, layer: int) -> np.ndarray | None:
    """Gate vector of a sigmoid-gated shared expert [D], stored like a router row (bf16 bits or
    fp32), N(0, 1/D); None without a gate."""
    if not (wl.shared_gate and wl.n_shared):
        return None
    w = words_np(stream_key(seed, wl.wid, layer, T_SHARED_GATE), 0, wl.d_model)
    return normal_table(1.0 / math.sqrt(wl.d_model), wl.router_dtype)[w & 0xFFFF]


def gen_bias(wl: Workload, seed: int, layer: int) -> np.ndarray | None:
    """Router bias [E] fp32 with Zipf(1.1) popularity over a seeded permutation, or None."""
    if not wl.zipf_bias:
        return None
    e = wl.n_experts
    keys = words_np(stream_key(seed, wl.wid, layer, T_BIAS_PERM), 0, e)
    perm = np.argsort(keys * e + np.arange(e), kind="stable")
    r = np.arange(1, e + 1, dtype=np.float64)
    h = np.sum(r ** -1.1)
    b = np.empty(e, dtype=np.float64)
    b[perm] = wl.beta * np.log(r ** -1.1 / h)
    return b.astype(np.float32)


def gen_x(wl: Workload, seed: int, n_tokens: int, pass_idx: int = 0, start_token: int = 0) -> np.ndarray:
    """Activations [n x D]: bf16 bits (uint16) or fp32, N(0, 1)."""
    d = wl.d_model
    w = words_np(stream_key(seed, wl.wid, pass_idx, T_X), start_token * d, n_tokens * d)
    return normal_table(1.0, wl.act_dtype)[w & 0xFFFF].reshape(n_tokens, d)


def _nvfp4_matrix_np(key_base: tuple, rows: int, cols: int) -> np.ndarray:
    nb = rows * cols // 16
    head = np.array([2.0 ** -9 * (1 + int(words_np(stream_key(*key_base, F_TSCALE), 0, 1)[0] & 7) / 8)],
                    dtype=np.float32).view(np.uint8)
    out = np.empty((nb, 9), dtype=np.uint8)
    sw = words_np(stream_key(*key_base, F_SCALE), 0, nb)
    out[:, 0] = (((5 + (sw & 3)) << 3) | ((sw >> 2) & 7)).astype(np.uint8)
    c = words_np(stream_key(*key_base, F_CODES), 0, 2 * nb).astype(np.uint32)
    out[:, 1:9] = c.view(np.uint8).reshape(nb, 8)
    return np.concatenate([head, out.reshape(-1)])


def _matrix_blocks_np(wl: Workload, key_base: tuple, rows: int, cols: int) -> np.ndarray:
    if wl.fmt == FMT_NVFP4:
        return _nvfp4_matrix_np(key_base, rows, cols)
    nb = rows * cols // 32
    bb = wl.block_bytes
    out = np.empty((nb, bb), dtype=np.uint8)
    s = scale_table_f16()[words_np(stream_key(*key_base, F_SCALE), 0, nb) & 0xFFFF]
    out[:, 0] = s & 0xFF
    out[:, 1] = s >> 8
    if wl.fmt == FMT_Q2:
        c = words_np(stream_key(*key_base, F_CODES), 0, 2 * nb).astype(np.uint32)
        out[:, 2:10] = c.view(np.uint8).reshape(nb, 8)
    else:
        ix = words_np(stream_key(*key_base, F_IDX), 0, 2 * nb).astype(np.uint32)
        out[:, 2:10] = ix.view(np.uint8).reshape(nb, 8)
        sg = words_np(stream_key(*key_base, F_SIGN), 0, nb).astype(np.uint32)
        out[:, 10:14] = sg.view(np.uint8).reshape(nb, 4)
    return out.reshape(-1)


def gen_expert(wl: Workload, seed: int, layer: int, expert: int) -> np.ndarray:
    """Interchange bytes of one expert [gate][up][down]; expert == n_experts is the shared one."""
    shared = expert >= wl.n_experts
    f = wl.shared_d_ff if shared else wl.d_ff
    d = wl.d_model
    parts = []
    for m, (r, c) in enumerate(((f, d), (f, d), (d, f))):
        parts.append(_matrix_blocks_np(wl, (seed, wl.wid, layer, T_EXPERT, expert, m), r, c))
    return np.concatenate(parts)


def gen_layer_experts(wl: Workload, seed: int, layer: int) -> np.ndarray:
    """All routed experts of a layer, [E][expert bytes] (small workloads only)."""
    return np.stack([gen_expert(wl, seed, layer, e) for e in range(wl.n_experts)])


def gen_shared(wl: Workload, seed: int, layer: int) -> np.ndarray | None:
    if wl.n_shared == 0:
        return None
    return gen_expert(wl, seed, layer, wl.n_experts)


# ----------------------------------------------------------------------------------------------
# generators (torch, on a device) -- byte-identical to the numpy ones
# ----------------------------------------------------------------------------------------------
_TORCH_TABLES: dict = {}


def _torch_table(name, arr, device):
    import torch

    k = (name, str(device))
    if k not in _TORCH_TABLES:
        a = np.asarray(arr)
        if a.dtype == np.uint16:
            t = torch.from_numpy(a.view(np.int16).copy()).to(device)
        else:
            t = torch.from_numpy(a.copy()).to(device)
        _TORCH_TABLES[k] = t
    return _TORCH_TABLES[k]


def _u32_bytes_torch(w, nbytes_per_word: int = 4):
    import torch

    sh = torch.tensor([0, 8, 16, 24][:nbytes_per_word], dtype=torch.int64, device=w.device)
    return ((w.unsqueeze(-1) >> sh) & 0xFF).to(torch.uint8)


def _matrix_blocks_torch(wl: Workload, key_base: tuple, rows: int, cols: int, out):
    """Fill ``out`` (uint8 tensor viewed [nb, block_bytes]) with a matrix's interchange blocks."""
    import torch

    dev = out.device
    nb = rows * cols // 32
    stab = _torch_table("scale", scale_table_f16(), dev)
    s = stab[words_torch(stream_key(*key_base, F_SCALE), 0, nb, dev) & 0xFFFF].to(torch.int64)
    out[:, 0] = (s & 0xFF).to(torch.uint8)
    out[:, 1] = (s >> 8).to(torch.uint8)
    if wl.fmt == FMT_Q2:
        c = words_torch(stream_key(*key_base, F_CODES), 0, 2 * nb, dev)
        out[:, 2:10] = _u32_bytes_torch(c).reshape(nb, 8)
    else:
        ix = words_torch(stream_key(*key_base, F_IDX), 0, 2 * nb, dev)
        out[:, 2:10] = _u32_bytes_torch(ix).reshape(nb, 8)
        sg = words_torch(stream_key(*key_base, F_SIGN), 0, nb, dev)
        out[:, 10:14] = _u32_bytes_torch(sg).reshape(nb, 4)


def gen_experts_torch(wl: Workload, seed: int, layer: int, experts, out):
    """Write the interchange bytes of ``experts`` (ids, all routed or all the shared one) into
    ``out`` (uint8 [len, expert bytes]); every matrix of the batch is hashed in one pass."""
    import torch

    experts = list(experts)
    if not experts:
        return
    dev = out.device
    d = wl.d_model
    shared = experts[0] >= wl.n_experts
    assert all((e >= wl.n_experts) == shared for e in experts)
    f = wl.shared_d_ff if shared else wl.d_ff
    bb = wl.block_bytes
    stab = _torch_table("scale", scale_table_f16(), dev)
    nb = f * d // BLOCK_WEIGHTS[wl.fmt]  # blocks per matrix (gate, up and down have the same count)
    off = 0
    for m in range(3):
        keys = [(seed, wl.wid, layer, T_EXPERT, e, m) for e in experts]
        if wl.fmt == FMT_NVFP4:
            _nvfp4_matrices_torch(keys, nb, out[:, off:off + 4 + nb * 9])
            off += 4 + nb * 9
            continue

        def kk(field_id):
            ks = [stream_key(*k, field_id) for k in keys]
            k0 = torch.tensor([a for a, _ in ks], dtype=torch.int64, device=dev)[:, None]
            k1 = torch.tensor([b for _, b in ks], dtype=torch.int64, device=dev)[:, None]
            return k0, k1

        def words(field_id, count):
            k0, k1 = kk(field_id)
            i = torch.arange(count, dtype=torch.int64, device=dev)[None, :]
            return hash32((hash32(i ^ k0) + k1) & M32)

        view = out[:, off:off + nb * bb].view(len(experts), nb, bb)
        sc = stab[words(F_SCALE, nb) & 0xFFFF].to(torch.int64)
        view[:, :, 0] = (sc & 0xFF).to(torch.uint8)
        view[:, :, 1] = (sc >> 8).to(torch.uint8)
        del sc
        if wl.fmt == FMT_Q2:
            c = words(F_CODES, 2 * nb)
            view[:, :, 2:10] = _u32_bytes_torch(c).reshape(len(experts), nb, 8)
        else:
            ix = words(F_IDX, 2 * nb)
            view[:, :, 2:10] = _u32_bytes_torch(ix).reshape(len(experts), nb, 8)
            del ix
            sg = words(F_SIGN, nb)
            view[:, :, 10:14] = _u32_bytes_torch(sg).reshape(len(experts), nb, 4)
        off += nb * bb


def _nvfp4_matrices_torch(keys, nb: int, out):
    """NVFP4 matrices (one per key) into out (uint8 [len(keys), 4 + 9 nb]): the fp32 tensor scale,
    then the blocks (the numpy recipe of _nvfp4_matrix_np)."""
    import torch

    dev = out.device
    heads = np.array([2.0 ** -9 * (1 + int(words_np(stream_key(*k, F_TSCALE), 0, 1)[0] & 7) / 8) for k in keys],
                     dtype=np.float32).view(np.uint8).reshape(len(keys), 4)
    out[:, 0:4] = torch.from_numpy(heads).to(dev)

    def words(field_id, count):
        ks = [stream_key(*k, field_id) for k in keys]
        k0 = torch.tensor([a for a, _ in ks], dtype=torch.int64, device=dev)[:, None]
        k1 = torch.tensor([b for _, b in ks], dtype=torch.int64, device=dev)[:, None]
        i = torch.arange(count, dtype=torch.int64, device=dev)[None, :]
        return hash32((hash32(i ^ k0) + k1) & M32)

    view = out[:, 4:].view(len(keys), nb, 9)
    sw = words(F_SCALE, nb)
    view[:, :, 0] = (((5 + (sw & 3)) << 3) | ((sw >> 2) & 7)).to(torch.uint8)
    del sw
    c = words(F_CODES, 2 * nb)
    view[:, :, 1:9] = _u32_bytes_torch(c).reshape(len(keys), nb, 8)


def gen_router_torch(wl: Workload, seed: int, layer: int, device):
    import torch

    n = wl.n_experts * wl.d_model
    w = words_torch(stream_key(seed, wl.wid, layer, T_ROUTER), 0, n, device)
    tab = _torch_table(("router", wl.d_model, wl.router_dtype),
                       normal_table(1.0 / math.sqrt(wl.d_model), wl.router_dtype), device)
    v = tab[w & 0xFFFF]
    if wl.router_dtype == DT_BF16:
        return v.view(torch.bfloat16).reshape(wl.n_experts, wl.d_model)
    return v.reshape(wl.n_experts, wl.d_model)


def gen_shared_gate_torch(wl: Workload, seed: int, layer: int, device):
    import torch

    if not (wl.shared_gate and wl.n_shared):
        return None
    w = words_torch(stream_key(seed, wl.wid, layer, T_SHARED_GATE), 0, wl.d_model, device)
    tab = _torch_table(("router", wl.d_model, wl.router_dtype),
                       normal_table(1.0 / math.sqrt(wl.d_model), wl.router_dtype), device)
    v = tab[w & 0xFFFF]
    return v.view(torch.bfloat16) if wl.router_dtype == DT_BF16 else v


def gen_x_torch(wl: Workload, seed: int, n_tokens: int, pass_idx: int, device, start_token: int = 0):
    import torch

    d = wl.d_model
    w = words_torch(stream_key(seed, wl.wid, pass_idx, T_X), start_token * d, n_tokens * d, device)
    tab = _torch_table(("x", wl.act_dtype), normal_table(1.0, wl.act_dtype), device)
    v = tab[w & 0xFFFF]
    if wl.act_dtype == DT_BF16:
        return v.view(torch.bfloat16).reshape(n_tokens, d)
    return v.reshape(n_tokens, d)


def to_torch_bf16(bits: np.ndarray):
    """numpy bf16 bit patterns -> torch.bfloat16 tensor (CPU)."""
    import torch

    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
