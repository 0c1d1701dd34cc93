"""fp64 CPU oracle of the routed-MoE FFN computed from low-bit weight blocks.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the bench's
CPU-baseline leg use it; the product (``expert_ffn_gemv_b200``) never imports it
and it never imports the product.  The arithmetic lives in ``moe_oracle.c``
(plain C, fp64); this module only marshals numpy arrays with ctypes.

Definitions and their sources are listed in ``moe_oracle.h``.  Pins: see
``tests/test_oracle_*.py`` (hand-worked blocks, brute force against dense
matrices, closed forms and invariants).
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_LIB_PATH = _HERE / "_build" / "liboracle.so"
_lib = None

FMT_Q2 = 0
FMT_CB35 = 1
FMT_NVFP4 = 2
F32 = 0
BF16 = 1
F64 = 2


def build(force: bool = False) -> Path:
    """Compile moe_oracle.c with gcc (OpenMP over tokens) into _build/liboracle.so."""
    src = _HERE / "moe_oracle.c"
    if not force and _LIB_PATH.exists() and _LIB_PATH.stat().st_mtime >= max(
            src.stat().st_mtime, (_HERE / "moe_oracle.h").stat().st_mtime):
        return _LIB_PATH
    _LIB_PATH.parent.mkdir(exist_ok=True)
    tmp = _LIB_PATH.with_suffix(f".{os.getpid()}.tmp")
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-o", str(tmp), str(src), "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class _Layer(C.Structure):
    _fields_ = [
        ("fmt", C.c_int), ("d_model", C.c_int), ("d_ff", C.c_int), ("n_experts", C.c_int),
        ("top_k", C.c_int), ("n_shared", C.c_int), ("shared_d_ff", C.c_int),
        ("grid", C.c_void_p), ("router_w", C.c_void_p), ("router_dtype", C.c_int),
        ("bias", C.c_void_p), ("experts", C.c_void_p), ("shared", C.c_void_p),
        ("shared_gate", C.c_void_p), ("bias_mode", C.c_int),
    ]

BIAS_LOGIT = 0
BIAS_SELECT = 1


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(str(build()))
        P, I = C.c_void_p, C.c_int
        _lib.or_f16_to_f64.restype = C.c_double
        _lib.or_f16_to_f64.argtypes = [C.c_uint16]
        _lib.or_bf16_to_f64.restype = C.c_double
        _lib.or_bf16_to_f64.argtypes = [C.c_uint16]
        _lib.or_convert_to_f64.argtypes = [P, I, C.c_size_t, P]
        _lib.or_dequant_block.argtypes = [I, P, P, P]
        _lib.or_e2m1_to_f64.restype = C.c_double
        _lib.or_e2m1_to_f64.argtypes = [I]
        _lib.or_e4m3_to_f64.restype = C.c_double
        _lib.or_e4m3_to_f64.argtypes = [C.c_uint8]
        _lib.or_block_weights.argtypes = [I]
        _lib.or_matrix_bytes.restype = C.c_size_t
        _lib.or_matrix_bytes.argtypes = [I, I, I]
        _lib.or_dequant_matrix.argtypes = [I, P, I, I, P, P]
        _lib.or_matvec.argtypes = [I, P, I, I, P, P, P]
        _lib.or_silu.restype = C.c_double
        _lib.or_silu.argtypes = [C.c_double]
        _lib.or_expert_ffn.argtypes = [I, P, I, I, P, P, P, P]
        _lib.or_router_logits.argtypes = [P, I, P, I, I, P, P]
        _lib.or_topk_softmax.argtypes = [P, I, I, P, P, P]
        _lib.or_topk_select_softmax.argtypes = [P, P, I, I, P, P, P]
        _lib.or_sigmoid.restype = C.c_double
        _lib.or_sigmoid.argtypes = [C.c_double]
        _lib.or_moe_layer.argtypes = [P, P, I, P, P, P, P, P, I]
        _lib.or_moe_layer.restype = I
        _lib.or_route.argtypes = [P, P, I, P, P, P]
        _lib.or_route.restype = I
        _lib.or_max_threads.restype = I
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# --------------------------------------------------------------------------------------------
def f16_to_f64(bits: int) -> float:
    return lib().or_f16_to_f64(int(bits))


def bf16_to_f64(bits: int) -> float:
    return lib().or_bf16_to_f64(int(bits))


def to_f64(a: np.ndarray, dtype: int) -> np.ndarray:
    """Exact conversion of fp32 values or bf16 bit patterns (uint16) to fp64."""
    src = _c(a, np.float32 if dtype == F32 else (np.uint16 if dtype == BF16 else np.float64))
    out = np.empty(src.shape, dtype=np.float64)
    lib().or_convert_to_f64(_p(src), dtype, src.size, _p(out))
    return out


def e2m1_to_f64(code: int) -> float:
    return lib().or_e2m1_to_f64(int(code))


def e4m3_to_f64(b: int) -> float:
    return lib().or_e4m3_to_f64(int(b))


def block_weights(fmt: int) -> int:
    return lib().or_block_weights(fmt)


def matrix_bytes(fmt: int, rows: int, cols: int) -> int:
    return lib().or_matrix_bytes(fmt, rows, cols)


def dequant_block(fmt: int, blk: np.ndarray, grid: np.ndarray | None = None) -> np.ndarray:
    """One block's weights (32; NVFP4: 16, without its matrix's tensor scale)."""
    b = _c(blk, np.uint8)
    g = None if grid is None else _c(grid, np.int8)
    out = np.empty(32, dtype=np.float64)
    lib().or_dequant_block(fmt, _p(b), _p(g), _p(out))
    return out[:block_weights(fmt)]


def dequant_matrix(fmt, blocks, rows, cols, grid=None) -> np.ndarray:
    b = _c(blocks, np.uint8)
    g = None if grid is None else _c(grid, np.int8)
    out = np.empty((rows, cols), dtype=np.float64)
    lib().or_dequant_matrix(fmt, _p(b), rows, cols, _p(g), _p(out))
    return out


def matvec(fmt, blocks, rows, cols, x, grid=None) -> np.ndarray:
    b = _c(blocks, np.uint8)
    g = None if grid is None else _c(grid, np.int8)
    xx = _c(x, np.float64)
    y = np.empty(rows, dtype=np.float64)
    lib().or_matvec(fmt, _p(b), rows, cols, _p(g), _p(xx), _p(y))
    return y


def silu(z: float) -> float:
    return lib().or_silu(float(z))


def expert_ffn(fmt, expert, d_model, d_ff, x, grid=None, want_h=False):
    b = _c(expert, np.uint8)
    g = None if grid is None else _c(grid, np.int8)
    xx = _c(x, np.float64)
    h = np.empty(d_ff, dtype=np.float64)
    y = np.empty(d_model, dtype=np.float64)
    lib().or_expert_ffn(fmt, _p(b), d_model, d_ff, _p(g), _p(xx), _p(h), _p(y))
    return (y, h) if want_h else y


def router_logits(router_w, router_dtype, bias, x):
    w = _c(router_w, np.float32 if router_dtype == F32 else np.uint16)
    e, d = w.shape
    bb = None if bias is None else _c(bias, np.float32)
    xx = _c(x, np.float64)
    out = np.empty(e, dtype=np.float64)
    lib().or_router_logits(_p(w), router_dtype, _p(bb), e, d, _p(xx), _p(out))
    return out


def topk_select_softmax(score, wlogit, k):
    sc = _c(score, np.float64)
    wl = _c(wlogit, np.float64)
    idx = np.empty(k, dtype=np.int32)
    w = np.empty(k, dtype=np.float64)
    m = np.empty(1, dtype=np.float64)
    lib().or_topk_select_softmax(_p(sc), _p(wl), sc.size, k, _p(idx), _p(w), _p(m))
    return idx, w, float(m[0])


def sigmoid(z: float) -> float:
    return lib().or_sigmoid(float(z))


def topk_softmax(logits, k):
    lg = _c(logits, np.float64)
    idx = np.empty(k, dtype=np.int32)
    w = np.empty(k, dtype=np.float64)
    m = np.empty(1, dtype=np.float64)
    lib().or_topk_softmax(_p(lg), lg.size, k, _p(idx), _p(w), _p(m))
    return idx, w, float(m[0])


class Layer:
    """One MoE layer's weights as the oracle sees them (interchange bytes).

    ``experts``: dict {expert id: uint8 bytes} or an [E, bytes] array; experts not
    present are "not supplied" (an error if the router selects them).
    """

    def __init__(self, *, fmt, d_model, d_ff, n_experts, top_k, n_shared, shared_d_ff,
                 router_w, router_dtype, bias=None, experts=None, shared=None, grid=None,
                 shared_gate=None, bias_mode=BIAS_LOGIT):
        self.fmt, self.d_model, self.d_ff = fmt, d_model, d_ff
        self.n_experts, self.top_k = n_experts, top_k
        self.n_shared, self.shared_d_ff = n_shared, shared_d_ff
        self.router_dtype = router_dtype
        self.router_w = _c(router_w, np.float32 if router_dtype == F32 else np.uint16)
        self.bias = None if bias is None else _c(bias, np.float32)
        self.grid = None if grid is None else _c(grid, np.int8)
        self.shared = None if shared is None else _c(shared, np.uint8)
        self.shared_gate = None if shared_gate is None else _c(
            shared_gate, np.float32 if router_dtype == F32 else np.uint16)
        self.bias_mode = int(bias_mode)
        self._experts: dict[int, np.ndarray] = {}
        if experts is not None:
            if isinstance(experts, dict):
                items = experts.items()
            else:
                items = enumerate(experts)
            for e, b in items:
                self._experts[int(e)] = _c(b, np.uint8)

    def set_expert(self, e: int, blocks: np.ndarray):
        self._experts[int(e)] = _c(blocks, np.uint8)

    def _struct(self):
        ptrs = (C.c_void_p * self.n_experts)()
        for e, b in self._experts.items():
            ptrs[e] = b.ctypes.data
        s = _Layer(self.fmt, self.d_model, self.d_ff, self.n_experts, self.top_k, self.n_shared,
                   self.shared_d_ff, _p(self.grid), _p(self.router_w), self.router_dtype,
                   _p(self.bias), C.cast(ptrs, C.c_void_p), _p(self.shared), _p(self.shared_gate),
                   self.bias_mode)
        return s, ptrs

    def route(self, x: np.ndarray):
        """Steps 1-3 for x (n x D fp64): idx (n x k), w (n x k), margin (n)."""
        xx = _c(np.atleast_2d(x), np.float64)
        n = xx.shape[0]
        idx = np.empty((n, self.top_k), dtype=np.int32)
        w = np.empty((n, self.top_k), dtype=np.float64)
        m = np.empty(n, dtype=np.float64)
        s, keep = self._struct()
        rc = lib().or_route(C.byref(s), _p(xx), n, _p(idx), _p(w), _p(m))
        if rc:
            raise ValueError(f"or_route failed ({rc})")
        return idx, w, m

    def forward(self, x: np.ndarray, n_threads: int = 0):
        """Steps 1-5 for x (n x D fp64).  Returns dict y, idx, w, margin, counts."""
        xx = _c(np.atleast_2d(x), np.float64)
        n = xx.shape[0]
        y = np.empty_like(xx)
        idx = np.empty((n, self.top_k), dtype=np.int32)
        w = np.empty((n, self.top_k), dtype=np.float64)
        m = np.empty(n, dtype=np.float64)
        cnt = np.empty(self.n_experts, dtype=np.int32)
        s, keep = self._struct()
        rc = lib().or_moe_layer(C.byref(s), _p(xx), n, _p(y), _p(idx), _p(w), _p(m), _p(cnt),
                                int(n_threads))
        if rc == -1:
            raise KeyError("a selected expert was not supplied to the oracle")
        if rc:
            raise ValueError(f"or_moe_layer failed ({rc})")
        return dict(y=y, idx=idx, w=w, margin=m, counts=cnt)


def stack_forward(layers, x, supply=None, n_threads: int = 0):
    """Layer-by-layer stack with a residual add after every layer: x <- x + MoE_l(x).

    ``layers``: sequence of ``Layer`` (or callables returning one for index l).
    ``supply(l, layer, needed_experts)``: optional hook that adds the selected experts
    to ``layer`` before its forward (lazy generation of large layers).
    Returns the final x and the per-layer routing records.
    """
    xs = _c(np.atleast_2d(x), np.float64).copy()
    recs = []
    for l, L in enumerate(layers):
        if callable(L) and not isinstance(L, Layer):
            L = L(l)
        if supply is not None:
            idx, _, _ = L.route(xs)
            supply(l, L, sorted(set(int(e) for e in idx.reshape(-1))))
        r = L.forward(xs, n_threads=n_threads)
        recs.append(dict(idx=r["idx"], w=r["w"], margin=r["margin"], counts=r["counts"], x_in=xs))
        xs = xs + r["y"]
    return xs, recs


def max_threads() -> int:
    return lib().or_max_threads()
