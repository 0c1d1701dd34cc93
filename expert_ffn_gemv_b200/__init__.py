"""Python binding of the B200 routed-MoE FFN library (include/moe.h).

Argument marshalling only: every step of the computation runs in the CUDA kernels of
``_lib/libmoe_b200.so``.  The functions carry the C names (``moe_create``,
``moe_load_layer``, ``moe_forward``, ``moe_forward_stack``, ``moe_check``,
``moe_destroy``); ``MoE`` wraps them for torch tensors (device memory and the current
stream come from PyTorch).  Importing this package raises if the library has not been
built (``python -m expert_ffn_gemv_b200.build``): there is no fallback path.
"""
from __future__ import annotations

import ctypes as C
from pathlib import Path

import os

# MOE_B200_LIB may point at another build of the same library (e.g. a tuning variant)
_LIB_PATH = Path(os.environ.get("MOE_B200_LIB") or Path(__file__).resolve().parent / "_lib" / "libmoe_b200.so")

MOE_OK = 0
MOE_ERR_INVALID_ARGUMENT = 1
MOE_ERR_OUT_OF_MEMORY = 2
MOE_ERR_CUDA = 3
MOE_ERR_NOT_LOADED = 4
MOE_ERR_UNSUPPORTED = 5
MOE_ERR_TIMEOUT = 6
MOE_ERR_DEVICE_FAULT = 7

MOE_FMT_Q2_32 = 0
MOE_FMT_CB35_32 = 1
MOE_FMT_NVFP4_16 = 2
MOE_F32 = 0
MOE_BF16 = 1
MOE_BIAS_LOGIT = 0
MOE_BIAS_SELECT = 1

DECODE_MAX_TOKENS = 8


class moe_config(C.Structure):
    _fields_ = [
        ("struct_size", C.c_uint32), ("n_layers", C.c_int32), ("d_model", C.c_int32),
        ("d_ff", C.c_int32), ("n_experts", C.c_int32), ("top_k", C.c_int32),
        ("n_shared", C.c_int32), ("shared_d_ff", C.c_int32), ("fmt", C.c_int32),
        ("act_dtype", C.c_int32), ("router_dtype", C.c_int32), ("out_dtype", C.c_int32),
        ("max_tokens", C.c_int32), ("codebook_grid", C.c_void_p), ("device", C.c_int32),
        ("bias_mode", C.c_int32), ("shared_gate", C.c_int32),
    ]


class moe_layer_weights(C.Structure):
    _fields_ = [("router_w", C.c_void_p), ("router_bias", C.c_void_p),
                ("expert_blocks", C.c_void_p), ("shared_blocks", C.c_void_p), ("shared_gate_w", C.c_void_p)]


class moe_route_out(C.Structure):
    _fields_ = [("topk_idx", C.c_void_p), ("topk_w", C.c_void_p), ("expert_counts", C.c_void_p)]


EXPORTED = [
    "moe_create", "moe_load_layer", "moe_forward", "moe_forward_stack", "moe_check", "moe_destroy",
    "moe_status_string", "moe_last_error", "moe_device_bytes", "moe_debug_set_spin_limit",
    "moe_debug_set_alloc_cap", "moe_debug_wait_test", "moe_profile_enable", "moe_profile_read",
    "moe_route_noalloc",
]

_lib = None


def library_path() -> Path:
    return _LIB_PATH


def lib() -> C.CDLL:
    """Load the CUDA library (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not _LIB_PATH.exists():
            raise RuntimeError(f"{_LIB_PATH} is missing: build it with `python -m expert_ffn_gemv_b200.build`")
        L = C.CDLL(str(_LIB_PATH))
        P, I, U64 = C.c_void_p, C.c_int32, C.c_uint64
        L.moe_create.argtypes = [C.POINTER(moe_config), C.POINTER(P)]
        L.moe_load_layer.argtypes = [P, I, C.POINTER(moe_layer_weights), P]
        L.moe_forward.argtypes = [P, I, P, P, I, P, C.POINTER(moe_route_out)]
        L.moe_forward_stack.argtypes = [P, I, I, P, P, I, P, C.POINTER(moe_route_out), P]
        L.moe_check.argtypes = [P]
        L.moe_destroy.argtypes = [P]
        L.moe_status_string.argtypes = [I]
        L.moe_status_string.restype = C.c_char_p
        L.moe_last_error.argtypes = [P]
        L.moe_last_error.restype = C.c_char_p
        L.moe_device_bytes.argtypes = [P]
        L.moe_device_bytes.restype = U64
        L.moe_debug_set_spin_limit.argtypes = [P, U64]
        L.moe_debug_set_alloc_cap.argtypes = [P, U64]
        L.moe_debug_wait_test.argtypes = [P, P]
        L.moe_profile_enable.argtypes = [P, I]
        L.moe_profile_read.argtypes = [P, I, C.POINTER(C.c_float), C.POINTER(I)]
        L.moe_route_noalloc.argtypes = [P, I, P, I, I, I, P, I, I, P, P, P]
        for name in ("moe_create", "moe_load_layer", "moe_forward", "moe_forward_stack", "moe_check",
                     "moe_destroy", "moe_debug_set_spin_limit", "moe_debug_set_alloc_cap",
                     "moe_debug_wait_test", "moe_profile_enable", "moe_profile_read", "moe_route_noalloc"):
            getattr(L, name).restype = I
        _lib = L
    return _lib


class MoeError(RuntimeError):
    def __init__(self, status: int, detail: str):
        self.status = status
        super().__init__(f"{lib().moe_status_string(status).decode()} ({status}): {detail}")


# ----------------------------------------------------------------------------------- C names
def moe_create(cfg: moe_config) -> C.c_void_p:
    h = C.c_void_p()
    st = lib().moe_create(C.byref(cfg), C.byref(h))
    if st != MOE_OK:
        raise MoeError(st, "moe_create")
    return h


def moe_load_layer(h, layer: int, w: moe_layer_weights, stream) -> int:
    return lib().moe_load_layer(h, layer, C.byref(w), stream)


def moe_forward(h, layer: int, x: int, y: int, n_tokens: int, stream, route: moe_route_out | None = None) -> int:
    return lib().moe_forward(h, layer, x, y, n_tokens, stream, None if route is None else C.byref(route))


def moe_forward_stack(h, first_layer: int, n_layers: int, x_in: int, x_out: int, n_tokens: int, stream,
                      per_layer_route=None, x_trace: int | None = None) -> int:
    return lib().moe_forward_stack(h, first_layer, n_layers, x_in, x_out, n_tokens, stream, per_layer_route,
                                   x_trace)


def moe_check(h) -> int:
    return lib().moe_check(h)


def moe_destroy(h) -> int:
    return lib().moe_destroy(h)


def moe_last_error(h) -> str:
    return lib().moe_last_error(h).decode()


def moe_device_bytes(h) -> int:
    return lib().moe_device_bytes(h)


def moe_debug_set_spin_limit(h, cycles: int) -> int:
    return lib().moe_debug_set_spin_limit(h, cycles)


def moe_debug_set_alloc_cap(h, nbytes: int) -> int:
    return lib().moe_debug_set_alloc_cap(h, nbytes)


def moe_debug_wait_test(h, stream) -> int:
    return lib().moe_debug_wait_test(h, stream)


def moe_profile_enable(h, on) -> int:
    """on: False/0 = off, True = all kernel classes, or a bit mask of classes."""
    mask = 0x7 if on is True else int(on)
    return lib().moe_profile_enable(h, mask)


def moe_profile_read(h, kind: int):
    """(status, total_ms, launches) of kernel class ``kind`` in the most recent call."""
    ms = C.c_float()
    n = C.c_int32()
    st = lib().moe_profile_read(h, kind, C.byref(ms), C.byref(n))
    return st, ms.value, n.value


PROF_ROUTE, PROF_GATEUP, PROF_DOWN = 0, 1, 2


def moe_route_noalloc(router_w: int, router_dtype: int, router_bias: int | None, n_experts: int, d_model: int,
                      top_k: int, x: int, x_dtype: int, n_tokens: int, topk_idx: int, topk_w: int, stream) -> int:
    """Handle-less routing that allocates no device memory (device pointers; see include/moe.h)."""
    return lib().moe_route_noalloc(router_w, router_dtype, router_bias, n_experts, d_model, top_k, x, x_dtype,
                                   n_tokens, topk_idx, topk_w, stream)


# ----------------------------------------------------------------------------------- torch wrapper
def _ptr(t) -> int | None:
    if t is None:
        return None
    if hasattr(t, "data_ptr"):
        return t.data_ptr()
    if hasattr(t, "ctypes"):  # numpy (host memory)
        return t.ctypes.data
    return int(t)


def _stream():
    import torch

    return C.c_void_p(torch.cuda.current_stream().cuda_stream)


class MoE:
    """A handle with its configuration; methods take torch tensors (or numpy arrays for host data)."""

    def __init__(self, *, n_layers, d_model, d_ff, n_experts, top_k, n_shared=0, shared_d_ff=None,
                 fmt=MOE_FMT_Q2_32, act_dtype=MOE_BF16, router_dtype=MOE_BF16, out_dtype=MOE_F32,
                 max_tokens=8, codebook_grid=None, device=0, bias_mode=MOE_BIAS_LOGIT, shared_gate=0):
        self._grid = None
        if codebook_grid is not None:
            import numpy as np

            self._grid = np.ascontiguousarray(codebook_grid, dtype=np.int8).reshape(-1)
        self.cfg = moe_config(C.sizeof(moe_config), n_layers, d_model, d_ff, n_experts, top_k, n_shared,
                              shared_d_ff if shared_d_ff is not None else d_ff, fmt, act_dtype, router_dtype,
                              out_dtype, max_tokens,
                              None if self._grid is None else self._grid.ctypes.data, device, bias_mode,
                              int(shared_gate))
        self.h = moe_create(self.cfg)

    def _check(self, st: int, what: str):
        if st != MOE_OK:
            raise MoeError(st, f"{what}: {moe_last_error(self.h)}")

    def load_layer(self, layer, router_w, router_bias, expert_blocks, shared_blocks=None, shared_gate_w=None):
        w = moe_layer_weights(_ptr(router_w), _ptr(router_bias), _ptr(expert_blocks), _ptr(shared_blocks),
                              _ptr(shared_gate_w))
        self._keep = (router_w, router_bias, expert_blocks, shared_blocks, shared_gate_w)
        self._check(moe_load_layer(self.h, layer, w, _stream()), "moe_load_layer")

    def forward(self, layer, x, y, n_tokens=None, route=None):
        n = x.shape[0] if n_tokens is None else n_tokens
        r = None
        if route is not None:
            r = moe_route_out(*[_ptr(route.get(k)) for k in ("idx", "w", "counts")])
        self._check(moe_forward(self.h, layer, _ptr(x), _ptr(y), n, _stream(), r), "moe_forward")

    def forward_stack(self, first_layer, n_layers, x_in, x_out, n_tokens=None, routes=None, x_trace=None):
        n = x_in.shape[0] if n_tokens is None else n_tokens
        arr = None
        if routes is not None:
            arr = (moe_route_out * n_layers)(
                *[moe_route_out(*[_ptr(r.get(k)) for k in ("idx", "w", "counts")]) for r in routes])
        self._check(moe_forward_stack(self.h, first_layer, n_layers, _ptr(x_in), _ptr(x_out), n, _stream(), arr,
                                      _ptr(x_trace)), "moe_forward_stack")

    def check(self) -> int:
        return moe_check(self.h)

    def device_bytes(self) -> int:
        return moe_device_bytes(self.h)

    def close(self):
        if getattr(self, "h", None):
            moe_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
