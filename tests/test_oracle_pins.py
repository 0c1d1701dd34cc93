"""Pins of the fp64 oracle against facts fixed by the format definitions and by mathematics.

Every test here runs on the CPU.  Each one is chosen so that a plausible slip in the oracle
(a dropped term, a wrong sign, index or bit position, a transposed operand, a missing bias or
shared expert) fails at least one of them.
"""
import math
from pathlib import Path

import numpy as np
import pytest

import oracle
import synth

GOLDEN = Path(__file__).resolve().parent / "golden"


def _read_golden(name):
    out = {}
    for line in (GOLDEN / name).read_text().splitlines():
        if not line or line.startswith("#"):
            continue
        k, v = line.split(":", 1)
        out[k.strip()] = v.split()
    return out


# ------------------------------------------------------------------ exact scalar conversions
@pytest.mark.parametrize("bits,val", [
    (0x3C00, 1.0), (0xC000, -2.0), (0x7BFF, 65504.0), (0x0001, 2.0 ** -24),
    (0x0400, 2.0 ** -14), (0x211F, 1311 / 131072), (0x3800, 0.5), (0x0000, 0.0),
])
def test_f16_decode(bits, val):
    assert oracle.f16_to_f64(bits) == val


@pytest.mark.parametrize("bits,val", [
    (0x3F80, 1.0), (0xBFC0, -1.5), (0x4040, 3.0), (0x0001, 2.0 ** -133), (0x3C00, 2.0 ** -7),
])
def test_bf16_decode(bits, val):
    assert oracle.bf16_to_f64(bits) == val


# ------------------------------------------------------------------ hand-worked blocks
def test_q2_block_golden():
    g = _read_golden("q2_block.txt")
    blk = np.array([int(b, 16) for b in g["bytes"]], dtype=np.uint8)
    k = np.array([int(v) for v in g["k"]], dtype=np.float64)
    w = oracle.dequant_block(oracle.FMT_Q2, blk)
    assert np.array_equal(w, k * 1311 / 262144)


def test_q2_block_extremes():
    s = 0x3C00  # 1.0
    zero = np.array([s & 0xFF, s >> 8] + [0] * 8, dtype=np.uint8)
    ones = np.array([s & 0xFF, s >> 8] + [0xFF] * 8, dtype=np.uint8)
    assert np.all(oracle.dequant_block(oracle.FMT_Q2, zero) == -1.5)
    assert np.all(oracle.dequant_block(oracle.FMT_Q2, ones) == 1.5)


def _golden_grid():
    g = _read_golden("cb35_block.txt")
    grid = np.zeros((256, 4), dtype=np.int8)
    for r in (0, 5, 255):
        grid[r] = [int(v) for v in g[f"grid{r}"]]
    return g, grid


def test_cb35_block_golden():
    g, grid = _golden_grid()
    blk = np.array([int(b, 16) for b in g["bytes"]], dtype=np.uint8)
    want = 0.5 * np.array([int(v) for v in g["w_over_s"]], dtype=np.float64)
    assert np.array_equal(oracle.dequant_block(oracle.FMT_CB35, blk, grid), want)


def test_dequant_matrix_block_placement():
    # every block is the all-zero-code block (-1.5 s) except one marked block at (r, b) = (5, 2)
    rows, cols = 7, 128
    nb = cols // 32
    base = np.array([0x00, 0x3C] + [0x00] * 8, dtype=np.uint8)  # s = 1
    mark = np.array([0x00, 0x40] + [0xFF] * 8, dtype=np.uint8)  # s = 2, codes 3 -> +3.0
    blocks = np.tile(base, rows * nb).reshape(rows, nb, 10)
    blocks[5, 2] = mark
    w = oracle.dequant_matrix(oracle.FMT_Q2, blocks.reshape(-1), rows, cols)
    want = np.full((rows, cols), -1.5)
    want[5, 64:96] = 3.0
    assert np.array_equal(w, want)


# ------------------------------------------------------------------ matvec: brute force
@pytest.mark.parametrize("fmt", [oracle.FMT_Q2, oracle.FMT_CB35, oracle.FMT_NVFP4])
def test_matvec_equals_dense_bruteforce(fmt):
    wl = synth.small_workload(d_model=64, d_ff=96, fmt=fmt)
    e = synth.gen_expert(wl, 3, 0, 1)
    grid = synth.gen_grid(wl, 3) if fmt == oracle.FMT_CB35 else None
    rng = np.random.default_rng(0)
    x = rng.standard_normal(64)
    mat = wl.matrix_bytes()
    assert mat == oracle.matrix_bytes(fmt, 96, 64)
    gate_dense = oracle.dequant_matrix(fmt, e[:mat], 96, 64, grid)
    y = oracle.matvec(fmt, e[:mat], 96, 64, x, grid)
    assert np.allclose(y, gate_dense @ x, rtol=1e-12, atol=1e-12)
    down_dense = oracle.dequant_matrix(fmt, e[2 * mat:], 64, 96, grid)
    h = rng.standard_normal(96)
    assert np.allclose(oracle.matvec(fmt, e[2 * mat:], 64, 96, h, grid), down_dense @ h,
                       rtol=1e-12, atol=1e-12)


def test_matvec_transposition_detected():
    # a non-square matrix with distinct rows: W x must differ from the (padded) transpose use
    wl = synth.small_workload(d_model=64, d_ff=32)
    e = synth.gen_expert(wl, 1, 0, 0)
    mat = 32 * 64 // 32 * 10
    dense = oracle.dequant_matrix(oracle.FMT_Q2, e[:mat], 32, 64)
    x = np.zeros(64)
    x[40] = 1.0  # picks column 40
    assert np.array_equal(oracle.matvec(oracle.FMT_Q2, e[:mat], 32, 64, x), dense[:, 40])


# ------------------------------------------------------------------ SwiGLU closed forms
def test_silu_closed_forms():
    assert oracle.silu(0.0) == 0.0
    assert oracle.silu(1.0) == pytest.approx(1.0 / (1.0 + math.exp(-1.0)), rel=1e-15)
    assert oracle.silu(-1.0) == pytest.approx(-1.0 / (1.0 + math.e), rel=1e-15)
    assert oracle.silu(40.0) == pytest.approx(40.0, rel=1e-15)
    assert abs(oracle.silu(-40.0)) < 1e-15
    # silu(z) - silu(-z) = z
    for z in (0.3, 1.7, 5.0):
        assert oracle.silu(z) - oracle.silu(-z) == pytest.approx(z, rel=1e-14)


# ------------------------------------------------------------------ router / top-k
def test_topk_softmax_hand_worked():
    idx, w, m = oracle.topk_softmax(np.array([2.0, 1.0, 0.0, -1.0]), 2)
    assert list(idx) == [0, 1]
    e = math.e
    assert w[0] == pytest.approx(e / (e + 1), rel=1e-15)
    assert w[1] == pytest.approx(1 / (e + 1), rel=1e-15)
    assert m == 1.0


def test_topk_order_independent_of_position():
    idx, w, m = oracle.topk_softmax(np.array([-1.0, 0.0, 2.0, 1.0]), 3)
    assert list(idx) == [2, 3, 1]
    assert m == 1.0
    z = np.exp([0.0, -1.0, -2.0])
    assert np.allclose(w, z / z.sum(), rtol=1e-15)


def test_topk_tie_lower_index_wins():
    idx, w, m = oracle.topk_softmax(np.array([1.0, 3.0, 3.0, 0.0]), 1)
    assert list(idx) == [1] and w[0] == 1.0 and m == 0.0


def test_topk_k_equals_e():
    idx, w, m = oracle.topk_softmax(np.array([0.5, -0.5]), 2)
    assert list(idx) == [0, 1] and m == math.inf
    assert w.sum() == pytest.approx(1.0, abs=1e-15)


def test_topk_matches_full_sort():
    rng = np.random.default_rng(1)
    for _ in range(20):
        lg = rng.standard_normal(512)
        idx, w, m = oracle.topk_softmax(lg, 10)
        order = np.argsort(-lg, kind="stable")
        assert list(idx) == list(order[:10])
        assert m == lg[order[9]] - lg[order[10]]
        assert abs(w.sum() - 1.0) < 1e-12
        assert np.all(np.diff(w) <= 0)


def test_router_logits_identity_rows_and_bias():
    # fp32 router with unit rows: logit e = x[e] + b[e]
    E, D = 4, 32
    W = np.zeros((E, D), dtype=np.float32)
    for e in range(E):
        W[e, e] = 1.0
    b = np.array([0.5, -0.25, 0.0, 2.0], dtype=np.float32)
    x = np.arange(D, dtype=np.float64) / 8
    lg = oracle.router_logits(W, oracle.F32, b, x)
    assert np.array_equal(lg, np.array([0.5, 0.125 - 0.25, 0.25, 0.375 + 2.0]))


def test_router_logits_bf16_weights():
    # bf16 bits 0x3F80 = 1, 0xC000 = -2: logit = x0 - 2 x1
    W = np.zeros((1, 32), dtype=np.uint16)
    W[0, 0], W[0, 1] = 0x3F80, 0xC000
    x = np.zeros(32)
    x[0], x[1] = 3.0, 0.25
    assert oracle.router_logits(W, oracle.BF16, None, x)[0] == 2.5


# ------------------------------------------------------------------ hand-worked tiny layer
def _const_blocks(rows, cols, scale_bits_per_row, code_byte):
    nb = cols // 32
    out = np.zeros((rows, nb, 10), dtype=np.uint8)
    for r in range(rows):
        s = scale_bits_per_row[r]
        out[r, :, 0] = s & 0xFF
        out[r, :, 1] = s >> 8
        out[r, :, 2:] = code_byte
    return out.reshape(-1)


def test_hand_worked_tiny_layer():
    """D = F = 32, two experts, top-1, fp32 router with unit rows, x = (1, 0.5, 0, ...).

    Router: logits (x0, x1) = (1, 0.5) -> expert 0, weight 1, margin 0.5.
    Expert 0: gate codes 3 (w = 1.5), up codes 2 (w = 0.5), all scales 1:
      g_f = 1.5*1 + 1.5*0.5 = 2.25, u_f = 0.5*1 + 0.5*0.5 = 0.75, h_f = 0.75 silu(2.25).
    Down row d has scale (d+1)/16 (exact fp16) and codes 3 (w = 1.5 (d+1)/16):
      y_d = 32 * 1.5 (d+1)/16 * 0.75 silu(2.25) = 2.25 (d+1) silu(2.25).
    Expert 1 (not selected) has different weights.
    """
    D = F = 32
    one = 0x3C00
    down_scales = [int(np.float16((d + 1) / 16).view(np.uint16)) for d in range(D)]
    e0 = np.concatenate([
        _const_blocks(F, D, [one] * F, 0xFF),
        _const_blocks(F, D, [one] * F, 0xAA),
        _const_blocks(D, F, down_scales, 0xFF),
    ])
    e1 = np.concatenate([
        _const_blocks(F, D, [one] * F, 0x00),
        _const_blocks(F, D, [one] * F, 0x00),
        _const_blocks(D, F, [one] * D, 0x00),
    ])
    W = np.zeros((2, D), dtype=np.float32)
    W[0, 0] = W[1, 1] = 1.0
    L = oracle.Layer(fmt=oracle.FMT_Q2, d_model=D, d_ff=F, n_experts=2, top_k=1, n_shared=0,
                     shared_d_ff=F, router_w=W, router_dtype=oracle.F32, experts=[e0, e1])
    x = np.zeros((1, D))
    x[0, 0], x[0, 1] = 1.0, 0.5
    r = L.forward(x)
    s225 = 2.25 / (1.0 + math.exp(-2.25))
    want = 2.25 * np.arange(1, D + 1) * s225
    assert list(r["idx"][0]) == [0] and r["w"][0, 0] == 1.0 and r["margin"][0] == 0.5
    assert np.allclose(r["y"][0], want, rtol=1e-14, atol=0)
    assert list(r["counts"]) == [1, 0]


# ------------------------------------------------------------------ invariants on random layers
def _layer(wl, seed=0, layer=0):
    grid = synth.gen_grid(wl, seed) if wl.fmt == synth.FMT_CB35 else None
    return oracle.Layer(
        fmt=wl.fmt, d_model=wl.d_model, d_ff=wl.d_ff, n_experts=wl.n_experts, top_k=wl.top_k,
        n_shared=wl.n_shared, shared_d_ff=wl.shared_d_ff, router_w=synth.gen_router(wl, seed, layer),
        router_dtype=wl.router_dtype, bias=synth.gen_bias(wl, seed, layer),
        experts=synth.gen_layer_experts(wl, seed, layer), shared=synth.gen_shared(wl, seed, layer),
        grid=grid)


def _x(wl, n, seed=0):
    return oracle.to_f64(synth.gen_x(wl, seed, n), wl.act_dtype)


def _dense_ffn(fmt, blocks, D, F, x, grid=None):
    """Textbook SwiGLU FFN on dense fp64 matrices (numpy matmul)."""
    mat = oracle.matrix_bytes(fmt, F, D)
    Wg = oracle.dequant_matrix(fmt, blocks[:mat], F, D, grid)
    Wu = oracle.dequant_matrix(fmt, blocks[mat:2 * mat], F, D, grid)
    Wd = oracle.dequant_matrix(fmt, blocks[2 * mat:], D, F, grid)
    g, u = Wg @ x, Wu @ x
    return Wd @ (g / (1 + np.exp(-g)) * u)


@pytest.mark.parametrize("fmt", [synth.FMT_Q2, synth.FMT_CB35, synth.FMT_NVFP4])
def test_weights_sum_to_one_and_counts(fmt):
    wl = synth.small_workload(fmt=fmt)
    L = _layer(wl)
    r = L.forward(_x(wl, 6))
    assert np.all(np.abs(r["w"].sum(1) - 1) < 1e-12)
    assert r["counts"].sum() == 6 * wl.top_k
    for t in range(6):
        assert len(set(r["idx"][t])) == wl.top_k


@pytest.mark.parametrize("fmt", [synth.FMT_Q2, synth.FMT_CB35, synth.FMT_NVFP4])
def test_top1_equals_dense_expert_plus_shared(fmt):
    wl = synth.small_workload(fmt=fmt, top_k=1, d_model=128, d_ff=96, shared_d_ff=64)
    L = _layer(wl, seed=4)
    grid = L.grid
    x = _x(wl, 3, seed=4)
    r = L.forward(x)
    sh = synth.gen_shared(wl, 4, 0)
    for t in range(3):
        e = int(r["idx"][t, 0])
        assert r["w"][t, 0] == 1.0
        want = _dense_ffn(fmt, L._experts[e], 128, 96, x[t], grid) + _dense_ffn(fmt, sh, 128, 64, x[t], grid)
        assert np.allclose(r["y"][t], want, rtol=1e-12, atol=1e-12)


def test_shared_expert_counted_with_weight_one():
    # one routed expert (E = k = 1, so w = 1) and a shared expert with the same bytes: y = 2 FFN(x)
    wl = synth.small_workload(n_experts=1, top_k=1, d_model=64, d_ff=64, shared_d_ff=64)
    e = synth.gen_expert(wl, 2, 0, 0)
    L = oracle.Layer(fmt=wl.fmt, d_model=64, d_ff=64, n_experts=1, top_k=1, n_shared=1, shared_d_ff=64,
                     router_w=synth.gen_router(wl, 2, 0), router_dtype=wl.router_dtype,
                     experts=[e], shared=e)
    x = _x(wl, 2, seed=2)
    r = L.forward(x)
    for t in range(2):
        assert np.allclose(r["y"][t], 2 * _dense_ffn(wl.fmt, e, 64, 64, x[t]), rtol=1e-12, atol=1e-12)


def test_zero_input_gives_zero_output():
    wl = synth.small_workload()
    L = _layer(wl)
    r = L.forward(np.zeros((2, wl.d_model)))
    assert np.array_equal(r["y"], np.zeros((2, wl.d_model)))


def test_weighted_combine_two_experts():
    # E = k = 2: y = w0 FFN_e0 + w1 FFN_e1 with w the softmax of the two router logits
    wl = synth.small_workload(n_experts=2, top_k=2, n_shared=0, d_model=64, d_ff=32)
    L = _layer(wl, seed=7)
    x = _x(wl, 1, seed=7)[0]
    r = L.forward(x[None])
    lg = oracle.router_logits(L.router_w, L.router_dtype, L.bias, x)
    p = np.exp(lg - lg.max())
    p /= p.sum()
    want = sum(p[e] * _dense_ffn(wl.fmt, L._experts[e], 64, 32, x) for e in range(2))
    assert np.allclose(r["y"][0], want, rtol=1e-12, atol=1e-13)


def test_relabelling_experts_permutes_indices_only():
    wl = synth.small_workload()
    L = _layer(wl, seed=5)
    x = _x(wl, 4, seed=5)
    r = L.forward(x)
    perm = np.random.default_rng(0).permutation(wl.n_experts)  # new id of old expert e = inv[e]
    inv = np.argsort(perm)
    L2 = oracle.Layer(fmt=wl.fmt, d_model=wl.d_model, d_ff=wl.d_ff, n_experts=wl.n_experts,
                      top_k=wl.top_k, n_shared=wl.n_shared, shared_d_ff=wl.shared_d_ff,
                      router_w=L.router_w[perm], router_dtype=L.router_dtype, bias=L.bias[perm],
                      experts=[L._experts[int(perm[i])] for i in range(wl.n_experts)], shared=L.shared)
    r2 = L2.forward(x)
    assert np.allclose(r2["y"], r["y"], rtol=1e-12, atol=1e-13)
    for t in range(4):
        assert set(perm[r2["idx"][t]]) == set(r["idx"][t])
    assert np.array_equal(r2["counts"], r["counts"][perm])


def test_batch_invariance():
    wl = synth.small_workload()
    L = _layer(wl, seed=6)
    x = _x(wl, 5, seed=6)
    full = L.forward(x)
    for t in range(5):
        one = L.forward(x[t:t + 1])
        assert np.array_equal(one["y"][0], full["y"][t])
        assert np.array_equal(one["idx"][0], full["idx"][t])


def test_stack_one_layer_is_layer_plus_x_and_residual_chain():
    wl = synth.small_workload()
    L0, L1 = _layer(wl, 8, 0), _layer(wl, 8, 1)
    x = _x(wl, 3, seed=8)
    out1, _ = oracle.stack_forward([L0], x)
    assert np.array_equal(out1, x + L0.forward(x)["y"])
    out2, recs = oracle.stack_forward([L0, L1], x)
    x1 = x + L0.forward(x)["y"]
    assert np.array_equal(out2, x1 + L1.forward(x1)["y"])
    assert np.array_equal(recs[1]["x_in"], x1)


def test_lazy_expert_supply_matches_full_layer():
    wl = synth.small_workload()
    full = _layer(wl, 9)
    x = _x(wl, 2, seed=9)
    lazy = oracle.Layer(fmt=wl.fmt, d_model=wl.d_model, d_ff=wl.d_ff, n_experts=wl.n_experts,
                        top_k=wl.top_k, n_shared=wl.n_shared, shared_d_ff=wl.shared_d_ff,
                        router_w=full.router_w, router_dtype=full.router_dtype, bias=full.bias,
                        shared=full.shared)
    with pytest.raises(KeyError):
        lazy.forward(x)

    def supply(l, layer, need):
        for e in need:
            layer.set_expert(e, synth.gen_expert(wl, 9, 0, e))

    out, _ = oracle.stack_forward([lazy], x, supply=supply)
    assert np.array_equal(out, x + full.forward(x)["y"])


def test_bias_changes_selection():
    # a huge bias on expert 3 forces it into every token's top-k
    wl = synth.small_workload(zipf_bias=False)
    L = _layer(wl)
    b = np.zeros(wl.n_experts, dtype=np.float32)
    b[3] = 100.0
    L.bias = b
    r = L.forward(_x(wl, 4))
    assert all(3 in r["idx"][t] for t in range(4))
    assert np.all(r["idx"][:, 0] == 3)


def test_threads_do_not_change_results():
    wl = synth.small_workload()
    L = _layer(wl, 10)
    x = _x(wl, 7, seed=10)
    a = L.forward(x, n_threads=1)["y"]
    b = L.forward(x, n_threads=4)["y"]
    assert np.array_equal(a, b)


# ------------------------------------------------------------------ variants: selection-only bias, gated shared expert
def test_select_only_bias_hand_worked():
    # logits (2, 1, 0, -1), bias (0, 0, 3, 0), k = 2: scores (2, 1, 3, -1) select experts 2 then 0;
    # the weights use the unbiased logits of {2, 0} = (0, 2): w = (1, e^2) / (1 + e^2)
    l = np.array([2.0, 1.0, 0.0, -1.0])
    b = np.array([0.0, 0.0, 3.0, 0.0])
    idx, w, m = oracle.topk_select_softmax(l + b, l, 2)
    e2 = math.e ** 2
    assert list(idx) == [2, 0]
    assert w[0] == pytest.approx(1 / (1 + e2), rel=1e-15)
    assert w[1] == pytest.approx(e2 / (1 + e2), rel=1e-15)
    assert m == 1.0  # score of the 2nd pick (2) minus the best unpicked score (1)
    # with the bias in the weights too, the same selection weighs (3, 2)
    idx2, w2, _ = oracle.topk_softmax(l + b, 2)
    assert list(idx2) == [2, 0] and w2[0] == pytest.approx(math.e / (math.e + 1), rel=1e-15)


def _unit_router_layer(bias, bias_mode, D=32, E=4, k=2):
    W = np.zeros((E, D), dtype=np.float32)
    for e in range(E):
        W[e, e] = 1.0
    return oracle.Layer(fmt=oracle.FMT_Q2, d_model=D, d_ff=32, n_experts=E, top_k=k, n_shared=0,
                        shared_d_ff=32, router_w=W, router_dtype=oracle.F32, bias=bias, bias_mode=bias_mode)


def test_select_only_bias_through_the_router():
    # unit router rows: logit e = x[e]; the layer's route() applies the bias mode
    x = np.zeros((1, 32))
    x[0, :4] = [2.0, 1.0, 0.0, -1.0]
    b = np.array([0.0, 0.0, 3.0, 0.0], dtype=np.float32)
    e2 = math.e ** 2
    idx, w, m = _unit_router_layer(b, oracle.BIAS_SELECT).route(x)
    assert list(idx[0]) == [2, 0] and m[0] == 1.0
    assert np.allclose(w[0], [1 / (1 + e2), e2 / (1 + e2)], rtol=1e-15)
    idx, w, m = _unit_router_layer(b, oracle.BIAS_LOGIT).route(x)
    assert list(idx[0]) == [2, 0]
    assert np.allclose(w[0], [math.e / (math.e + 1), 1 / (math.e + 1)], rtol=1e-15)
    # a zero bias makes the two modes equal
    z = np.zeros(4, dtype=np.float32)
    a = _unit_router_layer(z, oracle.BIAS_SELECT).route(x)
    c = _unit_router_layer(z, oracle.BIAS_LOGIT).route(x)
    assert all(np.array_equal(u, v) for u, v in zip(a, c))


def test_sigmoid_closed_forms():
    assert oracle.sigmoid(0.0) == 0.5
    assert oracle.sigmoid(math.log(3.0)) == pytest.approx(0.75, rel=1e-15)
    assert oracle.sigmoid(-math.log(3.0)) == pytest.approx(0.25, rel=1e-15)
    assert oracle.sigmoid(50.0) == pytest.approx(1.0, abs=1e-15)


def _gated(wl, gate, seed=0):
    L = _layer(wl, seed)
    L2 = oracle.Layer(fmt=wl.fmt, d_model=wl.d_model, d_ff=wl.d_ff, n_experts=wl.n_experts, top_k=wl.top_k,
                      n_shared=wl.n_shared, shared_d_ff=wl.shared_d_ff, router_w=L.router_w,
                      router_dtype=wl.router_dtype, bias=L.bias, experts=synth.gen_layer_experts(wl, seed, 0),
                      shared=L.shared, shared_gate=gate)
    return L, L2


@pytest.mark.parametrize("fmt", [synth.FMT_Q2, synth.FMT_CB35])
def test_gated_shared_expert_closed_forms(fmt):
    """y_gated = y_routed + sigmoid(gate . x) o_shared: with gate = 0 the shared term is halved
    exactly; with gate = c x / |x|^2 (fp32 router dtype) the scale is sigmoid(c)."""
    wl = synth.small_workload(fmt=fmt, router_dtype=synth.DT_F32, act_dtype=synth.DT_F32)
    x = _x(wl, 1)[0]
    grid = synth.gen_grid(wl, 0) if fmt == synth.FMT_CB35 else None
    o_s = _dense_ffn(fmt, synth.gen_shared(wl, 0, 0), wl.d_model, wl.shared_d_ff, x, grid)
    for gate, scale in ((np.zeros(wl.d_model, dtype=np.float32), 0.5),
                        ((math.log(3.0) * x / np.dot(x, x)).astype(np.float32), None)):
        L, Lg = _gated(wl, gate)
        if grid is not None:
            L.grid = Lg.grid = np.ascontiguousarray(grid)
        y = L.forward(x[None])["y"][0]
        yg = Lg.forward(x[None])["y"][0]
        if scale is None:  # the fp32-rounded gate: scale from its exact dot product
            scale = 1.0 / (1.0 + math.exp(-float(np.dot(gate.astype(np.float64), x))))
            assert abs(scale - 0.75) < 1e-6
        assert np.allclose(y - yg, (1.0 - scale) * o_s, rtol=1e-9, atol=1e-12 * np.abs(o_s).max())
        assert np.array_equal(L.forward(x[None])["idx"], Lg.forward(x[None])["idx"])


# ------------------------------------------------------------------ NVFP4 blocks
@pytest.mark.parametrize("code,val", [
    (0, 0.0), (1, 0.5), (2, 1.0), (3, 1.5), (4, 2.0), (5, 3.0), (6, 4.0), (7, 6.0),
    (9, -0.5), (10, -1.0), (13, -3.0), (15, -6.0),
])
def test_e2m1_decode(code, val):
    assert oracle.e2m1_to_f64(code) == val


def test_e2m1_negative_zero():
    v = oracle.e2m1_to_f64(8)
    assert v == 0.0 and math.copysign(1.0, v) == -1.0


@pytest.mark.parametrize("b,val", [
    (0x38, 1.0), (0x40, 2.0), (0x3C, 1.5), (0x41, 2.25), (0x37, 0.9375), (0x7E, 448.0),
    (0x08, 2.0 ** -6), (0x01, 2.0 ** -9), (0x07, 7 * 2.0 ** -9), (0x00, 0.0), (0xB8, -1.0),
])
def test_e4m3_decode(b, val):
    assert oracle.e4m3_to_f64(b) == val


def test_e4m3_nan():
    assert math.isnan(oracle.e4m3_to_f64(0x7F)) and math.isnan(oracle.e4m3_to_f64(0xFF))


def test_nvfp4_block_golden():
    gd = _read_golden("nvfp4_block.txt")
    blk = np.array([int(b, 16) for b in gd["bytes"]], dtype=np.uint8)
    k = np.array([int(v) for v in gd["k"]], dtype=np.float64)
    w = oracle.dequant_block(oracle.FMT_NVFP4, blk)
    assert w.shape == (16,)
    assert np.array_equal(w, k * 2.25 / 2)


def test_nvfp4_matrix_tensor_scale_and_layout():
    """Header = the fp32 tensor scale; blocks of 16 row-major along the columns: a 2 x 32
    matrix of 4 hand-set blocks, dequantised and compared element by element."""
    g = np.array([0.75], dtype=np.float32)
    blocks = []
    for r in range(2):
        for b in range(2):
            scale = 0x38 + 8 * (2 * r + b)  # 1, 2, 4, 8 (exponent steps of one)
            codes = [(2 * r + b + i) % 8 for i in range(16)]  # positive codes
            byts = [codes[2 * j] | (codes[2 * j + 1] << 4) for j in range(8)]
            blocks.append([scale] + byts)
    mat = np.concatenate([g.view(np.uint8), np.array(blocks, dtype=np.uint8).reshape(-1)])
    assert mat.size == oracle.matrix_bytes(oracle.FMT_NVFP4, 2, 32)
    W = oracle.dequant_matrix(oracle.FMT_NVFP4, mat, 2, 32)
    e2m1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    for r in range(2):
        for b in range(2):
            s = 2.0 ** (2 * r + b)
            for i in range(16):
                assert W[r, 16 * b + i] == 0.75 * s * e2m1[(2 * r + b + i) % 8]
