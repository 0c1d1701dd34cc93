"""The seeded input generators: determinism, numpy/torch byte identity and distributions."""
import numpy as np
import pytest
import torch

import synth


def test_hash_known_values():
    # lowbias32 is a bijection with hash32(0) = 0; spot values computed by hand-checked python ints
    assert synth.hash32(0) == 0
    vals = [synth.hash32(i) for i in range(1, 1000)]
    assert len(set(vals)) == len(vals)
    arr = synth.hash32(np.arange(1, 1000, dtype=np.int64))
    assert list(arr) == vals
    t = synth.hash32(torch.arange(1, 1000, dtype=torch.int64))
    assert t.tolist() == vals


@pytest.mark.parametrize("fmt", [synth.FMT_Q2, synth.FMT_CB35])
def test_numpy_torch_expert_bytes_identical(fmt):
    wl = synth.small_workload(fmt=fmt)
    for e in (0, 5, wl.n_experts):
        ref = synth.gen_expert(wl, 11, 2, e)
        out = torch.empty((1, ref.size), dtype=torch.uint8)
        synth.gen_experts_torch(wl, 11, 2, [e], out)
        assert np.array_equal(out[0].numpy(), ref)


def test_numpy_torch_router_and_x_identical():
    for wl in (synth.DECODE, synth.TINY):
        r = synth.gen_router(wl, 3, 1)
        rt = synth.gen_router_torch(wl, 3, 1, "cpu")
        if wl.router_dtype == synth.DT_BF16:
            assert np.array_equal(rt.view(torch.int16).numpy().view(np.uint16), r)
        else:
            assert np.array_equal(rt.numpy(), r)
        x = synth.gen_x(wl, 3, 5, pass_idx=2)
        xt = synth.gen_x_torch(wl, 3, 5, 2, "cpu")
        if wl.act_dtype == synth.DT_BF16:
            assert np.array_equal(xt.view(torch.int16).numpy().view(np.uint16), x)
        else:
            assert np.array_equal(xt.numpy(), x)


def test_distributions():
    x = synth.bf16_bits_to_f32(synth.gen_x(synth.DECODE, 0, 64)).astype(np.float64)
    assert abs(x.mean()) < 0.02 and abs(x.std() - 1) < 0.02
    r = synth.bf16_bits_to_f32(synth.gen_router(synth.DECODE, 0, 0)).astype(np.float64)
    assert abs(r.std() * np.sqrt(2048) - 1) < 0.01
    s = synth.scale_table_f16().view(np.float16).astype(np.float64)
    assert 0.00499 < s.min() and s.max() < 0.02001
    e = synth.gen_expert(synth.small_workload(), 0, 0, 0).reshape(-1, 10)
    codes = np.unpackbits(e[:, 2:], bitorder="little").reshape(-1, 2)
    q = codes[:, 0] + 2 * codes[:, 1]
    assert np.allclose(np.bincount(q, minlength=4) / q.size, 0.25, atol=0.01)
    g = synth.gen_grid(synth.CODEBOOK, 0)
    assert set(np.unique(g)) == {1, 3, 5, 7, 9, 11, 13, 15}


def test_zipf_bias():
    b = synth.gen_bias(synth.DECODE, 0, 0).astype(np.float64)
    srt = np.sort(b)[::-1]
    r = np.arange(1, 513)
    h = np.sum(r ** -1.1)
    assert np.allclose(srt, 0.5 * np.log(r ** -1.1 / h), rtol=1e-6)
    assert synth.gen_bias(synth.TINY, 0, 0) is None
    assert not np.array_equal(synth.gen_bias(synth.DECODE, 0, 1), b.astype(np.float32))


def test_numpy_torch_shared_gate_identical():
    import dataclasses

    for base in (synth.DECODE, synth.TINY):
        wl = dataclasses.replace(base, shared_gate=True, n_shared=1)
        g = synth.gen_shared_gate(wl, 3, 1)
        gt = synth.gen_shared_gate_torch(wl, 3, 1, "cpu")
        assert g.shape == (wl.d_model,)
        if wl.router_dtype == synth.DT_BF16:
            assert np.array_equal(gt.view(torch.int16).numpy().view(np.uint16), g)
        else:
            assert np.array_equal(gt.numpy(), g)
    assert synth.gen_shared_gate(synth.DECODE, 3, 1) is None  # no gate unless asked for


def test_nvfp4_expert_bytes_identical_and_sized():
    wl = synth.small_workload(fmt=synth.FMT_NVFP4, d_model=256, d_ff=128, n_experts=4, top_k=2)
    assert wl.matrix_bytes() == 4 + 128 * 256 // 16 * 9
    out = torch.empty((2, wl.expert_bytes()), dtype=torch.uint8)
    synth.gen_experts_torch(wl, 3, 1, [1, 2], out)
    for i, e in enumerate((1, 2)):
        assert np.array_equal(out[i].numpy(), synth.gen_expert(wl, 3, 1, e))
    # E4M3 scales within the recipe (exponent field 5..8, sign 0), tensor scales 2^-9 (1 + u/8)
    m = synth.gen_expert(wl, 3, 1, 1)[:wl.matrix_bytes()]
    g = float(m[:4].view(np.float32)[0])
    assert g * 512 * 8 in range(8, 16)
    s = m[4:].reshape(-1, 9)[:, 0]
    assert np.all((s >> 3) >= 5) and np.all((s >> 3) <= 8) and np.all(s < 0x80)
