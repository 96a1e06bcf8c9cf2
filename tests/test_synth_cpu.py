"""The seeded input recipe (m3_synth) on the CPU.

The workload table's shapes, the draw order and the value distributions are
what both sides of every parity test read, so they are checked here against
an independent re-draw with the same generator and against the ranges the
transforms fix: dt = softplus(.) > 0, A = -exp(U(-2, 1)) in [-e, -e^-2],
lambda = sigmoid(.) in (0, 1), theta in [-pi, pi], bf16 storage the
round-to-nearest-even image of the float32 draw.
"""
import math

import numpy as np
import torch

import m3_synth


def test_workload_table():
    t = {k: (s.batch, s.nheads, s.ngroups, s.seqlen, s.headdim, s.dstate, s.rank, s.chunk, s.dtype, s.seed)
         for k, s in m3_synth.LAYERS.items()}
    assert t == {
        "siso_tiny": (1, 1, 1, 256, 16, 16, 1, 32, "f32", 0),
        "siso_layer": (4, 8, 1, 2048, 64, 128, 1, 64, "bf16", 1),
        "mimo_r4_layer": (8, 32, 32, 4096, 64, 128, 4, 64, "bf16", 2),
        "long_siso": (1, 32, 32, 32768, 64, 128, 1, 128, "bf16", 3),
    }
    assert m3_synth.LONG_SISO.dt_mu == -1.0 and m3_synth.MIMO_R4_LAYER.dt_mu == 0.0
    d = m3_synth.DECODE
    assert (d.batch, d.nheads, d.ngroups, d.headdim, d.dstate, d.rank, d.steps, d.dtype, d.seed) == \
        (256, 32, 32, 64, 128, 4, 1000, "bf16", 4)
    for k, s in m3_synth.LAYERS.items():
        assert m3_synth.NAMES[k].startswith(k)


def test_draw_order_and_transforms_match_an_independent_redraw():
    s = m3_synth.ScanShape(2, 9, 4, 2, 8, 6, 3, 4, "f32", -1.0, 123)
    got = m3_synth.make_scan_inputs(s)
    rng = np.random.Generator(np.random.PCG64(123))
    b, L, H, G, P, N, R = 2, 9, 4, 2, 8, 6, 3
    x = rng.standard_normal((b, L, H, R, P), dtype=np.float32)
    B = rng.standard_normal((b, L, G, R, N), dtype=np.float32)
    C = rng.standard_normal((b, L, G, R, N), dtype=np.float32)
    z_dt = rng.normal(-1.0, 1.0, size=(b, L, H))
    u_a = rng.uniform(-2.0, 1.0, size=(H,))
    z_lam = rng.normal(0.0, 1.0, size=(b, L, H))
    th = rng.uniform(-math.pi, math.pi, size=(b, L, G, N // 2))
    np.testing.assert_array_equal(got["x"].numpy(), x)
    np.testing.assert_array_equal(got["B"].numpy(), B)
    np.testing.assert_array_equal(got["C"].numpy(), C)
    np.testing.assert_allclose(got["dt"].numpy(), np.log(1 + np.exp(z_dt)), rtol=1e-6)
    np.testing.assert_allclose(got["A"].numpy(), -np.exp(u_a), rtol=1e-6)
    np.testing.assert_allclose(got["lam"].numpy(), 1 / (1 + np.exp(-z_lam)), rtol=1e-6)
    np.testing.assert_allclose(got["theta"].numpy(), th, rtol=1e-6)
    assert all(v.dtype == torch.float32 for v in got.values())


def test_ranges_and_bf16_storage():
    s = m3_synth.shrink(m3_synth.MIMO_R4_LAYER, batch=1, seqlen=64)
    got = m3_synth.make_scan_inputs(s)
    f32 = m3_synth.make_scan_inputs(m3_synth.ScanShape(**{**s.__dict__, "dtype": "f32"}))
    for k in ("x", "B", "C"):
        assert got[k].dtype == torch.bfloat16
        assert torch.equal(got[k], f32[k].to(torch.bfloat16))     # RNE image of the same draw
    assert float(got["dt"].min()) > 0
    a = got["A"].numpy()
    assert np.all(a <= -math.exp(-2) + 1e-6) and np.all(a >= -math.e - 1e-6)
    lam = got["lam"].numpy()
    assert np.all((lam > 0) & (lam < 1))
    th = got["theta"].numpy()
    assert np.all(np.abs(th) <= math.pi + 1e-6)
    xs = got["x"].float()
    assert abs(float(xs.mean())) < 0.02 and abs(float(xs.std()) - 1) < 0.02


def test_same_seed_same_draw_and_decode_tokens_differ_by_step():
    s = m3_synth.SISO_TINY
    a, b = m3_synth.make_scan_inputs(s), m3_synth.make_scan_inputs(s)
    assert all(torch.equal(a[k], b[k]) for k in a)
    t0 = m3_synth.make_decode_token(m3_synth.DECODE, 0, batch=2)
    t1 = m3_synth.make_decode_token(m3_synth.DECODE, 1, batch=2)
    assert not torch.equal(t0["x"], t1["x"])
    assert t0["x"].shape == (2, 32, 4, 64) and t0["theta"].shape == (2, 32, 64)
