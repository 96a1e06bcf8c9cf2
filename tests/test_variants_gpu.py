"""Parity of the transition variants' CUDA kernels with the fp64 oracle
(needs a B200): the damping regimes (m3_scan_fwd_damped against
oracle.scan_damped) and the low-rank reflection (m3_scan_fwd_reflect against
oracle.scan_reflect), through the C ABI, on seeded inputs from m3_synth.

Tolerances are the workloads': relative L2 <= 1e-4 for float32 io and
<= 2e-2 for bfloat16 io, on y and on the final state separately, with the
per-element max-abs difference printed.  The overdamped regime uses theta
rescaled into its stable range (m3_synth.overdamped_theta).
"""
import numpy as np
import pytest
import torch

import m3_synth
import oracle
from tests._util import dims_of, empty_carry, f64, max_abs, rel_l2, tol_for

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import selective_state_space_m3_b200 as m3

REGIMES = {"under": 0, "critical": 1, "over": 2}

SHAPES = [
    (m3_synth.SISO_TINY, "siso_tiny_f32"),
    (m3_synth.shrink(m3_synth.SISO_TINY, batch=2, seqlen=77, nheads=2, ngroups=1, headdim=32, dstate=64, rank=2,
                     seed=11), "f32_r2_shared_group_N64"),
    (m3_synth.shrink(m3_synth.MIMO_R4_LAYER, batch=2, seqlen=97, nheads=3, ngroups=3), "bf16_r4_N128"),
    (m3_synth.shrink(m3_synth.SISO_LAYER, batch=1, seqlen=130, nheads=4, ngroups=2, dstate=256, seed=12),
     "bf16_r1_N256_shared"),
]


def _inputs(shape, regime):
    inp = m3_synth.make_scan_inputs(shape)
    if regime == "over":
        inp["theta"] = m3_synth.overdamped_theta(inp, shape)
    return inp


def _check(name, got, want, tol):
    r = rel_l2(got, want)
    print(f"{name}: rel_l2={r:.3e} max_abs={max_abs(got, want):.3e}")
    assert np.all(np.isfinite(np.asarray(got, np.float64))), name
    assert r <= tol, f"{name}: rel_l2 {r:.3e} > {tol:.1e}"


def _run(shape, inp, regime=None, u=None, init=None):
    dev = {k: v.cuda() for k, v in inp.items()}
    d = dims_of(shape)
    y = torch.empty_like(dev["x"])
    fin = empty_carry(shape)
    args = (dev["x"], dev["B"], dev["C"], dev["dt"], dev["A"], dev["lam"], dev["theta"], y)
    if u is None:
        m3.m3_scan_fwd_damped(d, REGIMES[regime], *args, init=init, final_state=fin)
    else:
        m3.m3_scan_fwd_reflect(d, u.cuda(), *args, init=init, final_state=fin)
    torch.cuda.synchronize()
    return y, fin


def _carry_np(c):
    return dict(init_h=f64(c.h), init_pB=f64(c.prev_B), init_pX=f64(c.prev_x))


@pytest.mark.parametrize("regime", sorted(REGIMES))
@pytest.mark.parametrize("shape,name", SHAPES, ids=[n for _, n in SHAPES])
def test_damped_matches_oracle(shape, name, regime):
    inp = _inputs(shape, regime)
    y, fin = _run(shape, inp, regime=regime)
    yo, ho, bo, xo = oracle.scan_damped(regime, **{k: f64(v) for k, v in inp.items()})
    tol = tol_for(shape.dtype)
    _check(f"{name}/{regime} y", f64(y), yo, tol)
    _check(f"{name}/{regime} h", f64(fin.h), ho, tol)
    np.testing.assert_array_equal(f64(fin.prev_B), bo)
    np.testing.assert_array_equal(f64(fin.prev_x), xo)


@pytest.mark.parametrize("shape,name", SHAPES, ids=[n for _, n in SHAPES])
def test_reflect_matches_oracle(shape, name):
    inp = m3_synth.make_scan_inputs(shape)
    u = m3_synth.make_reflect_direction(shape, zero_tokens=(0, 5, shape.seqlen - 1))
    y, fin = _run(shape, inp, u=u)
    yo, ho, bo, xo = oracle.scan_reflect(f64(u), **{k: f64(v) for k, v in inp.items()})
    tol = tol_for(shape.dtype)
    _check(f"{name}/reflect y", f64(y), yo, tol)
    _check(f"{name}/reflect h", f64(fin.h), ho, tol)
    np.testing.assert_array_equal(f64(fin.prev_B), bo)
    np.testing.assert_array_equal(f64(fin.prev_x), xo)


@pytest.mark.parametrize("variant", ["critical", "over", "reflect"])
def test_variant_with_carry_and_split_sequence(variant):
    """A random carry in, and the sequence run as two calls chained through
    the carry, both against the oracle run as one call."""
    shape = m3_synth.shrink(m3_synth.MIMO_R4_LAYER, batch=2, seqlen=90, nheads=2, ngroups=1, seed=21)
    inp = _inputs(shape, variant)
    c = m3_synth.make_carry(2, 2, 128, 64, 4, "bf16", seed=21, scale=0.5)
    init = m3.Carry(c["h"].cuda(), c["prev_B"].cuda(), c["prev_x"].cuda())
    u = m3_synth.make_reflect_direction(shape) if variant == "reflect" else None
    cut = 37
    first = {k: (v[:, :cut].contiguous() if v.dim() > 1 else v) for k, v in inp.items()}
    rest = {k: (v[:, cut:].contiguous() if v.dim() > 1 else v) for k, v in inp.items()}
    s1 = m3_synth.shrink(shape, seqlen=cut)
    s2 = m3_synth.shrink(shape, seqlen=shape.seqlen - cut)
    reg = None if u is not None else variant
    y1, f1 = _run(s1, first, regime=reg, u=None if u is None else u[:, :cut].contiguous(), init=init)
    y2, f2 = _run(s2, rest, regime=reg, u=None if u is None else u[:, cut:].contiguous(), init=f1)
    args = {k: f64(v) for k, v in inp.items()}
    if u is None:
        yo, ho, _, _ = oracle.scan_damped(variant, **args, **_carry_np(init))
    else:
        yo, ho, _, _ = oracle.scan_reflect(f64(u), **args, **_carry_np(init))
    _check(f"{variant} split y", np.concatenate([f64(y1), f64(y2)], axis=1), yo, 2e-2)
    _check(f"{variant} split h", f64(f2.h), ho, 2e-2)


def test_underdamped_regime_agrees_with_the_chunked_scan():
    """s = +1 is Mamba-3 itself: the token-by-token kernel and the chunked
    prefill (m3_scan_fwd, tensor cores) compute the same y."""
    shape = m3_synth.shrink(m3_synth.MIMO_R4_LAYER, batch=2, seqlen=256, nheads=4, ngroups=4, seed=22)
    inp = m3_synth.make_scan_inputs(shape)
    y, _ = _run(shape, inp, regime="under")
    dev = {k: v.cuda() for k, v in inp.items()}
    d = dims_of(shape)
    y2 = torch.empty_like(dev["x"])
    ws = torch.zeros(m3.m3_scan_workspace_size(d), dtype=torch.uint8, device="cuda")
    m3.m3_scan_fwd(d, dev["x"], dev["B"], dev["C"], dev["dt"], dev["A"], dev["lam"], dev["theta"], y2, ws)
    torch.cuda.synchronize()
    _check("under vs m3_scan_fwd", f64(y), f64(y2), 2e-2)


def test_variants_empty_and_single_token():
    """L = 0 passes the carry through unchanged; L = 1 is one recurrence step."""
    shape = m3_synth.shrink(m3_synth.SISO_TINY, seqlen=1, seed=23)
    inp = m3_synth.make_scan_inputs(shape)
    c = m3_synth.make_carry(1, 1, 16, 16, 1, "f32", seed=23)
    init = m3.Carry(c["h"].cuda(), c["prev_B"].cuda(), c["prev_x"].cuda())
    y, fin = _run(shape, inp, regime="critical", init=init)
    yo, ho, _, _ = oracle.scan_damped("critical", **{k: f64(v) for k, v in inp.items()}, **_carry_np(init))
    _check("L=1 y", f64(y), yo, 1e-4)
    _check("L=1 h", f64(fin.h), ho, 1e-4)
    s0 = m3_synth.shrink(shape, seqlen=0)
    inp0 = m3_synth.make_scan_inputs(s0)
    y0, f0 = _run(s0, inp0, regime="over", init=init)
    np.testing.assert_array_equal(f64(f0.h), f64(init.h))
    np.testing.assert_array_equal(f64(f0.prev_B), f64(init.prev_B))
    u0 = m3_synth.make_reflect_direction(s0)
    y0, f0 = _run(s0, inp0, u=u0, init=init)
    np.testing.assert_array_equal(f64(f0.prev_x), f64(init.prev_x))


def _sampled(regime_or_reflect, samples):
    """The SISO layer workload at full size (batch 4, 8 heads sharing one
    group, L = 2048, bf16): one launch on the whole batch, the oracle on the
    sampled (batch, head) sequences."""
    shape = m3_synth.SISO_LAYER
    inp = _inputs(shape, regime_or_reflect)
    u = m3_synth.make_reflect_direction(shape) if regime_or_reflect == "reflect" else None
    y, fin = _run(shape, inp, regime=None if u is not None else regime_or_reflect, u=u)
    yg, hg = f64(y), f64(fin.h)
    for b, h in samples:
        sl = dict(x=f64(inp["x"][b:b + 1, :, h:h + 1]), B=f64(inp["B"][b:b + 1]), C=f64(inp["C"][b:b + 1]),
                  dt=f64(inp["dt"][b:b + 1, :, h:h + 1]), A=f64(inp["A"][h:h + 1]),
                  lam=f64(inp["lam"][b:b + 1, :, h:h + 1]), theta=f64(inp["theta"][b:b + 1]))
        if u is None:
            yo, ho, _, _ = oracle.scan_damped(regime_or_reflect, **sl)
        else:
            yo, ho, _, _ = oracle.scan_reflect(f64(u[b:b + 1]), **sl)
        _check(f"siso_layer {regime_or_reflect} b{b}h{h} y", yg[b:b + 1, :, h:h + 1], yo, 2e-2)
        _check(f"siso_layer {regime_or_reflect} b{b}h{h} h", hg[b:b + 1, h:h + 1], ho, 2e-2)
        # per element: within 2e-2 of the sequence's largest |y|
        assert max_abs(yg[b:b + 1, :, h:h + 1], yo) <= 2e-2 * float(np.max(np.abs(yo)))


@pytest.mark.parametrize("variant", ["critical", "over", "reflect"])
def test_siso_layer_full_size_sampled(variant):
    _sampled(variant, [(0, 0), (1, 5), (3, 7)])
