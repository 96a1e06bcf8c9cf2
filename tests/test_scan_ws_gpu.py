"""Parity of the opt-in persistent prefill kernel (k_scan_ws.cu,
M3_TC_KERNEL=persistent) with the fp64 oracle, in both of its work splits
(needs a B200):

* ranges with hand-off: at least as many (batch, head) sequences as SMs;
  the sequences' tiles are cut into one range per CTA and a sequence cut by
  a range boundary passes its state from the CTA that ran its head to the
  one that runs its tail;
* segments: fewer sequences than SMs; each sequence is cut into segments
  whose incoming states come from the summary and combine passes.

Shapes span several tiles with a ragged last tile; every element of y and of
the final carry is compared (relative L2 <= 2e-2, bf16 io with float32
accumulation; prev_B / prev_x bit for bit).
"""
import numpy as np
import pytest
import torch

import m3_synth
import oracle
from tests._util import dims_of, empty_carry, f64, max_abs, rel_l2

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import selective_state_space_m3_b200 as m3


@pytest.fixture(autouse=True)
def _persistent_kernel(monkeypatch):
    """Every case here runs the opt-in persistent kernel."""
    monkeypatch.setenv("M3_TC_KERNEL", "persistent")


def _check(name, got, want, tol=2e-2):
    r = rel_l2(got, want)
    print(f"{name}: rel_l2={r:.3e} max_abs={max_abs(got, want):.3e}")
    assert np.all(np.isfinite(np.asarray(got, np.float64))), name
    assert r <= tol, f"{name}: rel_l2 {r:.3e} > {tol:.1e}"


def _shape(R, batch, nheads, ngroups, tiles, ragged=3, seed=40):
    T = 128 // R
    return m3_synth.shrink(m3_synth.MIMO_R4_LAYER, batch=batch, seqlen=tiles * T - ragged, nheads=nheads,
                           ngroups=ngroups, rank=R, seed=seed + R)


def _run(shape, inp, init=None, ws=None):
    dev = {k: v.cuda() for k, v in inp.items()}
    d = dims_of(shape)
    y = torch.empty_like(dev["x"])
    if ws is None:
        ws = torch.zeros(m3.m3_scan_workspace_size(d), dtype=torch.uint8, device="cuda")
    fin = empty_carry(shape)
    m3.m3_scan_fwd(d, dev["x"], dev["B"], dev["C"], dev["dt"], dev["A"], dev["lam"], dev["theta"], y, ws,
                   init=init, final_state=fin)
    assert m3.m3_device_status(ws) == m3.M3_OK
    torch.cuda.synchronize()
    return y, fin


def _oracle(inp, init=None):
    kw = {}
    if init is not None:
        kw = dict(init_h=f64(init.h), init_pB=f64(init.prev_B), init_pX=f64(init.prev_x))
    return oracle.scan(**{k: f64(v) for k, v in inp.items()}, **kw)


def _compare(tag, shape, inp, init=None):
    y, fin = _run(shape, inp, init)
    yo, ho, bo, xo = _oracle(inp, init)
    _check(f"{tag} y", f64(y), yo)
    _check(f"{tag} h", f64(fin.h), ho)
    np.testing.assert_array_equal(f64(fin.prev_B), bo)
    np.testing.assert_array_equal(f64(fin.prev_x), xo)


def _sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


@pytest.mark.parametrize("R", [4, 1, 2, 8])
def test_ranges_with_handoff_match_oracle(R):
    """160 sequences (>= the SM count) of 8 tiles, the last one ragged: the
    ranges cut most sequences between two CTAs."""
    shape = _shape(R, batch=5, nheads=32, ngroups=32, tiles=8)
    assert shape.batch * shape.nheads >= _sms()
    plan = m3.m3_scan_plan(dims_of(shape))
    assert plan["segments"] == 1 and plan["launches"] == 1 and plan["path"] == "tcgen05"
    _compare(f"ranges R={R}", shape, m3_synth.make_scan_inputs(shape))


def test_ranges_with_shared_groups_and_carry():
    """Groups shared by 4 heads, a random carry in: the hand-off carries the
    pending trapezoid term of a head's last token to its tail."""
    shape = _shape(4, batch=5, nheads=32, ngroups=8, tiles=7, ragged=0, seed=50)
    inp = m3_synth.make_scan_inputs(shape)
    c = m3_synth.make_carry(5, 32, 128, 64, 4, "bf16", seed=50, scale=0.5)
    init = m3.Carry(c["h"].cuda(), c["prev_B"].cuda(), c["prev_x"].cuda())
    _compare("ranges shared+carry", shape, inp, init)


@pytest.mark.parametrize("R", [4, 1])
@pytest.mark.parametrize("nseg", [1, 3])
def test_segments_match_oracle(R, nseg, monkeypatch):
    """Fewer sequences than SMs: one segment per CTA (forced segment counts),
    incoming states from the summary and combine passes."""
    monkeypatch.setenv("M3_SCAN_NSEG", str(nseg))
    shape = _shape(R, batch=2, nheads=3, ngroups=3, tiles=9, seed=60)
    plan = m3.m3_scan_plan(dims_of(shape))
    assert plan["segments"] == nseg
    _compare(f"segments R={R} nseg={nseg}", shape, m3_synth.make_scan_inputs(shape))


def test_planner_segments_for_few_sequences():
    """32 sequences on the SMs: the planner cuts each into segments (one CTA
    each, at most one CTA per SM in all)."""
    shape = _shape(1, batch=1, nheads=32, ngroups=32, tiles=12, seed=70)
    plan = m3.m3_scan_plan(dims_of(shape))
    assert plan["segments"] == _sms() // 32 and plan["launches"] == 3
    _compare("planner segments", shape, m3_synth.make_scan_inputs(shape))


def test_back_to_back_calls_and_graph_replay():
    """The same workspace used by consecutive calls, then the call captured in
    a CUDA graph and replayed twice: every hand-off flag is cleared by the CTA
    that consumed it, so each call (or replay) sees only its own hand-offs."""
    shape = _shape(4, batch=5, nheads=32, ngroups=32, tiles=6, seed=80)
    inp = m3_synth.make_scan_inputs(shape)
    yo, ho, _, _ = _oracle(inp)
    dev = {k: v.cuda() for k, v in inp.items()}
    d = dims_of(shape)
    ws = torch.zeros(m3.m3_scan_workspace_size(d), dtype=torch.uint8, device="cuda")
    y = torch.empty_like(dev["x"])
    fin = empty_carry(shape)

    def call(stream=None):
        m3.m3_scan_fwd(d, dev["x"], dev["B"], dev["C"], dev["dt"], dev["A"], dev["lam"], dev["theta"], y, ws,
                       final_state=fin, stream=stream)

    for i in range(3):
        y.zero_()
        call()
        torch.cuda.synchronize()
        _check(f"call {i} y", f64(y), yo)
        _check(f"call {i} h", f64(fin.h), ho)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            call(stream=s)
    for i in range(2):
        y.zero_()
        g.replay()
        torch.cuda.synchronize()
        _check(f"replay {i} y", f64(y), yo)
        _check(f"replay {i} h", f64(fin.h), ho)
    assert m3.m3_device_status(ws) == m3.M3_OK
    del g


def test_agrees_with_the_tile_kernel(monkeypatch):
    """The persistent kernel and the default tile kernel (k_scan_tc.cu) give
    the same y within the bf16 tolerance."""
    shape = _shape(4, batch=5, nheads=32, ngroups=32, tiles=5, seed=90)
    inp = m3_synth.make_scan_inputs(shape)
    y1, f1 = _run(shape, inp)
    monkeypatch.delenv("M3_TC_KERNEL")
    y2, f2 = _run(shape, inp)
    _check("persistent vs tile y", f64(y1), f64(y2))
    _check("persistent vs tile h", f64(f1.h), f64(f2.h))
