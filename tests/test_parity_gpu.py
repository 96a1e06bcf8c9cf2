"""Parity of the CUDA path with the fp64 oracle (needs a B200).

Every case draws seeded inputs from m3_synth, runs the library through its
C ABI (the Python binding), runs the oracle on the same stored values, and
compares element by element: relative L2 within the workload table's bound
(1e-4 for float32 io, 2e-2 for bfloat16 io with float32 accumulation), with
the per-element max-abs difference reported.
"""
import os

import numpy as np
import pytest
import torch

import m3_synth
import oracle
from tests._util import dims_of, empty_carry, f64, gpu_scan, max_abs, rel_l2, slice_bh, tol_for

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import selective_state_space_m3_b200 as m3


def _oracle_full(inp, init=None):
    args = {k: f64(v) for k, v in inp.items()}
    kw = {}
    if init is not None:
        kw = dict(init_h=f64(init.h), init_pB=f64(init.prev_B), init_pX=f64(init.prev_x))
    return oracle.scan(**args, **kw)


def _check(name, got, want, tol):
    """Relative L2 within `tol`, and every element within `tol` times the
    largest |want| of the compared block (so a local error in one tile of an
    otherwise exact block cannot hide under the L2 norm of the rest)."""
    r = rel_l2(got, want)
    ma = max_abs(got, want)
    scale = float(np.max(np.abs(want))) if np.size(want) else 0.0
    print(f"{name}: rel_l2={r:.3e} max_abs={ma:.3e} (max|want|={scale:.3e})")
    assert np.all(np.isfinite(np.asarray(got, np.float64))), name
    assert r <= tol, f"{name}: rel_l2 {r:.3e} > {tol:.1e}"
    assert ma <= tol * scale, f"{name}: max_abs {ma:.3e} > {tol:.1e} x {scale:.3e}"


# ------------------------------------------------------------ small cases --
SMALL = [
    # shape, id  -- span several chunks and a ragged tail
    (m3_synth.ScanShape(1, 256, 1, 1, 16, 16, 1, 32, "f32", 0.0, 0), "siso_tiny_full"),
    (m3_synth.ScanShape(2, 300, 4, 2, 16, 16, 2, 32, "f32", 0.0, 11), "f32_mimo_ragged"),
    (m3_synth.ScanShape(2, 333, 4, 2, 64, 128, 1, 64, "bf16", 0.0, 12), "bf16_siso_ragged"),
    (m3_synth.ScanShape(1, 200, 3, 3, 64, 128, 4, 64, "bf16", 0.0, 13), "bf16_mimo_r4"),
    (m3_synth.ScanShape(2, 260, 8, 1, 64, 128, 1, 64, "bf16", 0.0, 14), "bf16_shared_group"),
    (m3_synth.ScanShape(1, 520, 2, 2, 64, 128, 1, 128, "bf16", -1.0, 15), "bf16_long_dt"),
]


@pytest.mark.parametrize("path", ["auto", "simt"])
@pytest.mark.parametrize("shape,name", SMALL, ids=[n for _, n in SMALL])
def test_scan_matches_oracle(shape, name, path, monkeypatch):
    """Every small case on the default path (tcgen05 for bf16 N=128 P=64) and
    on the SIMT path forced."""
    if path == "simt":
        monkeypatch.setenv("M3_SCAN_PATH", "simt")
    inp = m3_synth.make_scan_inputs(shape)
    y, fin = gpu_scan(shape, inp)
    yo, ho, pBo, pXo = _oracle_full(inp)
    tol = tol_for(shape.dtype)
    _check(f"{name} y", f64(y), yo, tol)
    _check(f"{name} h", f64(fin.h), ho, tol)
    assert np.array_equal(f64(fin.prev_B), pBo)      # exact copies of stored inputs
    assert np.array_equal(f64(fin.prev_x), pXo)


@pytest.mark.parametrize("nseg", [1, 2, 3, 7])
def test_scan_segment_split_matches_oracle(nseg, monkeypatch):
    """The multi-segment path (summary, combine, main) against the oracle,
    float32 SIMT."""
    monkeypatch.setenv("M3_SCAN_NSEG", str(nseg))
    shape = m3_synth.ScanShape(2, 290, 2, 1, 16, 16, 2, 16, "f32", 0.0, 21)
    inp = m3_synth.make_scan_inputs(shape)
    init = m3_synth.make_carry(2, 2, 16, 16, 2, "f32", 21)
    init = m3.Carry(init["h"].cuda(), init["prev_B"].cuda(), init["prev_x"].cuda())
    y, fin = gpu_scan(shape, inp, init=init)
    yo, ho, _, _ = _oracle_full(inp, init)
    _check(f"nseg{nseg} y", f64(y), yo, 1e-4)
    _check(f"nseg{nseg} h", f64(fin.h), ho, 1e-4)


@pytest.mark.parametrize("R", [1, 2, 4, 8])
@pytest.mark.parametrize("nseg", [1, 3])
def test_tc_segments_and_ranks(R, nseg, monkeypatch):
    """tcgen05 path: every supported rank, one and several segments, ragged
    tail, nonzero initial carry."""
    monkeypatch.setenv("M3_SCAN_NSEG", str(nseg))
    T = 128 // R
    L = 5 * T + 7
    shape = m3_synth.ScanShape(2, L, 2, 2, 64, 128, R, 64, "bf16", 0.0, 60 + R)
    inp = m3_synth.make_scan_inputs(shape)
    c = m3_synth.make_carry(2, 2, 128, 64, R, "bf16", 60 + R, scale=0.3)
    init = m3.Carry(c["h"].cuda(), c["prev_B"].cuda(), c["prev_x"].cuda())
    d = dims_of(shape)
    plan = m3.m3_scan_plan(d)
    assert plan["path"] == "tcgen05" and plan["segments"] == nseg
    y, fin = gpu_scan(shape, inp, init=init)
    yo, ho, _, _ = _oracle_full(inp, init)
    _check(f"tc R{R} nseg{nseg} y", f64(y), yo, 2e-2)
    _check(f"tc R{R} nseg{nseg} h", f64(fin.h), ho, 2e-2)


@pytest.mark.parametrize("R", [1, 2, 4])
def test_tc_strong_decay(R):
    """Heads whose decay inside a 16-column block of the mask is far beyond
    the float range (A = -20 with dt ~ 0.7) next to ordinary heads: the
    long-tile mask takes its element-wise path for the former and the
    factored path for the latter."""
    T = 128 // R
    shape = m3_synth.ScanShape(2, 3 * T + 5, 4, 4, 64, 128, R, 64, "bf16", 0.0, 80 + R)
    inp = m3_synth.make_scan_inputs(shape)
    inp["A"] = inp["A"].clone()
    inp["A"][0] = -20.0
    inp["A"][2] = -6.0
    assert m3.m3_scan_plan(dims_of(shape))["path"] == "tcgen05"
    y, fin = gpu_scan(shape, inp)
    yo, ho, _, _ = _oracle_full(inp)
    _check(f"strong decay R{R} y", f64(y), yo, 2e-2)
    _check(f"strong decay R{R} h", f64(fin.h), ho, 2e-2)


def test_scan_with_initial_carry_bf16():
    shape = m3_synth.ScanShape(2, 190, 4, 4, 64, 128, 4, 64, "bf16", 0.0, 22)
    inp = m3_synth.make_scan_inputs(shape)
    c = m3_synth.make_carry(2, 4, 128, 64, 4, "bf16", 22, scale=0.3)
    init = m3.Carry(c["h"].cuda(), c["prev_B"].cuda(), c["prev_x"].cuda())
    y, fin = gpu_scan(shape, inp, init=init)
    yo, ho, _, _ = _oracle_full(inp, init)
    _check("carry y", f64(y), yo, 2e-2)
    _check("carry h", f64(fin.h), ho, 2e-2)


def test_split_sequence_equals_single_call():
    """scan(L1) then scan(L - L1) through the carry equals scan(L)."""
    shape = m3_synth.ScanShape(1, 400, 2, 2, 64, 128, 2, 64, "bf16", 0.0, 23)
    inp = m3_synth.make_scan_inputs(shape)
    y, fin = gpu_scan(shape, inp)
    L1 = 150
    s1 = m3_synth.shrink(shape, seqlen=L1)
    s2 = m3_synth.shrink(shape, seqlen=400 - L1)
    i1 = {k: (v[:, :L1].contiguous() if k != "A" else v) for k, v in inp.items()}
    i2 = {k: (v[:, L1:].contiguous() if k != "A" else v) for k, v in inp.items()}
    ya, fa = gpu_scan(s1, i1)
    yb, fb = gpu_scan(s2, i2, init=fa)
    yo, ho, _, _ = _oracle_full(inp)
    _check("split y", np.concatenate([f64(ya), f64(yb)], axis=1), yo, 2e-2)
    _check("split h", f64(fb.h), ho, 2e-2)
    _check("split vs single y", np.concatenate([f64(ya), f64(yb)], axis=1), f64(y), 2e-2)


@pytest.mark.parametrize("chunk", [16, 32, 64, 128])
def test_chunk_length_does_not_change_the_result(chunk):
    shape = m3_synth.ScanShape(1, 256, 2, 2, 16, 16, 1, 32, "f32", 0.0, 24)
    inp = m3_synth.make_scan_inputs(shape)
    y, fin = gpu_scan(shape, inp, chunk=chunk)
    yo, ho, _, _ = _oracle_full(inp)
    _check(f"chunk{chunk} y", f64(y), yo, 1e-4)
    _check(f"chunk{chunk} h", f64(fin.h), ho, 1e-4)


def test_empty_sequence_passes_the_carry_through():
    shape = m3_synth.ScanShape(2, 0, 2, 1, 16, 16, 1, 32, "f32", 0.0, 25)
    d = dims_of(shape)
    c = m3_synth.make_carry(2, 2, 16, 16, 1, "f32", 25)
    init = m3.Carry(c["h"].cuda(), c["prev_B"].cuda(), c["prev_x"].cuda())
    fin = empty_carry(shape)
    ws = torch.zeros(m3.m3_scan_workspace_size(d), dtype=torch.uint8, device="cuda")
    z = torch.empty(0, device="cuda")
    m3.m3_scan_fwd(d, z, z, z, z, torch.zeros(2, device="cuda"), z, z, z, ws, init=init, final_state=fin)
    torch.cuda.synchronize()
    assert torch.equal(fin.h, init.h) and torch.equal(fin.prev_B, init.prev_B)
    # batch 0: nothing to do, no error
    d0 = dims_of(m3_synth.shrink(shape, batch=0, seqlen=10))
    m3.m3_scan_fwd(d0, z, z, z, z, z, z, z, z, ws)


def test_single_token_sequence():
    shape = m3_synth.ScanShape(3, 1, 2, 2, 64, 128, 4, 64, "bf16", 0.0, 26)
    inp = m3_synth.make_scan_inputs(shape)
    y, fin = gpu_scan(shape, inp)
    yo, ho, _, _ = _oracle_full(inp)
    _check("L1 y", f64(y), yo, 2e-2)
    _check("L1 h", f64(fin.h), ho, 2e-2)


# ------------------------------------------------------------------ rope --
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_rope_bc_matches_oracle(dtype):
    shape = m3_synth.ScanShape(2, 300, 4, 2, 16, 32, 2, 32, dtype, 0.0, 31)
    inp = m3_synth.make_scan_inputs(shape)
    dev = {k: v.cuda() for k, v in inp.items()}
    d = dims_of(shape)
    io = dev["B"].dtype
    Bo = torch.empty((2, 300, 4, 2, 32), device="cuda", dtype=io)
    Co = torch.empty_like(Bo)
    ph = torch.empty((2, 300, 4, 16), device="cuda", dtype=torch.float32)
    m3.m3_rope_bc(d, dev["B"], dev["C"], dev["dt"], dev["theta"], Bo, Co, ph)
    torch.cuda.synchronize()
    Bw, Cw, Pw = oracle.rope_bc(f64(inp["B"]), f64(inp["C"]), f64(inp["dt"]), f64(inp["theta"]), nheads=4)
    tol = 1e-5 if dtype == "f32" else 2e-2
    _check("rope B", f64(Bo), Bw, tol)
    _check("rope C", f64(Co), Cw, tol)
    ang = np.angle(np.exp(1j * (f64(ph) - Pw)))
    print(f"rope phase max angular error {np.max(np.abs(ang)):.3e}")
    assert np.max(np.abs(ang)) < 1e-5
    assert np.max(np.abs(f64(ph))) <= np.pi + 1e-6


def test_rope_bc_layer_shape_sampled():
    """m3_rope_bc on the R=4 layer (8 x 4096 tokens, 32 heads, N=128, bf16) --
    the launch the bench times -- against the oracle on sampled (b, h)."""
    shape = m3_synth.MIMO_R4_LAYER
    inp = m3_synth.make_scan_inputs(shape)
    dev = {k: v.cuda() for k, v in inp.items()}
    d = dims_of(shape)
    b_, L, H, R, N = shape.batch, shape.seqlen, shape.nheads, shape.rank, shape.dstate
    Bo = torch.empty((b_, L, H, R, N), device="cuda", dtype=torch.bfloat16)
    Co = torch.empty_like(Bo)
    ph = torch.empty((b_, L, H, N // 2), device="cuda", dtype=torch.float32)
    m3.m3_rope_bc(d, dev["B"], dev["C"], dev["dt"], dev["theta"], Bo, Co, ph)
    torch.cuda.synchronize()
    for (b, h) in [(0, 0), (5, 19), (7, 31)]:
        sl = lambda v: f64(v[b:b + 1, :, h:h + 1])
        Bw, Cw, Pw = oracle.rope_bc(sl(inp["B"]), sl(inp["C"]), sl(inp["dt"]), sl(inp["theta"]), nheads=1)
        _check(f"rope layer b{b} h{h} B", f64(Bo[b:b + 1, :, h:h + 1]), Bw, 2e-2)
        _check(f"rope layer b{b} h{h} C", f64(Co[b:b + 1, :, h:h + 1]), Cw, 2e-2)
        ang = np.angle(np.exp(1j * (f64(ph[b:b + 1, :, h:h + 1]) - Pw)))
        print(f"rope layer b{b} h{h} phase max angular error {np.max(np.abs(ang)):.3e}")
        assert np.max(np.abs(ang)) < 1e-5


# ------------------------------------------------------------------ step --
@pytest.mark.parametrize("dtype,R", [("f32", 1), ("f32", 2), ("bf16", 4), ("bf16", 1), ("bf16", 8)])
def test_step_matches_oracle(dtype, R):
    dec = m3_synth.DecodeShape(batch=3, nheads=4, ngroups=2, headdim=64 if dtype == "bf16" else 16,
                               dstate=128 if dtype == "bf16" else 16, rank=R, steps=12, dtype=dtype, seed=40 + R)
    c = m3_synth.make_carry(3, 4, dec.dstate, dec.headdim, R, dtype, 40 + R, scale=0.5)
    state = m3.Carry(c["h"].cuda(), c["prev_B"].cuda(), c["prev_x"].cuda())
    A = -torch.exp(torch.linspace(-2, 1, 4))
    Ad = A.cuda()
    h, pB, pX = f64(c["h"]), f64(c["prev_B"]), f64(c["prev_x"])
    d = m3.Dims(3, 1, 4, 2, dec.headdim, dec.dstate, R, 1, m3.M3_BF16 if dtype == "bf16" else m3.M3_F32)
    tol = 1e-5 if dtype == "f32" else 2e-2
    for k in range(dec.steps):
        tok = m3_synth.make_decode_token(dec, k)
        dv = {n: v.cuda() for n, v in tok.items()}
        y = torch.empty_like(dv["x"])
        m3.m3_step(d, state, dv["x"], dv["B"], dv["C"], dv["dt"], Ad, dv["lam"], dv["theta"], y)
        yo, h, pB, pX = oracle.step(h, pB, pX, f64(tok["x"]), f64(tok["B"]), f64(tok["C"]),
                                    f64(tok["dt"]), f64(A), f64(tok["lam"]), f64(tok["theta"]))
        torch.cuda.synchronize()
        _check(f"step{k} y", f64(y), yo, tol)
    _check("step h", f64(state.h), h, 1e-4 if dtype == "bf16" else 1e-5)
    assert np.array_equal(f64(state.prev_B), pB) and np.array_equal(f64(state.prev_x), pX)


def test_scan_then_steps_equals_longer_scan():
    shape = m3_synth.ScanShape(2, 100, 2, 2, 64, 128, 4, 64, "bf16", 0.0, 50)
    inp = m3_synth.make_scan_inputs(shape)
    L0 = 90
    s0 = m3_synth.shrink(shape, seqlen=L0)
    i0 = {k: (v[:, :L0].contiguous() if k != "A" else v) for k, v in inp.items()}
    _, state = gpu_scan(s0, i0)
    d = dims_of(shape)
    ys = []
    for t in range(L0, 100):
        tok = {k: inp[k][:, t].contiguous().cuda() for k in ("x", "B", "C", "dt", "lam", "theta")}
        y = torch.empty_like(tok["x"])
        m3.m3_step(d, state, tok["x"], tok["B"], tok["C"], tok["dt"], inp["A"].cuda(), tok["lam"],
                   tok["theta"], y)
        ys.append(f64(y))
    torch.cuda.synchronize()
    yo, ho, _, _ = _oracle_full(inp)
    _check("scan+steps y", np.stack(ys, axis=1), yo[:, L0:], 2e-2)
    _check("scan+steps h", f64(state.h), ho, 2e-2)


# ----------------------------------------------- full-size, sampled outputs --
def _sampled_full(name, samples):
    shape = m3_synth.LAYERS[name]
    inp = m3_synth.make_scan_inputs(shape)
    y, fin = gpu_scan(shape, inp)
    tol = tol_for(shape.dtype)
    for (b, h) in samples:
        one = slice_bh(inp, shape, b, h)
        yo, ho, _, _ = oracle.scan(**one)
        _check(f"{name} b{b} h{h} y", f64(y[b:b + 1, :, h:h + 1]), yo, tol)
        _check(f"{name} b{b} h{h} h", f64(fin.h[b:b + 1, h:h + 1]), ho, tol)


def test_siso_tiny_full_size():
    _sampled_full("siso_tiny", [(0, 0)])


def test_siso_layer_full_size_sampled():
    # 32 sequences, one per CTA of each pass: a quarter of them, every batch row
    _sampled_full("siso_layer", [(0, 0), (0, 6), (1, 1), (1, 5), (2, 3), (2, 7), (3, 2), (3, 4)])


def test_mimo_r4_layer_full_size_sampled():
    # 256 sequences, one per CTA: one per batch row, heads spread over all 32
    _sampled_full("mimo_r4_layer", [(0, 0), (1, 9), (2, 13), (3, 17), (4, 22), (5, 26), (6, 3), (7, 31)])


def test_long_siso_full_size_sampled():
    # 32 sequences of 32768 tokens, each cut into segments: 6 of them
    _sampled_full("long_siso", [(0, 0), (0, 5), (0, 11), (0, 16), (0, 21), (0, 31)])


def test_decode_workload_from_the_prefill_carry():
    """The decode workload as specified: m3_step x 1000 tokens, 256 sequences x
    32 heads, R = 4, bf16 per-token inputs, float32 carried state initialised
    from the final state of the R = 4 layer's prefill (8 batch rows), sequence
    j taking row j mod 8; the 1000 steps captured in one CUDA graph, 64 seeded
    tokens cycled, as timed.  Each side runs the whole chain itself: the GPU
    its own prefill then the steps, the oracle its own scan then oracle.step;
    sampled sequences (every row residue) are compared at every one of the
    1000 steps, then the final carry."""
    dec = m3_synth.DECODE
    c2 = m3_synth.MIMO_R4_LAYER
    steps, pool = dec.steps, 64
    inp2 = m3_synth.make_scan_inputs(c2)
    _, fin = gpu_scan(c2, inp2)
    rows = [j % c2.batch for j in range(dec.batch)]
    state = m3.Carry(fin.h[rows].contiguous(), fin.prev_B[rows].contiguous(), fin.prev_x[rows].contiguous())
    del fin
    _, h8, pB8, pX8 = _oracle_full(inp2)                      # the oracle's own carry of all 8 rows
    sample = [0, 9, 18, 27, 36, 45, 54, 63, 100, 255]
    h, pB, pX = h8[[j % 8 for j in sample]], pB8[[j % 8 for j in sample]], pX8[[j % 8 for j in sample]]
    A = inp2["A"]
    Ad = A.cuda()
    toks = [m3_synth.make_decode_token(dec, k) for k in range(pool)]
    dtoks = [{n: v.cuda() for n, v in t.items()} for t in toks]
    d = m3.Dims(dec.batch, 1, dec.nheads, dec.ngroups, dec.headdim, dec.dstate, dec.rank, 1, m3.M3_BF16)
    ys = torch.empty((steps,) + tuple(dtoks[0]["x"].shape), dtype=torch.bfloat16, device="cuda")
    # one step outside the capture, on a throwaway copy of the carry
    warm = m3.Carry(state.h.clone(), state.prev_B.clone(), state.prev_x.clone())
    t = dtoks[0]
    m3.m3_step(d, warm, t["x"], t["B"], t["C"], t["dt"], Ad, t["lam"], t["theta"], ys[0])
    torch.cuda.synchronize()
    del warm
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        st = torch.cuda.current_stream()
        for k in range(steps):
            t = dtoks[k % pool]
            m3.m3_step(d, state, t["x"], t["B"], t["C"], t["dt"], Ad, t["lam"], t["theta"], ys[k], stream=st)
    g.replay()
    torch.cuda.synchronize()
    del g
    ys_s = f64(ys[:, sample])
    del ys
    sub = [{n: f64(v[sample]) for n, v in t.items()} for t in toks]
    Ao = f64(A)
    worst = 0.0
    for k in range(steps):
        s = sub[k % pool]
        yo, h, pB, pX = oracle.step(h, pB, pX, s["x"], s["B"], s["C"], s["dt"], Ao, s["lam"], s["theta"])
        r = rel_l2(ys_s[k], yo)
        worst = max(worst, r)
        if k % 100 == 0 or k == steps - 1 or r > 2e-2:
            _check(f"decode from prefill carry, step {k} y", ys_s[k], yo, 2e-2)
    print(f"worst per-step rel_l2 over {steps} steps: {worst:.3e}")
    assert worst <= 2e-2
    _check("decode from prefill carry h", f64(state.h)[sample], h, 2e-2)
    _check("decode from prefill carry prev_B", f64(state.prev_B)[sample], pB, 0.0)
    _check("decode from prefill carry prev_x", f64(state.prev_x)[sample], pX, 0.0)


def test_decode_1000_steps_in_one_graph_as_timed():
    """The decode workload as the bench times it: 256 sequences x 32 heads,
    R=4, 1000 m3_step calls captured in one CUDA graph, 64 seeded tokens
    cycled; sampled sequences are followed by the oracle through all 1000
    steps and the last y and the final carry are compared."""
    dec = m3_synth.DECODE
    steps, pool = 1000, 64
    c = m3_synth.make_carry(dec.batch, dec.nheads, dec.dstate, dec.headdim, dec.rank, dec.dtype,
                            dec.seed, scale=0.5)
    state = m3.Carry(c["h"].cuda(), c["prev_B"].cuda(), c["prev_x"].cuda())
    A = -torch.exp(torch.linspace(-2, 1, dec.nheads))
    Ad = A.cuda()
    toks = [m3_synth.make_decode_token(dec, k) for k in range(pool)]
    dtoks = [{n: v.cuda() for n, v in t.items()} for t in toks]
    d = m3.Dims(dec.batch, 1, dec.nheads, dec.ngroups, dec.headdim, dec.dstate, dec.rank, 1, m3.M3_BF16)
    y = torch.empty_like(dtoks[0]["x"])
    sample = list(range(3, dec.batch, 37))
    h, pB, pX = f64(c["h"])[sample], f64(c["prev_B"])[sample], f64(c["prev_x"])[sample]

    # one step outside the capture, on a throwaway copy of the carry
    warm = m3.Carry(state.h.clone(), state.prev_B.clone(), state.prev_x.clone())
    t = dtoks[0]
    m3.m3_step(d, warm, t["x"], t["B"], t["C"], t["dt"], Ad, t["lam"], t["theta"], y)
    torch.cuda.synchronize()
    del warm
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        st = torch.cuda.current_stream()
        for k in range(steps):
            t = dtoks[k % pool]
            m3.m3_step(d, state, t["x"], t["B"], t["C"], t["dt"], Ad, t["lam"], t["theta"], y, stream=st)
    g.replay()
    torch.cuda.synchronize()

    sub = [{n: f64(v[sample]) for n, v in t.items()} for t in toks]
    Ao = f64(A)
    for k in range(steps):
        s = sub[k % pool]
        yo, h, pB, pX = oracle.step(h, pB, pX, s["x"], s["B"], s["C"], s["dt"], Ao, s["lam"], s["theta"])
    _check("graph decode y(last)", f64(y)[sample], yo, 2e-2)
    _check("graph decode h", f64(state.h)[sample], h, 2e-2)
    _check("graph decode prev_B", f64(state.prev_B)[sample], pB, 0.0)
    _check("graph decode prev_x", f64(state.prev_x)[sample], pX, 0.0)
    del g


# ----------------------------------------------------------- failure path --
def test_bounded_wait_reports_timeout_and_context_survives():
    """A wait nobody satisfies gives up after its limit and reports
    M3_ERR_DEVICE_TIMEOUT through the workspace status word; the status is
    cleared on read and the device keeps working (a scan runs afterwards)."""
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    assert m3.m3_device_status(ws) == m3.M3_OK
    m3.m3_selftest_bounded_wait(ws)
    assert m3.m3_device_status(ws) == m3.M3_ERR_DEVICE_TIMEOUT
    assert m3.m3_device_status(ws) == m3.M3_OK          # read-and-clear
    shape = m3_synth.ScanShape(1, 100, 2, 2, 64, 128, 4, 64, "bf16", 0.0, 70)
    inp = m3_synth.make_scan_inputs(shape)
    y, fin = gpu_scan(shape, inp)
    yo, ho, _, _ = _oracle_full(inp)
    _check("after timeout y", f64(y), yo, 2e-2)
