"""Shared helpers of the parity tests: run the CUDA path through the binding,
run the oracle on the same stored inputs, and measure the difference."""
from __future__ import annotations

import numpy as np
import torch

import m3_synth


def rel_l2(got, want) -> float:
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    den = np.linalg.norm(want)
    return float(np.linalg.norm(got - want) / (den if den > 0 else 1.0))


def max_abs(got, want) -> float:
    return float(np.max(np.abs(np.asarray(got, np.float64) - np.asarray(want, np.float64)))) if np.size(want) else 0.0


def f64(t: torch.Tensor) -> np.ndarray:
    """Exact widening of a stored tensor (bf16 / fp32) to float64."""
    return t.detach().to("cpu", torch.float64).numpy()


def tol_for(dtype: str) -> float:
    # relative-L2 bounds of the workload table: 1e-4 for float32 io,
    # 2e-2 for bfloat16 io with float32 accumulation
    return 1e-4 if dtype == "f32" else 2e-2


def dims_of(s: m3_synth.ScanShape, **over):
    import selective_state_space_m3_b200 as m3
    d = m3.Dims(s.batch, s.seqlen, s.nheads, s.ngroups, s.headdim, s.dstate, s.rank, s.chunk,
                m3.M3_BF16 if s.dtype == "bf16" else m3.M3_F32)
    for k, v in over.items():
        setattr(d, k, v)
    return d


def empty_carry(s: m3_synth.ScanShape, device="cuda"):
    import selective_state_space_m3_b200 as m3
    io = torch.bfloat16 if s.dtype == "bf16" else torch.float32
    return m3.Carry(torch.empty((s.batch, s.nheads, s.dstate, s.headdim), device=device, dtype=torch.float32),
                    torch.empty((s.batch, s.nheads, s.rank, s.dstate), device=device, dtype=io),
                    torch.empty((s.batch, s.nheads, s.rank, s.headdim), device=device, dtype=io))


def gpu_scan(s: m3_synth.ScanShape, inp: dict, init=None, chunk=None, want_final=True):
    """Run m3_scan_fwd on device copies of ``inp``.  Returns (y, Carry)."""
    import selective_state_space_m3_b200 as m3
    dev = {k: v.cuda() for k, v in inp.items()}
    d = dims_of(s, chunk=chunk or s.chunk)
    y = torch.empty_like(dev["x"])
    ws = torch.zeros(m3.m3_scan_workspace_size(d), dtype=torch.uint8, device="cuda")
    fin = empty_carry(s) if want_final else None
    m3.m3_scan_fwd(d, dev["x"], dev["B"], dev["C"], dev["dt"], dev["A"], dev["lam"], dev["theta"],
                   y, ws, init=init, final_state=fin)
    assert m3.m3_device_status(ws) == m3.M3_OK
    torch.cuda.synchronize()
    return y, fin


def slice_bh(inp: dict, s: m3_synth.ScanShape, b: int, h: int) -> dict:
    """Inputs of one (batch, head) sequence as a 1-batch, 1-head problem."""
    g = h // (s.nheads // s.ngroups)
    return dict(x=f64(inp["x"][b:b + 1, :, h:h + 1]), B=f64(inp["B"][b:b + 1, :, g:g + 1]),
                C=f64(inp["C"][b:b + 1, :, g:g + 1]), dt=f64(inp["dt"][b:b + 1, :, h:h + 1]),
                A=f64(inp["A"][h:h + 1]), lam=f64(inp["lam"][b:b + 1, :, h:h + 1]),
                theta=f64(inp["theta"][b:b + 1, :, g:g + 1]))
