"""Seeded synthetic inputs for the Mamba-3 SSM layer scan (tests and bench).

This module holds the workload table and the random draws only -- none of the
scan's arithmetic.  Both the CUDA path's tests/bench and the fp64 oracle take
their inputs from here, so the two sides read identical stored values.

Recipe (every config):
  * generator: numpy ``Generator(PCG64(seed))``; draws in this order, each in
    C order over the layouts below: x, B, C, dt-pre, A-pre, lambda-pre, theta.
  * x, B, C ~ N(0, 1), drawn as float32 (numpy's float32 normal sampler), then
    stored as float32 (fp32 workloads) or rounded to bfloat16
    (round-to-nearest-even, via torch) for bf16 workloads.
  * dt = softplus(z), z ~ N(dt_mu, 1)   (dt_mu = 0, or -1 for long context)
  * A  = -exp(u), u ~ U(-2, 1), one value per head
  * lambda = sigmoid(z), z ~ N(0, 1)
  * theta ~ U(-pi, pi), one value per (b, t, group, rotary pair)
  dt-pre, A-pre, lambda-pre and theta are drawn in float64, transformed in
  float64 and stored as float32.

Layouts: x [b][t][h][r][p], B and C [b][t][g][r][n], dt and lambda [b][t][h],
A [h], theta [b][t][g][n/2].  Decode tokens drop the t axis.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class ScanShape:
    batch: int
    seqlen: int
    nheads: int
    ngroups: int
    headdim: int      # P
    dstate: int       # N (even: N/2 rotary pairs)
    rank: int         # R (1 = SISO)
    chunk: int        # Q
    dtype: str        # "f32" or "bf16" storage of x, B, C, y
    dt_mu: float = 0.0
    seed: int = 0


# The workloads of the Mamba-3 layer-scan study: a tiny fp32 case, three
# layers of 1.5B-scale models (seeds 1, 2, 3) and a decode case (below).
SISO_TINY = ScanShape(1, 256, 1, 1, 16, 16, 1, 32, "f32", 0.0, 0)
SISO_LAYER = ScanShape(4, 2048, 8, 1, 64, 128, 1, 64, "bf16", 0.0, 1)
MIMO_R4_LAYER = ScanShape(8, 4096, 32, 32, 64, 128, 4, 64, "bf16", 0.0, 2)
LONG_SISO = ScanShape(1, 32768, 32, 32, 64, 128, 1, 128, "bf16", -1.0, 3)
# short names (command lines) and full names (reports)
LAYERS = {"siso_tiny": SISO_TINY, "siso_layer": SISO_LAYER, "mimo_r4_layer": MIMO_R4_LAYER,
          "long_siso": LONG_SISO}
NAMES = {
    "siso_tiny": "siso_tiny_b1_h1_L256_P16_N16_Q32_f32",
    "siso_layer": "siso_layer_b4_h8_g1_L2048_P64_N128_Q64_bf16",
    "mimo_r4_layer": "mimo_r4_layer_b8_h32_L4096_P64_N128_Q64_bf16",
    "long_siso": "long_siso_b1_h32_L32768_P64_N128_Q128_bf16",
    "decode": "decode_mimo_r4_b256_h32_P64_N128_x1000",
}


@dataclasses.dataclass(frozen=True)
class DecodeShape:
    batch: int = 256
    nheads: int = 32
    ngroups: int = 32
    headdim: int = 64
    dstate: int = 128
    rank: int = 4
    steps: int = 1000
    dtype: str = "bf16"
    seed: int = 4
    # the carry starts from the final state of the MIMO R=4 layer's prefill


DECODE = DecodeShape()


def _store(a32: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a32, dtype=np.float32))
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def _softplus64(z):
    # log(1 + e^z), stable for both signs
    return np.where(z > 0, z + np.log1p(np.exp(-np.abs(z))), np.log1p(np.exp(z)))


def _sigmoid64(z):
    return 1.0 / (1.0 + np.exp(-z))


def make_scan_inputs(s: ScanShape) -> dict:
    """Draw one full-sequence input set for shape ``s`` (CPU torch tensors)."""
    rng = np.random.Generator(np.random.PCG64(s.seed))
    b, L, H, G, P, N, R = s.batch, s.seqlen, s.nheads, s.ngroups, s.headdim, s.dstate, s.rank
    x = rng.standard_normal((b, L, H, R, P), dtype=np.float32)
    B = rng.standard_normal((b, L, G, R, N), dtype=np.float32)
    C = rng.standard_normal((b, L, G, R, N), dtype=np.float32)
    dt_pre = rng.normal(s.dt_mu, 1.0, size=(b, L, H))
    a_pre = rng.uniform(-2.0, 1.0, size=(H,))
    lam_pre = rng.normal(0.0, 1.0, size=(b, L, H))
    theta = rng.uniform(-math.pi, math.pi, size=(b, L, G, N // 2))
    return {
        "x": _store(x, s.dtype),
        "B": _store(B, s.dtype),
        "C": _store(C, s.dtype),
        "dt": torch.from_numpy(_softplus64(dt_pre).astype(np.float32)),
        "A": torch.from_numpy((-np.exp(a_pre)).astype(np.float32)),
        "lam": torch.from_numpy(_sigmoid64(lam_pre).astype(np.float32)),
        "theta": torch.from_numpy(theta.astype(np.float32)),
    }


def make_decode_token(d: DecodeShape, k: int, batch: Optional[int] = None) -> dict:
    """Per-token inputs of decode step ``k`` (fresh draws, generator seeded by
    (seed, k)); distributions as the scan workloads.  ``batch`` may shrink the
    batch for small tests (the first ``batch`` rows of the same draw order are
    NOT preserved: a smaller batch is a different draw)."""
    b = d.batch if batch is None else batch
    rng = np.random.Generator(np.random.PCG64([d.seed, k]))
    H, G, P, N, R = d.nheads, d.ngroups, d.headdim, d.dstate, d.rank
    x = rng.standard_normal((b, H, R, P), dtype=np.float32)
    B = rng.standard_normal((b, G, R, N), dtype=np.float32)
    C = rng.standard_normal((b, G, R, N), dtype=np.float32)
    dt_pre = rng.normal(0.0, 1.0, size=(b, H))
    lam_pre = rng.normal(0.0, 1.0, size=(b, H))
    theta = rng.uniform(-math.pi, math.pi, size=(b, G, N // 2))
    return {
        "x": _store(x, d.dtype),
        "B": _store(B, d.dtype),
        "C": _store(C, d.dtype),
        "dt": torch.from_numpy(_softplus64(dt_pre).astype(np.float32)),
        "lam": torch.from_numpy(_sigmoid64(lam_pre).astype(np.float32)),
        "theta": torch.from_numpy(theta.astype(np.float32)),
    }


def make_carry(batch: int, nheads: int, dstate: int, headdim: int, rank: int,
               dtype: str, seed: int, scale: float = 1.0) -> dict:
    """A random carry (h fp32 ~ N(0, scale^2); prev_B, prev_x ~ N(0,1) in the io
    dtype) for continuation tests."""
    rng = np.random.Generator(np.random.PCG64([seed, 7919]))
    h = rng.standard_normal((batch, nheads, dstate, headdim), dtype=np.float32) * np.float32(scale)
    pB = rng.standard_normal((batch, nheads, rank, dstate), dtype=np.float32)
    pX = rng.standard_normal((batch, nheads, rank, headdim), dtype=np.float32)
    return {"h": torch.from_numpy(h), "prev_B": _store(pB, dtype), "prev_x": _store(pX, dtype)}


def make_reflect_direction(s: ScanShape, zero_tokens=()) -> torch.Tensor:
    """Reflection directions u [b][t][g][n] for the low-rank reflection
    variant: N(0, 1) draws (generator seeded by (seed, 4099)), stored in the
    io dtype; the tokens listed in ``zero_tokens`` get u = 0 (no reflection).
    Only the direction of u matters to the method."""
    rng = np.random.Generator(np.random.PCG64([s.seed, 4099]))
    u = rng.standard_normal((s.batch, s.seqlen, s.ngroups, s.dstate), dtype=np.float32)
    for t in zero_tokens:
        if 0 <= t < s.seqlen:
            u[:, t] = 0.0
    return _store(u, s.dtype)


def overdamped_theta(inp: dict, s: ScanShape, margin: float = 0.9) -> torch.Tensor:
    """theta rescaled for the overdamped regime: theta ~ U(-pi, pi) mapped to
    U(-margin m, margin m) with m the smallest |A| of the group's heads, so
    that every pair keeps both eigenvalues A +- theta below zero (the regime's
    stable range).  Returns a new float32 tensor."""
    H, G = s.nheads, s.ngroups
    A = inp["A"].to(torch.float64).abs().reshape(G, H // G).min(dim=1).values      # per group
    th = inp["theta"].to(torch.float64) / math.pi * margin * A.reshape(1, 1, G, 1)
    return th.to(torch.float32).contiguous()


def shrink(s: ScanShape, **kw) -> ScanShape:
    """Same distributions and seed, other sizes (parity cases the oracle runs
    in seconds)."""
    return dataclasses.replace(s, **kw)
