"""Seeded synthetic inputs for the selective scan and the decode step.

This module only draws numbers: it holds none of the scan's arithmetic. It is
the one piece shared by the CUDA path's tests/benchmark and the fp64 oracle, so
both see the very same input values.

Recipe (one ``torch.Generator`` on the CPU, seeded per workload; the draw order
is fixed): u, delta_raw, z, B, C ~ N(0, 1) drawn in fp32 and rounded to the
storage dtype; then U ~ Uniform[lo, hi] giving delta_bias = log(expm1(U)) (so
softplus(delta_bias) = U); then D ~ N(1, 0.1) (0.1 is the standard deviation).
A[d, n] = -(n + 1) for every channel (no draw) in the workloads; parity cases
also use ``a_matrix_varied`` (A drawn per channel and state, with one
slow-decay channel) and ``tail_inputs`` (raw steps, gates and biases far out
in the tails of softplus and silu). The tiny workload keeps bias = 0 and D = 1. The decode workload draws state0 ~ N(0, 0.1) and the
per-channel parameters from ``seed``, and the inputs of step k from seed 1 + k.

The workloads stand in for Mamba layers of 130M- and 2.8B-class models
(d_state = 16, expand = 2), a long-context layer, and batched generation.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Dict, Optional

import torch


@dataclass(frozen=True)
class ScanWorkload:
    name: str
    batch: int
    dim: int
    dstate: int
    seqlen: int
    in_dtype: torch.dtype
    bias_lo: Optional[float]  # None -> delta_bias = 0
    bias_hi: Optional[float]
    d_random: bool            # False -> D = 1
    seed: int = 0

    @property
    def channel_tokens(self) -> int:
        return self.batch * self.dim * self.seqlen


@dataclass(frozen=True)
class DecodeWorkload:
    name: str
    batch: int
    dim: int
    dstate: int
    steps: int
    in_dtype: torch.dtype = torch.bfloat16
    bias_lo: float = 1e-3
    bias_hi: float = 0.1
    seed: int = 0


TINY = ScanWorkload("tiny b1 d4 L64 N4 fp32", 1, 4, 4, 64, torch.float32, None, None, False)
M130 = ScanWorkload("mamba-130m-class b8 d1536 L2048 N16 bf16", 8, 1536, 16, 2048, torch.bfloat16,
                    1e-3, 0.1, True)
M2P8 = ScanWorkload("mamba-2.8b-class b4 d5120 L4096 N16 bf16", 4, 5120, 16, 4096, torch.bfloat16,
                    1e-3, 0.1, True)
LONG = ScanWorkload("long-context b1 d2048 L131072 N16 fp32", 1, 2048, 16, 131072, torch.float32,
                    1e-4, 1e-2, True)
DECODE = DecodeWorkload("decode b256 d5120 N16 bf16 x1000 steps", 256, 5120, 16, 1000)

SCAN_WORKLOADS: Dict[str, ScanWorkload] = {"tiny": TINY, "130m": M130, "2.8b": M2P8, "long": LONG}


def scaled(w: ScanWorkload, **changes) -> ScanWorkload:
    """Same recipe with some sizes/dtype changed (used for small parity cases)."""
    d = dict(w.__dict__)
    d.update(changes)
    return ScanWorkload(**d)


def _normal(g: torch.Generator, shape, dtype: torch.dtype, std: float = 1.0, mean: float = 0.0):
    x = torch.randn(*shape, generator=g, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    if mean != 0.0:
        x.add_(mean)
    return x.to(dtype)


def _inv_softplus_uniform(g: torch.Generator, n: int, lo: float, hi: float) -> torch.Tensor:
    uni = torch.rand(n, generator=g, dtype=torch.float64) * (hi - lo) + lo
    return torch.log(torch.expm1(uni)).to(torch.float32)


def a_matrix(dim: int, dstate: int) -> torch.Tensor:
    """A[d, n] = -(n + 1): the same real diagonal transition for every channel."""
    return -torch.arange(1, dstate + 1, dtype=torch.float32).repeat(dim, 1).contiguous()


def a_matrix_varied(dim: int, dstate: int, seed: int = 0, slow_channel: bool = True) -> torch.Tensor:
    """A[d, n] = -exp(N(0, 1)) drawn independently per channel and state (so a
    wrong channel or state index into A changes the result), from its own
    generator (seed + 2000); channel dim // 2 gets A[d, n] = -1e-4 (n + 1), a
    state that decays very slowly."""
    g = torch.Generator().manual_seed(seed + 2000)
    A = -torch.exp(torch.randn(dim, dstate, generator=g, dtype=torch.float32))
    if slow_channel and dim > 0:
        A[dim // 2] = -1e-4 * torch.arange(1, dstate + 1, dtype=torch.float32)
    return A.contiguous()


def tail_inputs(inp: Dict[str, torch.Tensor], seed: int = 0, lim: float = 40.0,
                bias_lim: float = 15.0) -> Dict[str, torch.Tensor]:
    """A copy of scan inputs whose raw step and gate are Uniform[-lim, lim]
    and whose delta_bias is Uniform[-bias_lim, bias_lim] (own generator, seed
    + 3000), stored in the inputs' dtype: softplus and silu are then evaluated
    far into both tails, and exp(Delta A) both underflows and sits near 1."""
    g = torch.Generator().manual_seed(seed + 3000)
    out = dict(inp)
    dt = inp["delta"].dtype
    out["delta"] = ((torch.rand(inp["delta"].shape, generator=g) * 2 - 1) * lim).to(dt)
    out["z"] = ((torch.rand(inp["z"].shape, generator=g) * 2 - 1) * lim).to(dt)
    out["delta_bias"] = ((torch.rand(inp["delta_bias"].shape, generator=g) * 2 - 1) * bias_lim).to(torch.float32)
    return out


def scan_inputs(w: ScanWorkload, seed: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """CPU tensors: u, delta, z [b, d, L] and B, C [b, N, L] in ``w.in_dtype``;
    A [d, N], D [d], delta_bias [d] in fp32."""
    g = torch.Generator().manual_seed(w.seed if seed is None else seed)
    b, d, n, L = w.batch, w.dim, w.dstate, w.seqlen
    u = _normal(g, (b, d, L), w.in_dtype)
    delta = _normal(g, (b, d, L), w.in_dtype)
    z = _normal(g, (b, d, L), w.in_dtype)
    B = _normal(g, (b, n, L), w.in_dtype)
    C = _normal(g, (b, n, L), w.in_dtype)
    if w.bias_lo is None:
        bias = torch.zeros(d, dtype=torch.float32)
    else:
        bias = _inv_softplus_uniform(g, d, w.bias_lo, w.bias_hi)
    D = _normal(g, (d,), torch.float32, std=0.1, mean=1.0) if w.d_random else torch.ones(d)
    return dict(u=u, delta=delta, z=z, B=B, C=C, A=a_matrix(d, n), D=D, delta_bias=bias)


def conv_params(w: ScanWorkload, width: int = 4, seed: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """Parameters of the causal conv front-end for a scan workload (whose ``u``
    draw serves as the conv input x): conv_w [d, width] and conv_b [d] fp32
    ~ Uniform(-1/sqrt(width), 1/sqrt(width)) (a depthwise conv's fan-in is
    its width), and a history conv_x0 [b, d, width-1] ~ N(0, 1) in
    ``w.in_dtype``; drawn in that order from seed + 1000."""
    g = torch.Generator().manual_seed((w.seed if seed is None else seed) + 1000)
    lim = 1.0 / math.sqrt(width)
    conv_w = (torch.rand(w.dim, width, generator=g, dtype=torch.float32) * 2.0 - 1.0) * lim
    conv_b = (torch.rand(w.dim, generator=g, dtype=torch.float32) * 2.0 - 1.0) * lim
    conv_x0 = _normal(g, (w.batch, w.dim, width - 1), w.in_dtype)
    return dict(conv_w=conv_w, conv_b=conv_b, conv_x0=conv_x0)


@dataclass(frozen=True)
class SsdWorkload:
    """A Mamba-2 SSD layer: x [b, L, H, P], dt [b, L, H], B/C [b, L, G, N]."""
    name: str
    batch: int
    seqlen: int
    nheads: int
    headdim: int
    dstate: int
    ngroups: int
    in_dtype: torch.dtype = torch.bfloat16
    seed: int = 0


# Mamba-2 2.7B-class layer: d_model 2560, expand 2 -> 80 heads of 64, d_state 128.
SSD_2P7B = SsdWorkload("mamba2-2.7b-class b4 L2048 H80 P64 N128 G1 bf16", 4, 2048, 80, 64, 128, 1)


def ssd_inputs(w: SsdWorkload, seed: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """CPU tensors drawn in the order x, dt, B, C (N(0,1), stored in
    ``w.in_dtype``), then A = -U[1, 16] per head, dt_bias = log(expm1(U)) with
    U ~ U[1e-3, 0.1], D ~ N(1, 0.1) (fp32)."""
    g = torch.Generator().manual_seed(w.seed if seed is None else seed)
    b, L, H, P, N, G = w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups
    x = _normal(g, (b, L, H, P), w.in_dtype)
    dt = _normal(g, (b, L, H), w.in_dtype)
    B = _normal(g, (b, L, G, N), w.in_dtype)
    C = _normal(g, (b, L, G, N), w.in_dtype)
    A = -(1.0 + 15.0 * torch.rand(H, generator=g, dtype=torch.float32))
    dt_bias = _inv_softplus_uniform(g, H, 1e-3, 0.1)
    D = _normal(g, (H,), torch.float32, std=0.1, mean=1.0)
    return dict(x=x, dt=dt, B=B, C=C, A=A, dt_bias=dt_bias, D=D)


def decode_params(w: DecodeWorkload, varied_A: bool = False) -> Dict[str, torch.Tensor]:
    """state0 [b, d, N] fp32 ~ N(0, 0.1); A, D, delta_bias as the 130M-class
    layer (``varied_A``: A from ``a_matrix_varied`` instead)."""
    g = torch.Generator().manual_seed(w.seed)
    state0 = _normal(g, (w.batch, w.dim, w.dstate), torch.float32, std=0.1)
    bias = _inv_softplus_uniform(g, w.dim, w.bias_lo, w.bias_hi)
    D = _normal(g, (w.dim,), torch.float32, std=0.1, mean=1.0)
    A = a_matrix_varied(w.dim, w.dstate, w.seed) if varied_A else a_matrix(w.dim, w.dstate)
    return dict(state0=state0, A=A, D=D, delta_bias=bias)


def decode_step_inputs(w: DecodeWorkload, k: int) -> Dict[str, torch.Tensor]:
    """Inputs of decode step k (0-based), drawn from seed 1 + k: x, delta, z
    [b, d] and B, C [b, N] in ``w.in_dtype``."""
    g = torch.Generator().manual_seed(w.seed + 1 + k)
    b, d, n = w.batch, w.dim, w.dstate
    x = _normal(g, (b, d), w.in_dtype)
    delta = _normal(g, (b, d), w.in_dtype)
    z = _normal(g, (b, d), w.in_dtype)
    B = _normal(g, (b, n), w.in_dtype)
    C = _normal(g, (b, n), w.in_dtype)
    return dict(x=x, delta=delta, z=z, B=B, C=C)


def to_f64(t: torch.Tensor):
    """Exact widening of the stored values (bf16/fp32 -> fp64) as numpy."""
    return t.to(torch.float64).numpy()
