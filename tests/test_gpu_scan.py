"""GPU parity of mamba_scan_fwd against the fp64 oracle (called through the C ABI).

Small cases are compared element by element in full, most of them with A drawn
per channel and state (so a wrong channel or state index into A fails) and
some with raw steps, gates and biases far in the tails of softplus and silu.
The full-size workloads (130M-class, 2.8B-class, long context) are run whole
on the GPU in the launch configuration the benchmark uses, and every output
(all of y and last_state) is compared with the oracle, which runs over blocks
of channels on the host's cores.
"""
import os

import numpy as np
import pytest
import torch

import oracle
from selective_state_space_40_b200 import binding as mb
from selective_state_space_40_b200 import synthetic as syn
from parity_util import StreamCheck, check, check_fp32, check_out_bf16, f64

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    assert mb.mamba_device_check() == mb.MS_OK
    mb.library()


def _to_dev(inp):
    return {k: v.to(DEV) for k, v in inp.items()}


def varied(inp, seed=0):
    """The same inputs with A drawn per channel and state (one slow channel)."""
    out = dict(inp)
    out["A"] = syn.a_matrix_varied(inp["A"].shape[0], inp["A"].shape[1], seed)
    return out


ORACLE_THREADS = max(1, min(32, os.cpu_count() or 1))


def run_gpu(inp, softplus=True, use_z=True, use_D=True, use_bias=True, initial_state=None,
            out_dtype=torch.float32, plan=None):
    g = _to_dev(inp)
    y, last = mb.scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"],
                          g["D"] if use_D else None, g["z"] if use_z else None,
                          g["delta_bias"] if use_bias else None, softplus,
                          initial_state=None if initial_state is None else initial_state.to(DEV),
                          out_dtype=out_dtype, plan=plan)
    torch.cuda.synchronize()
    return y, last


def run_oracle(inp, softplus=True, use_z=True, use_D=True, use_bias=True, h0=None):
    return oracle.scan(f64(inp["u"]), f64(inp["delta"]), f64(inp["A"]), f64(inp["B"]), f64(inp["C"]),
                       f64(inp["D"]) if use_D else None, f64(inp["z"]) if use_z else None,
                       f64(inp["delta_bias"]) if use_bias else None, softplus,
                       h0=None if h0 is None else f64(h0))


def compare_full(inp, what, scaled=False, **kw):
    okw = {k: kw[k] for k in ("softplus", "use_z", "use_D", "use_bias") if k in kw}
    h0 = kw.get("initial_state")
    y, last = run_gpu(inp, **kw)
    yr, lr = run_oracle(inp, h0=h0, **okw)
    dt = inp["u"].dtype
    if kw.get("out_dtype", torch.float32) == torch.bfloat16:
        check_out_bf16(f64(y), yr, f"{what} y(bf16 out)")
    else:
        check(f64(y), yr, dt, f"{what} y", scaled=scaled)
    check(f64(last), lr, dt, f"{what} last_state", scaled=scaled)
    return y, last


# ------------------------------------------------------------ small cases ---

def test_tiny_workload_full():
    """b1 d4 L64 N4 fp32, softplus on, bias 0, D 1: every output."""
    compare_full(syn.scan_inputs(syn.TINY), "tiny")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("L", [1, 7, 63, 64, 65, 1000])
def test_lengths_ragged(dtype, L):
    w = syn.scaled(syn.M130, batch=2, dim=40, seqlen=L, in_dtype=dtype, seed=L)
    compare_full(varied(syn.scan_inputs(w), L), f"L={L} {dtype}")


@pytest.mark.parametrize("N", [1, 2, 3, 4, 9, 16])
def test_dstate(N):
    w = syn.scaled(syn.M130, batch=2, dim=24, dstate=N, seqlen=300, in_dtype=torch.float32, seed=100 + N)
    compare_full(varied(syn.scan_inputs(w), N), f"N={N}")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("lanes,chunks", [(1, 1), (1, 2), (2, 1), (2, 2), (4, 1), (4, 2), (8, 1)])
@pytest.mark.parametrize("poly", [0, 2, 4, 8])
def test_every_plan(dtype, lanes, chunks, poly):
    w = syn.scaled(syn.M130, batch=3, dim=136, seqlen=517, in_dtype=dtype, seed=7)
    compare_full(varied(syn.scan_inputs(w), 7), f"plan {lanes}/{chunks}/{poly} {dtype}",
                 plan=(lanes, chunks, poly))


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("lanes,chunks", [(1, 1), (2, 2), (4, 1), (8, 1)])
@pytest.mark.parametrize("poly", [0, 8])
def test_tails(dtype, lanes, chunks, poly):
    """Raw steps and gates in [-40, 40], biases in [-15, 15], A per channel:
    softplus on both of its branches and far into both tails, silu at large
    |z|, exp(Delta A) from 1 down to underflow (the polynomial's clamp)."""
    w = syn.scaled(syn.M130, batch=2, dim=72, seqlen=300, in_dtype=dtype, seed=17)
    inp = syn.tail_inputs(varied(syn.scan_inputs(w), 17), seed=17)
    compare_full(inp, f"tails {lanes}/{chunks}/{poly} {dtype}", scaled=True, plan=(lanes, chunks, poly))


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_tails_automatic_plan(dtype):
    w = syn.scaled(syn.M130, batch=2, dim=200, seqlen=1000, in_dtype=dtype, seed=18)
    inp = syn.tail_inputs(varied(syn.scan_inputs(w), 18), seed=18)
    compare_full(inp, f"tails auto {dtype}", scaled=True)


@pytest.mark.parametrize("flags", [
    dict(use_z=False), dict(use_D=False), dict(use_bias=False), dict(softplus=False, use_bias=False),
    dict(use_z=False, use_D=False, use_bias=False)])
def test_optional_inputs(flags):
    w = syn.scaled(syn.M130, batch=2, dim=64, seqlen=200, in_dtype=torch.float32, seed=3)
    inp = varied(syn.scan_inputs(w), 3)
    if not flags.get("softplus", True):
        inp["delta"] = inp["delta"].abs() * 0.05  # keep the step positive without softplus
    compare_full(inp, f"flags {flags}", **flags)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_bf16_output(dtype):
    w = syn.scaled(syn.M130, batch=2, dim=64, seqlen=333, in_dtype=dtype, seed=5)
    compare_full(syn.scan_inputs(w), f"bf16 out {dtype}", out_dtype=torch.bfloat16)


def test_initial_state_and_split():
    w = syn.scaled(syn.M130, batch=2, dim=48, seqlen=700, in_dtype=torch.float32, seed=9)
    inp = varied(syn.scan_inputs(w), 9)
    h0 = torch.randn(2, 48, 16, generator=torch.Generator().manual_seed(1)) * 0.3
    compare_full(inp, "initial_state", initial_state=h0)
    # scan [0, m) then [m, L) from the returned state == scan [0, L)
    m = 261
    first = {k: (v[..., :m].contiguous() if v.dim() == 3 else v) for k, v in inp.items()}
    second = {k: (v[..., m:].contiguous() if v.dim() == 3 else v) for k, v in inp.items()}
    y1, h1 = run_gpu(first)
    y2, h2 = run_gpu(second, initial_state=h1.cpu())
    yr, lr = run_oracle(inp)
    check_fp32(np.concatenate([f64(y1), f64(y2)], axis=2), yr, "split y")
    check_fp32(f64(h2), lr, "split last_state")


def test_zero_B_gives_skip_only():
    w = syn.scaled(syn.M130, batch=2, dim=40, seqlen=129, in_dtype=torch.float32, seed=4)
    inp = syn.scan_inputs(w)
    inp["B"] = torch.zeros_like(inp["B"])
    y, last = compare_full(inp, "B=0")
    assert float(last.abs().max()) == 0.0


def test_very_slow_decay():
    """delta_bias very negative: A_bar within ~1e-5 of 1 for the slowest state."""
    w = syn.scaled(syn.LONG, dim=32, seqlen=4096, seed=11)
    inp = syn.scan_inputs(w)
    inp["delta_bias"] = torch.full_like(inp["delta_bias"], -11.0)
    compare_full(inp, "slow decay")


def test_noncontiguous_and_misaligned():
    b, d, L, N = 2, 40, 150, 16
    gen = torch.Generator().manual_seed(21)
    big = torch.randn(b, d, L + 5, generator=gen)
    inp = syn.scan_inputs(syn.scaled(syn.M130, batch=b, dim=d, seqlen=L, in_dtype=torch.float32, seed=21))
    # u: rows padded (d stride L+5) and starting one element in -> no vector loads
    inp["u"] = big[:, :, 1:L + 1]
    y, last = run_gpu(inp)
    yr, lr = run_oracle(inp)
    check_fp32(f64(y), yr, "strided u")
    check_fp32(f64(last), lr, "strided u state")


def test_empty_and_zero_length():
    w = syn.scaled(syn.M130, batch=2, dim=8, seqlen=0, in_dtype=torch.float32)
    inp = _to_dev(syn.scan_inputs(w))
    h0 = torch.randn(2, 8, 16, device=DEV)
    y, last = mb.scan_fwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"], inp["z"],
                          inp["delta_bias"], True, initial_state=h0)
    torch.cuda.synchronize()
    assert y.numel() == 0 and torch.equal(last, h0)
    w = syn.scaled(syn.M130, batch=0, dim=8, seqlen=16, in_dtype=torch.float32)
    inp = _to_dev(syn.scan_inputs(w))
    y, last = mb.scan_fwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"])
    assert y.numel() == 0


def test_repeat_is_bitwise_deterministic():
    w = syn.scaled(syn.M130, batch=2, dim=128, seqlen=512, seed=2)
    inp = syn.scan_inputs(w)
    y1, l1 = run_gpu(inp)
    y2, l2 = run_gpu(inp)
    assert torch.equal(y1, y2) and torch.equal(l1, l2)


# ------------------------------------------------- full-size workloads ----

def full_parity(w, block):
    """The whole workload on the GPU (automatic plan, as benchmarked); every
    element of y and last_state against the oracle, run over blocks of
    `block` channels (all batch rows) on the host's cores."""
    inp = syn.scan_inputs(w)
    y, last = run_gpu(inp)
    y, last = y.cpu(), last.cpu()
    cy = StreamCheck(w.in_dtype, f"{w.name} y (every element)")
    cl = StreamCheck(w.in_dtype, f"{w.name} last_state (every element)")
    for d0 in range(0, w.dim, block):
        d1 = min(w.dim, d0 + block)
        yr, lr = oracle.scan(f64(inp["u"][:, d0:d1]), f64(inp["delta"][:, d0:d1]), f64(inp["A"][d0:d1]),
                             f64(inp["B"]), f64(inp["C"]), f64(inp["D"][d0:d1]), f64(inp["z"][:, d0:d1]),
                             f64(inp["delta_bias"][d0:d1]), True, nthreads=ORACLE_THREADS)
        cy.add(f64(y[:, d0:d1]), yr)
        cl.add(f64(last[:, d0:d1]), lr)
    cy.finish()
    cl.finish()


@pytest.mark.slow
def test_full_130m_every_output():
    full_parity(syn.M130, 768)


@pytest.mark.slow
def test_full_2p8b_every_output():
    full_parity(syn.M2P8, 512)


@pytest.mark.slow
def test_full_long_context_every_output():
    full_parity(syn.LONG, 128)


# ------------------------------------------------------ sequence split ------

@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("b,d,L", [(1, 64, 20000), (2, 40, 9000), (1, 128, 16384)])
def test_sequence_split_against_oracle(dtype, b, d, L):
    """Few channels and a long sequence: mamba_scan_fwd splits each row into
    segments (ragged last segment for 20000 and 9000 tokens, equal segments
    for 16384), chains the carries and rescans; every output is checked."""
    w = syn.scaled(syn.LONG, batch=b, dim=d, seqlen=L, in_dtype=dtype, seed=L + d)
    inp = varied(syn.scan_inputs(w), L + d)
    dims = mb.scan_dims_for(inp["u"], inp["delta"], inp["B"], inp["C"], inp["z"],
                            torch.empty(b, d, L))
    assert mb.mamba_scan_workspace_size(dims) > 0  # the split path runs
    h0 = 0.5 * torch.randn(b, d, 16, generator=torch.Generator().manual_seed(4))
    compare_full(inp, f"split b{b} d{d} L{L} {dtype}", initial_state=h0)


@pytest.mark.parametrize("flags", [dict(use_z=False), dict(use_D=False), dict(use_bias=False)])
def test_sequence_split_options(flags):
    w = syn.scaled(syn.LONG, batch=1, dim=48, seqlen=12000, in_dtype=torch.float32, seed=77)
    compare_full(varied(syn.scan_inputs(w), 77), f"split {flags}", **flags)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_sequence_split_tails(dtype):
    w = syn.scaled(syn.LONG, batch=1, dim=64, seqlen=10000, in_dtype=dtype, seed=79)
    inp = syn.tail_inputs(varied(syn.scan_inputs(w), 79), seed=79)
    compare_full(inp, f"split tails {dtype}", scaled=True)


def test_sequence_split_matches_unsplit_plan():
    """The split result equals an explicit (never split) plan up to rounding."""
    w = syn.scaled(syn.LONG, batch=1, dim=96, seqlen=16384, in_dtype=torch.bfloat16, seed=78)
    inp = syn.scan_inputs(w)
    y1, l1 = run_gpu(inp)
    y0, l0 = run_gpu(inp, plan=(8, 1, 0))
    check_fp32(f64(y1), f64(y0), "split vs unsplit y")
    check_fp32(f64(l1), f64(l0), "split vs unsplit last_state")
