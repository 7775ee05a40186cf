"""GPU parity of mamba_conv_scan_fwd (the scan with the block's causal conv
front-end computed in its load stage) against the fp64 oracle's causal conv
followed by its scan, through the C ABI.

The oracle is fed the same stored x values; u stays fp64 there and fp32 in the
kernel, so y and last_state follow the scan's tolerances and u_out (rounded to
the input dtype by the kernel) is checked to one unit of that rounding.
"""
import os

import numpy as np
import pytest
import torch

import oracle
from selective_state_space_40_b200 import binding as mb
from selective_state_space_40_b200 import synthetic as syn
from parity_util import check, check_fp32, check_out_bf16, f64

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    assert mb.mamba_device_check() == mb.MS_OK
    mb.library()


def _case(w, width, seed=None, varied_A=True):
    inp = syn.scan_inputs(w, seed=seed)
    if varied_A:  # A per channel and state, one slow channel
        inp["A"] = syn.a_matrix_varied(w.dim, w.dstate, w.seed if seed is None else seed)
    cp = syn.conv_params(w, width, seed=seed)
    return inp, cp


def run_gpu(inp, cp, use_bias=True, use_x0=False, silu=True, return_u=True, plan=None,
            out_dtype=torch.float32, initial_state=None, x=None, use_z=True):
    g = {k: v.to(DEV) for k, v in inp.items()}
    c = {k: v.to(DEV) for k, v in cp.items()}
    xx = g["u"] if x is None else x.to(DEV)
    return mb.conv_scan_fwd(xx, c["conv_w"], g["delta"], g["A"], g["B"], g["C"], g["D"],
                            g["z"] if use_z else None, g["delta_bias"], True,
                            conv_b=c["conv_b"] if use_bias else None,
                            conv_x0=c["conv_x0"] if use_x0 else None, conv_silu=silu,
                            return_u=return_u, plan=plan, out_dtype=out_dtype,
                            initial_state=None if initial_state is None else initial_state.to(DEV))


def run_oracle(inp, cp, use_bias=True, use_x0=False, silu=True, use_z=True, h0=None, nthreads=1):
    return oracle.conv_scan(f64(inp["u"]), f64(cp["conv_w"]), f64(cp["conv_b"]) if use_bias else None,
                            f64(cp["conv_x0"]) if use_x0 else None, silu, f64(inp["delta"]),
                            f64(inp["A"]), f64(inp["B"]), f64(inp["C"]), f64(inp["D"]),
                            f64(inp["z"]) if use_z else None, f64(inp["delta_bias"]), True,
                            h0=None if h0 is None else f64(h0), nthreads=nthreads)


def check_u(u_gpu, u_ref, dtype, what):
    if dtype == torch.bfloat16:
        check_out_bf16(f64(u_gpu), u_ref, what)
    else:
        check_fp32(f64(u_gpu), u_ref, what)


def compare(inp, cp, what, out_dtype=torch.float32, **kw):
    okw = {k: kw[k] for k in ("use_bias", "use_x0", "silu", "use_z") if k in kw}
    y, last, u = run_gpu(inp, cp, out_dtype=out_dtype, **kw)
    torch.cuda.synchronize()
    yr, lr, ur = run_oracle(inp, cp, **okw)
    dt = inp["u"].dtype
    if out_dtype == torch.bfloat16:
        check_out_bf16(f64(y), yr, f"{what} y(bf16 out)")
    else:
        check(f64(y), yr, dt, f"{what} y")
    check(f64(last), lr, dt, f"{what} last_state")
    if u is not None:
        check_u(u, ur, dt, f"{what} u")
    return y, last, u


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("width", [1, 2, 3, 4])
@pytest.mark.parametrize("L", [5, 64, 333])
def test_widths_and_lengths(dtype, width, L):
    w = syn.scaled(syn.M130, batch=2, dim=40, seqlen=L, in_dtype=dtype, seed=7 + L + width)
    inp, cp = _case(w, width)
    compare(inp, cp, f"W={width} L={L} {dtype}", use_x0=(L % 2 == 1))


@pytest.mark.parametrize("flags", [dict(use_bias=False), dict(silu=False), dict(use_x0=True),
                                   dict(use_z=False), dict(return_u=False)])
def test_options(flags):
    w = syn.scaled(syn.M130, batch=3, dim=24, seqlen=200, in_dtype=torch.float32, seed=31)
    inp, cp = _case(w, 4)
    compare(inp, cp, f"{flags}", **flags)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("lanes", [1, 2, 4, 8])
@pytest.mark.parametrize("poly8", [0, 8])
def test_every_plan(dtype, lanes, poly8):
    w = syn.scaled(syn.M130, batch=2, dim=36, seqlen=257, in_dtype=dtype, seed=41)
    inp, cp = _case(w, 4)
    compare(inp, cp, f"plan ({lanes},1,{poly8}) {dtype}", plan=(lanes, 1, poly8), use_x0=True)


def _tmem_plan(w):
    # the plain scan's automatic plan for the same sizes: the conv front-end
    # takes the tensor-memory engine exactly where the plain scan does
    u = torch.empty(w.batch, w.dim, w.seqlen, dtype=w.in_dtype)
    B = torch.empty(w.batch, w.dstate, w.seqlen, dtype=w.in_dtype)
    y = torch.empty(w.batch, w.dim, w.seqlen)
    rc, pl = mb.mamba_scan_choose_plan(mb.scan_dims_for(u, u, B, B, u, y))
    return rc == mb.MS_OK and pl.engine == mb.MS_ENGINE_TMEM


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("width", [1, 2, 3, 4])
@pytest.mark.parametrize("L,dim", [(64, 40), (256, 100), (1024, 136)])
def test_tensor_memory_engine(dtype, width, L, dim):
    """Lengths the tensor-memory engine takes (multiples of 8), channel counts
    that leave the last CTA's block ragged, history and u_out: the conv halo
    crosses lanes and 32-token tiles."""
    w = syn.scaled(syn.M130, batch=2, dim=dim, seqlen=L, in_dtype=dtype, seed=300 + L + width)
    assert _tmem_plan(w)
    inp, cp = _case(w, width)
    compare(inp, cp, f"tensor-memory W={width} L={L} d={dim} {dtype}", use_x0=True, return_u=True)


def test_tensor_memory_identity_filter_equals_plain_scan():
    """As below, at a length the tensor-memory engine takes: u = x exactly,
    y and last_state bit for bit those of the plain scan."""
    w = syn.scaled(syn.M130, batch=2, dim=64, seqlen=304, in_dtype=torch.bfloat16, seed=49)
    assert _tmem_plan(w)
    inp = {k: v.to(DEV) for k, v in syn.scan_inputs(w).items()}
    ones = torch.ones(w.dim, 1, device=DEV)
    y1, l1, u1 = mb.conv_scan_fwd(inp["u"], ones, inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"],
                                  inp["z"], inp["delta_bias"], True, conv_silu=False, return_u=True)
    y0, l0 = mb.scan_fwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"], inp["z"],
                         inp["delta_bias"], True)
    torch.cuda.synchronize()
    assert torch.equal(u1, inp["u"])
    assert torch.equal(y1, y0) and torch.equal(l1, l0)


def test_tensor_memory_split_resume():
    """[0, m) then [m, L) with the last W-1 inputs as history, both lengths
    multiples of 8, equals the whole sequence."""
    W, m = 4, 192
    w = syn.scaled(syn.M130, batch=2, dim=40, seqlen=520, in_dtype=torch.float32, seed=57)
    inp, cp = _case(w, W)
    g = {k: v.to(DEV) for k, v in inp.items()}
    c = {k: v.to(DEV) for k, v in cp.items()}

    def part(sl, x0=None, h0=None):
        return mb.conv_scan_fwd(g["u"][:, :, sl].contiguous(), c["conv_w"], g["delta"][:, :, sl].contiguous(),
                                g["A"], g["B"][:, :, sl].contiguous(), g["C"][:, :, sl].contiguous(), g["D"],
                                g["z"][:, :, sl].contiguous(), g["delta_bias"], True, conv_b=c["conv_b"],
                                conv_x0=x0, initial_state=h0)

    y1, h1, _ = part(slice(0, m))
    x0 = g["u"][:, :, m - W + 1:m].contiguous()
    y2, h2, _ = part(slice(m, w.seqlen), x0=x0, h0=h1)
    torch.cuda.synchronize()
    yr, lr, _ = run_oracle(inp, cp)
    check_fp32(f64(torch.cat([y1, y2], dim=2)), yr, "tensor-memory split y")
    check_fp32(f64(h2), lr, "tensor-memory split last_state")


def test_bf16_output():
    w = syn.scaled(syn.M130, batch=2, dim=40, seqlen=130, in_dtype=torch.bfloat16, seed=43)
    inp, cp = _case(w, 4)
    compare(inp, cp, "bf16 out", out_dtype=torch.bfloat16)


def test_identity_filter_equals_plain_scan():
    """W = 1, w = 1, no bias, no activation: u = x, so the conv path must give
    the plain scan's result bit for bit (same arithmetic after u)."""
    w = syn.scaled(syn.M130, batch=2, dim=64, seqlen=300, in_dtype=torch.bfloat16, seed=47)
    inp = {k: v.to(DEV) for k, v in syn.scan_inputs(w).items()}
    ones = torch.ones(w.dim, 1, device=DEV)
    y1, l1, u1 = mb.conv_scan_fwd(inp["u"], ones, inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"],
                                  inp["z"], inp["delta_bias"], True, conv_silu=False, return_u=True)
    y0, l0 = mb.scan_fwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"], inp["z"],
                         inp["delta_bias"], True)
    torch.cuda.synchronize()
    assert torch.equal(u1, inp["u"])
    assert torch.equal(y1, y0) and torch.equal(l1, l0)


def test_split_resume_on_gpu():
    """conv scan of [0, m) then of [m, L) with the last W-1 inputs as history
    and last_state as initial_state equals the whole sequence."""
    W, m = 4, 197
    w = syn.scaled(syn.M130, batch=2, dim=40, seqlen=520, in_dtype=torch.float32, seed=53)
    inp, cp = _case(w, W)
    g = {k: v.to(DEV) for k, v in inp.items()}
    c = {k: v.to(DEV) for k, v in cp.items()}

    def part(sl, x0=None, h0=None):
        return mb.conv_scan_fwd(g["u"][:, :, sl].contiguous(), c["conv_w"], g["delta"][:, :, sl].contiguous(),
                                g["A"], g["B"][:, :, sl].contiguous(), g["C"][:, :, sl].contiguous(), g["D"],
                                g["z"][:, :, sl].contiguous(), g["delta_bias"], True, conv_b=c["conv_b"],
                                conv_x0=x0, initial_state=h0)

    y1, h1, _ = part(slice(0, m))
    x0 = g["u"][:, :, m - W + 1:m].contiguous()
    y2, h2, _ = part(slice(m, w.seqlen), x0=x0, h0=h1)
    torch.cuda.synchronize()
    yr, lr, _ = run_oracle(inp, cp)
    check_fp32(f64(torch.cat([y1, y2], dim=2)), yr, "split y")
    check_fp32(f64(h2), lr, "split last_state")


def test_empty_sequence_passes_state_through():
    w = syn.scaled(syn.M130, batch=2, dim=32, seqlen=0, in_dtype=torch.float32, seed=59)
    inp, cp = _case(w, 4)
    h0 = torch.randn(2, 32, 16)
    y, last, _ = run_gpu(inp, cp, initial_state=h0, return_u=False)
    torch.cuda.synchronize()
    assert y.numel() == 0 and torch.equal(last.cpu(), h0)


@pytest.mark.slow
def test_full_130m_every_output():
    """The 130M-class layer through the conv front-end at full size, in the
    benchmark's launch configuration; every element of y, last_state and u
    against the oracle's conv + scan (the config's A = -(n+1))."""
    w = syn.M130
    inp, cp = _case(w, 4, varied_A=False)
    y, last, u = run_gpu(inp, cp, return_u=True)
    torch.cuda.synchronize()
    yr, lr, ur = run_oracle(inp, cp, nthreads=max(1, min(32, os.cpu_count() or 1)))
    check(f64(y), yr, w.in_dtype, "130M conv y (every element)")
    check(f64(last), lr, w.in_dtype, "130M conv last_state (every element)")
    check_u(u, ur, w.in_dtype, "130M conv u (every element)")
