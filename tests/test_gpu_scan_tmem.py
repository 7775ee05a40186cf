"""GPU parity of the tensor-memory scan engine (MS_ENGINE_TMEM: token tiles
streamed by TMA, B/C broadcast to the lanes by a tcgen05 product) against the
fp64 oracle, through the C ABI.

Shapes cover ragged channel blocks (dim not a multiple of 8, and of the
CTA's 8W channels), ragged last tiles (seqlen a multiple of 8 but not of 32),
both CTA sizes (up to 12 and up to 18 compute warps), every polynomial share,
fp32 inputs (B/C split into three bf16 parts for the tensor cores), bf16 y,
the optional inputs, an initial state, A drawn per channel and state, and the
tails of softplus and silu. Every output is compared.
"""
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


def tmem_plan(poly8=0):
    return (4, 1, poly8, mb.MS_ENGINE_TMEM)


def case(batch, dim, L, dtype, seed, varied_A=True, tails=False):
    w = syn.scaled(syn.M130, batch=batch, dim=dim, seqlen=L, in_dtype=dtype, seed=seed)
    inp = syn.scan_inputs(w)
    if varied_A:
        inp["A"] = syn.a_matrix_varied(dim, 16, seed)
    if tails:
        inp = syn.tail_inputs(inp, seed=seed)
    return inp


def run(inp, plan, softplus=True, use_z=True, use_D=True, use_bias=True, h0=None, out_dtype=torch.float32):
    g = {k: v.to(DEV) for k, v in inp.items()}
    y, last = mb.scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"] if use_D else None,
                          g["z"] if use_z else None, g["delta_bias"] if use_bias else None, softplus,
                          initial_state=None if h0 is None else h0.to(DEV), out_dtype=out_dtype, plan=plan)
    torch.cuda.synchronize()
    yr, lr = oracle.scan(f64(inp["u"]), f64(inp["delta"]), f64(inp["A"]), f64(inp["B"]), f64(inp["C"]),
                         f64(inp["D"]) if use_D else None, f64(inp["z"]) if use_z else None,
                         f64(inp["delta_bias"]) if use_bias else None, softplus,
                         h0=None if h0 is None else f64(h0))
    return y, last, yr, lr


def compare(inp, plan, what, scaled=False, out_dtype=torch.float32, **kw):
    y, last, yr, lr = run(inp, plan, out_dtype=out_dtype, **kw)
    dt = inp["u"].dtype
    if out_dtype == torch.bfloat16:
        check_out_bf16(f64(y), yr, f"{what} y(bf16 out)")
    else:
        check(f64(y), yr, dt, f"{what} y", scaled=scaled)
    check(f64(last), lr, dt, f"{what} last_state", scaled=scaled)
    return y, last


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("batch,dim,L", [(1, 8, 8), (2, 40, 40), (3, 100, 1000), (2, 136, 64), (1, 3000, 256),
                                         (4, 5120, 96)])
def test_shapes(dtype, batch, dim, L):
    """(4, 5120) takes 18 compute warps per CTA (the large instantiation);
    (1, 3000) a ragged last CTA; L = 40 and 1000 a ragged last tile."""
    inp = case(batch, dim, L, dtype, seed=batch * 7 + dim + L)
    compare(inp, tmem_plan(0 if dtype == torch.bfloat16 else 8), f"tmem b{batch} d{dim} L{L} {dtype}")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("poly8", [0, 2, 4, 8])
def test_every_poly_share(dtype, poly8):
    inp = case(3, 136, 512, dtype, seed=31 + poly8)
    compare(inp, tmem_plan(poly8), f"tmem poly {poly8} {dtype}")


@pytest.mark.parametrize("flags", [dict(use_z=False), dict(use_D=False), dict(use_bias=False),
                                   dict(softplus=False, use_bias=False), dict(use_z=False, use_D=False)])
def test_optional_inputs(flags):
    inp = case(2, 64, 200, torch.float32, seed=41)
    if not flags.get("softplus", True):
        inp["delta"] = inp["delta"].abs() * 0.05
    compare(inp, tmem_plan(8), f"tmem {flags}", **flags)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_bf16_output(dtype):
    inp = case(2, 64, 320, dtype, seed=43)
    compare(inp, tmem_plan(0 if dtype == torch.bfloat16 else 8), f"tmem bf16 out {dtype}", out_dtype=torch.bfloat16)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_initial_state_and_resume(dtype):
    inp = case(2, 48, 704, dtype, seed=45)
    h0 = 0.3 * torch.randn(2, 48, 16, generator=torch.Generator().manual_seed(2))
    plan = tmem_plan(0 if dtype == torch.bfloat16 else 8)
    compare(inp, plan, f"tmem h0 {dtype}", h0=h0)
    # [0, 256) then [256, 704) from the returned state == [0, 704)
    m = 256
    first = {k: (v[..., :m].contiguous() if v.dim() == 3 else v) for k, v in inp.items()}
    second = {k: (v[..., m:].contiguous() if v.dim() == 3 else v) for k, v in inp.items()}
    y1, h1, _, _ = run(first, plan)
    y2, h2, _, _ = run(second, plan, h0=h1.cpu())
    yr, lr = oracle.scan(f64(inp["u"]), f64(inp["delta"]), f64(inp["A"]), f64(inp["B"]), f64(inp["C"]),
                         f64(inp["D"]), f64(inp["z"]), f64(inp["delta_bias"]), True)
    check(np.concatenate([f64(y1), f64(y2)], axis=2), yr, dtype, "tmem resume y")
    check(f64(h2), lr, dtype, "tmem resume last_state")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("poly8", [0, 8])
def test_tails(dtype, poly8):
    inp = case(2, 72, 296, dtype, seed=47, tails=True)
    compare(inp, tmem_plan(poly8), f"tmem tails {poly8} {dtype}", scaled=True)


def test_strided_rows_and_batch():
    """u, delta, z as slices of wider rows and B/C as slices of a projection
    tensor: every stride a multiple of 16 bytes, rows not dense."""
    b, d, L = 2, 56, 160
    inp = case(b, d, L, torch.bfloat16, seed=49)
    gen = torch.Generator().manual_seed(3)
    wide = {}
    for k in ("u", "delta", "z"):
        big = torch.randn(b, d + 3, L + 16, generator=gen).to(torch.bfloat16)
        big[:, :d, 8:8 + L] = inp[k]
        wide[k] = big[:, :d, 8:8 + L]
    proj = torch.randn(b, 40, L + 8, generator=gen).to(torch.bfloat16)
    proj[:, 4:20, :L] = inp["B"]
    proj[:, 20:36, :L] = inp["C"]
    sub = dict(inp, u=wide["u"], delta=wide["delta"], z=wide["z"], B=proj[:, 4:20, :L], C=proj[:, 20:36, :L])
    y, last, yr, lr = run(sub, tmem_plan(0))
    check(f64(y), yr, torch.bfloat16, "tmem strided y")
    check(f64(last), lr, torch.bfloat16, "tmem strided last_state")


def test_automatic_plan_uses_tmem_and_matches_register_engine():
    """The automatic plan takes the tensor-memory engine for the 130M-class
    shape; its result equals the register engine's up to fp32 rounding."""
    inp = case(2, 256, 512, torch.bfloat16, seed=51, varied_A=False)
    g = {k: v.to(DEV) for k, v in inp.items()}
    dims = mb.scan_dims_for(g["u"], g["delta"], g["B"], g["C"], g["z"], torch.empty(2, 256, 512, device=DEV))
    rc, pl = mb.mamba_scan_choose_plan(dims)
    assert rc == mb.MS_OK and pl.engine == mb.MS_ENGINE_TMEM
    y1, l1 = mb.scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"], g["delta_bias"], True)
    y0, l0 = mb.scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"], g["delta_bias"], True,
                         plan=(4, 1, 0, mb.MS_ENGINE_REGISTER))
    torch.cuda.synchronize()
    check_fp32(f64(y1), f64(y0), "tmem vs register y")
    check_fp32(f64(l1), f64(l0), "tmem vs register last_state")


def test_repeat_is_bitwise_deterministic():
    inp = case(2, 128, 512, torch.bfloat16, seed=53)
    y1, l1, _, _ = run(inp, tmem_plan(2))
    y2, l2, _, _ = run(inp, tmem_plan(2))
    assert torch.equal(y1, y2) and torch.equal(l1, l2)
