"""GPU parity of mamba_state_update (decode) against the fp64 oracle.

Most cases use A drawn per channel and state (one slow channel) so that a
wrong channel or state index into A fails; one case puts the raw step, gate
and bias far in the tails. The full-size decode (b256 d5120, 1000 steps) is
compared on every y of every step and on the whole final state, with the
oracle split over batch rows on the host's cores.
"""
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import oracle
from selective_state_space_40_b200 import binding as mb
from selective_state_space_40_b200 import synthetic as syn
from parity_util import StreamCheck, check, check_bf16, check_fp32, check_out_bf16, f64

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    mb.library()


def _step_gpu(state, inp, params, use_z=True, use_D=True, use_bias=True, softplus=True):
    return mb.state_update(state, inp["x"].to(DEV), inp["delta"].to(DEV), params["A"],
                           inp["B"].to(DEV), inp["C"].to(DEV), params["D"] if use_D else None,
                           inp["z"].to(DEV) if use_z else None,
                           params["delta_bias"] if use_bias else None, softplus)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("N", [1, 3, 4, 5, 16])
def test_small_steps_full(dtype, N):
    w = syn.DecodeWorkload("small", batch=3, dim=37, dstate=N, steps=20, in_dtype=dtype)
    p = syn.decode_params(w, varied_A=True)
    params = {k: v.to(DEV) for k, v in p.items()}
    state = params["state0"].clone()
    h = f64(p["state0"])
    for k in range(w.steps):
        inp = syn.decode_step_inputs(w, k)
        y = _step_gpu(state, inp, params)
        yr, h = oracle.state_update(h, f64(inp["x"]), f64(inp["delta"]), f64(p["A"]), f64(inp["B"]),
                                    f64(inp["C"]), f64(p["D"]), f64(inp["z"]), f64(p["delta_bias"]), True)
        torch.cuda.synchronize()
        check(f64(y), yr, dtype, f"step {k} y")
    check(f64(state), h, dtype, "final state")


@pytest.mark.parametrize("flags", [dict(use_z=False), dict(use_D=False), dict(use_bias=False)])
def test_optional_inputs(flags):
    w = syn.DecodeWorkload("small", batch=4, dim=64, dstate=16, steps=5, in_dtype=torch.float32)
    p = syn.decode_params(w, varied_A=True)
    params = {k: v.to(DEV) for k, v in p.items()}
    state = params["state0"].clone()
    h = f64(p["state0"])
    for k in range(w.steps):
        inp = syn.decode_step_inputs(w, k)
        y = _step_gpu(state, inp, params, **flags)
        yr, h = oracle.state_update(
            h, f64(inp["x"]), f64(inp["delta"]), f64(p["A"]), f64(inp["B"]), f64(inp["C"]),
            None if not flags.get("use_D", True) else f64(p["D"]),
            None if not flags.get("use_z", True) else f64(inp["z"]),
            None if not flags.get("use_bias", True) else f64(p["delta_bias"]), True)
        torch.cuda.synchronize()
        check_fp32(f64(y), yr, f"{flags} y")
    check_fp32(f64(state), h, f"{flags} state")


def test_strided_state():
    """State rows padded (d stride 20 instead of 16): scalar path."""
    w = syn.DecodeWorkload("small", batch=2, dim=16, dstate=16, steps=3, in_dtype=torch.float32)
    p = syn.decode_params(w)
    params = {k: v.to(DEV) for k, v in p.items()}
    big = torch.zeros(2, 16, 20, device=DEV)
    big[:, :, 2:18] = params["state0"]
    state = big[:, :, 2:18]
    h = f64(p["state0"])
    for k in range(w.steps):
        inp = syn.decode_step_inputs(w, k)
        y = _step_gpu(state, inp, params)
        yr, h = oracle.state_update(h, f64(inp["x"]), f64(inp["delta"]), f64(p["A"]), f64(inp["B"]),
                                    f64(inp["C"]), f64(p["D"]), f64(inp["z"]), f64(p["delta_bias"]), True)
        torch.cuda.synchronize()
        check_fp32(f64(y), yr, "strided y")
    check_fp32(f64(state), h, "strided state")
    assert float(big[:, :, :2].abs().max()) == 0.0 and float(big[:, :, 18:].abs().max()) == 0.0


def test_scan_equals_decode_on_gpu():
    """L decode steps from zero give the scan's y and last_state."""
    w = syn.scaled(syn.M130, batch=2, dim=40, seqlen=50, in_dtype=torch.float32, seed=8)
    inp = syn.scan_inputs(w)
    g = {k: v.to(DEV) for k, v in inp.items()}
    y_scan, last = mb.scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"],
                               g["delta_bias"], True)
    state = torch.zeros(2, 40, 16, device=DEV)
    ys = []
    for t in range(w.seqlen):
        ys.append(mb.state_update(state, g["u"][:, :, t].contiguous(), g["delta"][:, :, t].contiguous(),
                                  g["A"], g["B"][:, :, t].contiguous(), g["C"][:, :, t].contiguous(),
                                  g["D"], g["z"][:, :, t].contiguous(), g["delta_bias"], True))
    torch.cuda.synchronize()
    yr, lr = oracle.scan(f64(inp["u"]), f64(inp["delta"]), f64(inp["A"]), f64(inp["B"]), f64(inp["C"]),
                         f64(inp["D"]), f64(inp["z"]), f64(inp["delta_bias"]), True)
    check_fp32(f64(torch.stack(ys, dim=2)), yr, "decode-as-scan y")
    check_fp32(f64(state), lr, "decode-as-scan state")
    check_fp32(f64(y_scan), yr, "scan y")


@pytest.mark.slow
def test_full_decode_1000_steps_every_output():
    """b256 d5120 N16, 1000 steps on the GPU at full size; the oracle follows
    every channel through every step: every y of every step and the whole
    final state are compared."""
    w = syn.DECODE
    p = syn.decode_params(w)
    params = {k: v.to(DEV) for k, v in p.items()}
    state = params["state0"].clone()
    h = f64(p["state0"])
    A, D, bias = f64(p["A"]), f64(p["D"]), f64(p["delta_bias"])
    nthreads = max(1, min(32, os.cpu_count() or 1))
    rows = [ix for ix in np.array_split(np.arange(w.batch), nthreads) if len(ix)]
    slices = [slice(int(ix[0]), int(ix[-1]) + 1) for ix in rows]
    hs = [h[sl].copy() for sl in slices]  # each thread's rows of the oracle state
    cy = StreamCheck(w.in_dtype, "decode every y of every step")

    def oracle_rows(i, inp):
        sl = slices[i]
        yr, hs[i] = oracle.state_update(hs[i], f64(inp["x"][sl]), f64(inp["delta"][sl]), A, f64(inp["B"][sl]),
                                        f64(inp["C"][sl]), D, f64(inp["z"][sl]), bias, True)
        return yr

    with ThreadPoolExecutor(len(slices)) as pool:  # ctypes calls release the GIL
        for k in range(w.steps):
            inp = syn.decode_step_inputs(w, k)
            y = _step_gpu(state, inp, params)
            yr = np.concatenate(list(pool.map(lambda i: oracle_rows(i, inp), range(len(slices)))))
            cy.add(f64(y), yr)
    torch.cuda.synchronize()
    cy.finish()
    check_bf16(f64(state), np.concatenate(hs), "decode final state (every element)")


def test_tails_both_kernels():
    """Raw steps and gates in [-40, 40], biases in [-15, 15], A per channel:
    the bulk-copy stream kernel (dim 256) and the general kernel (dim 37)."""
    for dim in (256, 37):
        w = syn.DecodeWorkload("tails", batch=3, dim=dim, dstate=16, steps=6, in_dtype=torch.float32)
        p = syn.decode_params(w, varied_A=True)
        gen = torch.Generator().manual_seed(dim)
        p["delta_bias"] = (torch.rand(dim, generator=gen) * 2 - 1) * 15.0
        params = {k: v.to(DEV) for k, v in p.items()}
        state = params["state0"].clone()
        h = f64(p["state0"])
        for k in range(w.steps):
            inp = syn.decode_step_inputs(w, k)
            inp["delta"] = (torch.rand(inp["delta"].shape, generator=gen) * 2 - 1) * 40.0
            inp["z"] = (torch.rand(inp["z"].shape, generator=gen) * 2 - 1) * 40.0
            y = _step_gpu(state, inp, params)
            yr, h = oracle.state_update(h, f64(inp["x"]), f64(inp["delta"]), f64(p["A"]), f64(inp["B"]),
                                        f64(inp["C"]), f64(p["D"]), f64(inp["z"]), f64(p["delta_bias"]), True)
            torch.cuda.synchronize()
            check_fp32(f64(y), yr, f"tails dim {dim} step {k} y")
        check_fp32(f64(state), h, f"tails dim {dim} final state")


@pytest.mark.parametrize("dtype,out_dtype,use_z", [
    (torch.float32, torch.float32, True), (torch.bfloat16, torch.float32, True),
    (torch.bfloat16, torch.bfloat16, True), (torch.bfloat16, torch.float32, False)])
def test_stream_path_small(dtype, out_dtype, use_z):
    """dim a multiple of 128 with dense 16-state rows: the bulk-copy stream
    kernel runs (several tiles per CTA, every step checked)."""
    w = syn.DecodeWorkload("stream", batch=5, dim=384, dstate=16, steps=12, in_dtype=dtype)
    p = syn.decode_params(w, varied_A=True)
    params = {k: v.to(DEV) for k, v in p.items()}
    state = params["state0"].clone()
    h = f64(p["state0"])
    for k in range(w.steps):
        inp = syn.decode_step_inputs(w, k)
        y = mb.state_update(state, inp["x"].to(DEV), inp["delta"].to(DEV), params["A"], inp["B"].to(DEV),
                            inp["C"].to(DEV), params["D"], inp["z"].to(DEV) if use_z else None,
                            params["delta_bias"], True, out_dtype=out_dtype)
        yr, h = oracle.state_update(h, f64(inp["x"]), f64(inp["delta"]), f64(p["A"]), f64(inp["B"]),
                                    f64(inp["C"]), f64(p["D"]), f64(inp["z"]) if use_z else None,
                                    f64(p["delta_bias"]), True)
        torch.cuda.synchronize()
        if out_dtype == torch.bfloat16:
            check_out_bf16(f64(y), yr, f"stream step {k} y")
        else:
            check(f64(y), yr, dtype, f"stream step {k} y")
    check(f64(state), h, dtype, "stream final state")
