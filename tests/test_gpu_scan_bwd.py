"""GPU parity of the scan's training forward (saved states) and backward
(mamba_scan_fwd_train, mamba_scan_bwd) against the fp64 oracle's gradients,
through the C ABI.

Tolerances are the forward's (tests/parity_util.py) applied to every gradient
tensor separately: the oracle is fed the same stored input values, so the
differences come only from fp32 arithmetic, the fast exponential and the
order of the fp32 atomic sums.
"""
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import oracle
from selective_state_space_40_b200 import binding as mb
from selective_state_space_40_b200 import synthetic as syn
from parity_util import check, f64

pytestmark = pytest.mark.gpu

DEV = "cuda"
GRADS = ("du", "ddelta", "dA", "dB", "dC", "dD", "dz", "ddelta_bias")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    assert mb.mamba_device_check() == mb.MS_OK
    mb.library()


def _grads_inputs(w, seed, out_dtype=torch.float32, with_dlast=True, with_h0=False, varied_A=True):
    inp = syn.scan_inputs(w)
    if varied_A:  # A per channel and state (one slow channel): dA and A's indexing are exercised
        inp["A"] = syn.a_matrix_varied(w.dim, w.dstate, seed)
    g = torch.Generator().manual_seed(seed)
    dout = torch.randn(w.batch, w.dim, w.seqlen, generator=g).to(out_dtype)
    dlast = torch.randn(w.batch, w.dim, w.dstate, generator=g) if with_dlast else None
    h0 = 0.3 * torch.randn(w.batch, w.dim, w.dstate, generator=g) if with_h0 else None
    return inp, dout, dlast, h0


def run_gpu(inp, dout, dlast, h0, use_ckpt=True, use_z=True, use_D=True, use_bias=True, softplus=True):
    g = {k: v.to(DEV) for k, v in inp.items()}
    D = g["D"] if use_D else None
    z = g["z"] if use_z else None
    bias = g["delta_bias"] if use_bias else None
    h0d = None if h0 is None else h0.to(DEV)
    ckpt = None
    if use_ckpt:
        _, _, ckpt = mb.scan_fwd_train(g["u"], g["delta"], g["A"], g["B"], g["C"], D, z, bias, softplus,
                                       initial_state=h0d, out_dtype=dout.dtype)
    return mb.scan_bwd(g["u"], g["delta"], g["A"], g["B"], g["C"], D, z, bias, softplus, dout.to(DEV),
                       dlast=None if dlast is None else dlast.to(DEV), initial_state=h0d, ckpt=ckpt)


def run_oracle(inp, dout, dlast, h0, use_z=True, use_D=True, use_bias=True, softplus=True):
    return oracle.scan_bwd(f64(inp["u"]), f64(inp["delta"]), f64(inp["A"]), f64(inp["B"]), f64(inp["C"]),
                           f64(inp["D"]) if use_D else None, f64(inp["z"]) if use_z else None,
                           f64(inp["delta_bias"]) if use_bias else None, softplus, f64(dout),
                           h0=None if h0 is None else f64(h0), dlast=None if dlast is None else f64(dlast))


def compare(gg, rr, dtype, what, scaled=False):
    torch.cuda.synchronize()
    for k in GRADS:
        if rr[k] is None:
            assert gg[k] is None, f"{what}: {k} returned for a missing input"
            continue
        check(f64(gg[k]), rr[k], dtype, f"{what} {k}", scaled=scaled)
    if gg["dinitial_state"] is not None:
        check(f64(gg["dinitial_state"]), rr["dh0"], dtype, f"{what} dinitial_state", scaled=scaled)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("L", [1, 8, 63, 64, 65, 200])
def test_lengths(dtype, L):
    w = syn.scaled(syn.M130, batch=2, dim=40, seqlen=L, in_dtype=dtype, seed=100 + L)
    inp, dout, dlast, h0 = _grads_inputs(w, 7 + L, with_h0=(L % 2 == 1))
    compare(run_gpu(inp, dout, dlast, h0), run_oracle(inp, dout, dlast, h0), dtype, f"L={L} {dtype}")


@pytest.mark.parametrize("N", [1, 4, 5, 16])
def test_dstate(N):
    w = syn.scaled(syn.M130, batch=2, dim=36, seqlen=130, dstate=N, in_dtype=torch.float32, seed=200 + N)
    inp, dout, dlast, h0 = _grads_inputs(w, 11, with_h0=True)
    compare(run_gpu(inp, dout, dlast, h0), run_oracle(inp, dout, dlast, h0), torch.float32, f"N={N}")


@pytest.mark.parametrize("flags", [dict(use_z=False), dict(use_D=False), dict(use_bias=False),
                                   dict(softplus=False)])
def test_optional_inputs(flags):
    w = syn.scaled(syn.M130, batch=2, dim=40, seqlen=150, in_dtype=torch.float32, seed=300)
    inp, dout, dlast, h0 = _grads_inputs(w, 13)
    if flags.get("softplus") is False:
        inp["delta"] = (0.05 * torch.rand(inp["delta"].shape)).to(inp["delta"].dtype)  # positive steps
        inp["delta_bias"] = torch.zeros_like(inp["delta_bias"])
    compare(run_gpu(inp, dout, dlast, h0, **flags), run_oracle(inp, dout, dlast, h0, **flags),
            torch.float32, f"{flags}")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_tails(dtype):
    """Raw steps and gates in [-20, 20], biases in [-10, 10]: softplus' and
    silu' far into their tails, A_bar from 1 down to underflow."""
    w = syn.scaled(syn.M130, batch=2, dim=40, seqlen=150, in_dtype=dtype, seed=450)
    inp, dout, dlast, h0 = _grads_inputs(w, 23, with_h0=True)
    inp = syn.tail_inputs(inp, seed=450, lim=20.0, bias_lim=10.0)
    compare(run_gpu(inp, dout, dlast, h0), run_oracle(inp, dout, dlast, h0), dtype, f"tails {dtype}", scaled=True)


def test_bf16_dout():
    w = syn.scaled(syn.M130, batch=2, dim=40, seqlen=100, in_dtype=torch.bfloat16, seed=400)
    inp, dout, dlast, h0 = _grads_inputs(w, 17, out_dtype=torch.bfloat16)
    compare(run_gpu(inp, dout, dlast, h0), run_oracle(inp, dout, dlast, h0), torch.bfloat16, "bf16 dout")


def test_recomputed_states_match_saved():
    """No saved states: the backward recomputes them into its workspace; the
    directly written gradients are then bit-identical, and the training
    forward's y is the plain forward's."""
    w = syn.scaled(syn.M130, batch=3, dim=64, seqlen=333, in_dtype=torch.bfloat16, seed=500)
    inp, dout, dlast, h0 = _grads_inputs(w, 19, with_h0=True)
    g1 = run_gpu(inp, dout, dlast, h0, use_ckpt=True)
    g2 = run_gpu(inp, dout, dlast, h0, use_ckpt=False)
    torch.cuda.synchronize()
    for k in ("du", "ddelta", "dz", "dinitial_state"):
        assert torch.equal(g1[k], g2[k]), k
    g = {k: v.to(DEV) for k, v in inp.items()}
    y1, l1, _ = mb.scan_fwd_train(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"], g["delta_bias"],
                                  True, initial_state=h0.to(DEV))
    y0, l0 = mb.scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"], g["delta_bias"], True,
                         initial_state=h0.to(DEV))
    torch.cuda.synchronize()
    assert torch.equal(y1, y0) and torch.equal(l1, l0)


@pytest.mark.parametrize("L,dtype,with_h0", [(200, torch.float32, False), (256, torch.bfloat16, False),
                                             (203, torch.bfloat16, False), (192, torch.bfloat16, True),
                                             (195, torch.float32, True)])
def test_saved_states_are_block_states(L, dtype, with_h0):
    """ckpt[:, :, k] is the state before token 64 k (the oracle's last_state
    of the prefix; ckpt[:, :, 0] is the initial state): lengths that are
    multiples of 8 run the tensor-memory engine, 203 and 195 the register
    engine."""
    w = syn.scaled(syn.M130, batch=2, dim=24, seqlen=L, in_dtype=dtype, seed=600 + L)
    inp = syn.scan_inputs(w)
    g = {k: v.to(DEV) for k, v in inp.items()}
    h0 = 0.3 * torch.randn(2, 24, 16, generator=torch.Generator().manual_seed(L)) if with_h0 else None
    h0d = None if h0 is None else h0.to(DEV)
    y, _, ck = mb.scan_fwd_train(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"], g["delta_bias"],
                                 True, initial_state=h0d)
    y0, _ = mb.scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"], g["delta_bias"], True,
                        initial_state=h0d)
    torch.cuda.synchronize()
    nck = (L + 63) // 64
    assert ck.shape == (2, 24, nck, 16)
    assert torch.equal(y, y0)  # the same engine as the plain forward
    if h0 is None:
        assert float(ck[:, :, 0].abs().max()) == 0.0
    else:
        assert torch.equal(ck[:, :, 0].cpu(), h0)
    for k in range(1, nck):
        t = 64 * k
        pre = {n: (v[:, :, :t] if n in ("u", "delta", "z", "B", "C") else v) for n, v in inp.items()}
        _, lr = oracle.scan(f64(pre["u"]), f64(pre["delta"]), f64(pre["A"]), f64(pre["B"]), f64(pre["C"]),
                            f64(pre["D"]), f64(pre["z"]), f64(pre["delta_bias"]), True,
                            h0=None if h0 is None else f64(h0))
        check(f64(ck[:, :, k]), lr, torch.float32, f"saved state {k}")


@pytest.mark.parametrize("dim,dtype", [(8192, torch.bfloat16), (10240, torch.bfloat16), (8192, torch.float32)])
def test_wide_layer_training_forward(dim, dtype):
    """Layers wider than one 12-warp CTA per SM covers (2 x 8192 channels: 14
    compute warps per CTA; 2 x 10240: 18) save their states in the wider
    instantiations of the tensor-memory kernel: y equals the plain forward's
    bit for bit (the same engine and arithmetic), and every saved state is the
    oracle's state before its 64-token block."""
    L = 192
    w = syn.scaled(syn.M130, batch=2, dim=dim, seqlen=L, in_dtype=dtype, seed=dim)
    inp = syn.scan_inputs(w)
    inp["A"] = syn.a_matrix_varied(dim, 16, dim)
    g = {k: v.to(DEV) for k, v in inp.items()}
    y, last, ck = mb.scan_fwd_train(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"], g["delta_bias"],
                                    True)
    y0, l0 = mb.scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"], g["delta_bias"], True)
    torch.cuda.synchronize()
    assert torch.equal(y, y0) and torch.equal(last, l0)
    assert float(ck[:, :, 0].abs().max()) == 0.0
    for k in (1, 2):
        t = 64 * k
        pre = {n: (v[:, :, :t] if n in ("u", "delta", "z", "B", "C") else v) for n, v in inp.items()}
        _, lr = oracle.scan(f64(pre["u"]), f64(pre["delta"]), f64(pre["A"]), f64(pre["B"]), f64(pre["C"]),
                            f64(pre["D"]), f64(pre["z"]), f64(pre["delta_bias"]), True)
        check(f64(ck[:, :, k]), lr, torch.float32, f"wide layer saved state {k}")


def test_no_dinitial_requested():
    w = syn.scaled(syn.M130, batch=1, dim=32, seqlen=70, in_dtype=torch.float32, seed=700)
    inp, dout, dlast, h0 = _grads_inputs(w, 23)
    g = {k: v.to(DEV) for k, v in inp.items()}
    out = mb.scan_bwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"], g["delta_bias"], True,
                      dout.to(DEV), dlast=dlast.to(DEV), want_dinitial=False)
    compare(out, run_oracle(inp, dout, dlast, None), torch.float32, "no dinitial")


@pytest.mark.slow
def test_full_130m_every_gradient():
    """130M-class layer at full size (the config's A = -(n+1)), every
    gradient of every element against the oracle. The oracle runs over blocks
    of channels on the host's cores; dB and dC (sums over a batch row's
    channels) are the sums of the blocks' parts. Per-token gradients follow
    the bf16 rule; the sums over thousands of tokens (dA, dD, ddelta_bias,
    dB, dC) follow it with the absolute bound scaled by their rms."""
    w = syn.M130
    inp, dout, dlast, h0 = _grads_inputs(w, 29, varied_A=False)
    gg = run_gpu(inp, dout, dlast, h0)
    torch.cuda.synchronize()
    gg = {k: (None if v is None else v.cpu()) for k, v in gg.items()}
    nthreads = max(1, min(32, os.cpu_count() or 1))
    blocks = [(d0, min(w.dim, d0 + 96)) for d0 in range(0, w.dim, 96)]

    def part(blk):
        d0, d1 = blk
        sub = {k: (v[:, d0:d1] if k in ("u", "delta", "z") else (v[d0:d1] if k in ("A", "D", "delta_bias") else v))
               for k, v in inp.items()}
        return run_oracle(sub, dout[:, d0:d1], dlast[:, d0:d1], None)

    with ThreadPoolExecutor(nthreads) as pool:  # ctypes calls release the GIL
        parts = list(pool.map(part, blocks))
    for k, ax in (("du", 1), ("ddelta", 1), ("dz", 1), ("dh0", 1), ("dA", 0), ("dD", 0), ("ddelta_bias", 0)):
        ref = np.concatenate([p_[k] for p_ in parts], axis=ax)
        got = gg["dinitial_state" if k == "dh0" else k]
        check(f64(got), ref, w.in_dtype, f"130M {k} (every element)", scaled=k in ("dA", "dD", "ddelta_bias"))
    for k in ("dB", "dC"):
        ref = sum(p_[k] for p_ in parts)
        check(f64(gg[k]), ref, w.in_dtype, f"130M {k} (every element)", scaled=True)
