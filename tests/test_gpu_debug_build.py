"""The MS_DEBUG build of the library (libmambascan_debug.so): its kernels test
their indexes against the buffers they address and record MS_ERR_BOUNDS in
the caller's status word instead of performing an out-of-range access.

* the probe hook: an in-range index writes, an out-of-range one is recorded
  (and skipped), in the debug build; the product build refuses the hook;
* tiny shapes through every kernel family (both scan engines, the sequence
  split, the conv front-end, the decode step, the training forward and the
  backward, the Mamba-2 SSD forward and its decode step) report no bounds
  failure and still match the oracle.
"""
import os

import pytest
import torch

import oracle
from selective_state_space_40_b200 import binding as mb
from selective_state_space_40_b200 import build as mbuild
from selective_state_space_40_b200 import synthetic as syn
from parity_util import check, check_bf16, f64

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def debug_lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    path = mbuild.build_debug()
    with mb.use_library(path) as lib:
        assert mb.mamba_debug_build() == 1
        yield lib


def _status():
    return torch.zeros(1, dtype=torch.int32, device=DEV)


def test_product_build_refuses_probe():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    st = _status()
    assert mb.mamba_debug_build() == 0
    assert mb.mamba_debug_bounds_probe(3, st.data_ptr(), None) == mb.MS_ERR_SHAPE


@pytest.mark.parametrize("index,code", [(0, 0), (15, 0), (16, 11), (-1, 11), (1 << 20, 11)])
def test_probe_records_out_of_range(debug_lib, index, code):
    st = _status()
    assert mb.mamba_debug_bounds_probe(index, st.data_ptr(), torch.cuda.current_stream().cuda_stream) == mb.MS_OK
    torch.cuda.synchronize()
    assert int(st.item()) == code == (mb.MS_ERR_BOUNDS if code else 0)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("plan,L", [((4, 1, 0, mb.MS_ENGINE_TMEM), 96), ((4, 1, 0, mb.MS_ENGINE_REGISTER), 77),
                                    ((8, 1, 8, mb.MS_ENGINE_REGISTER), 64), (None, 9000)])
def test_scan_engines_clean(debug_lib, dtype, plan, L):
    w = syn.scaled(syn.LONG if plan is None else syn.M130, batch=1 if plan is None else 2,
                   dim=48 if plan is None else 40, seqlen=L, in_dtype=dtype, seed=L)
    inp = syn.scan_inputs(w)
    inp["A"] = syn.a_matrix_varied(w.dim, 16, L)
    g = {k: v.to(DEV) for k, v in inp.items()}
    st = _status()
    y, last = mb.scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"], g["delta_bias"], True,
                          plan=plan, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    yr, lr = oracle.scan(*(f64(inp[k]) for k in ("u", "delta", "A", "B", "C", "D", "z", "delta_bias")), True)
    check(f64(y), yr, dtype, "debug build y")
    check(f64(last), lr, dtype, "debug build last_state")


def test_conv_and_decode_clean(debug_lib):
    w = syn.scaled(syn.M130, batch=2, dim=40, seqlen=70, in_dtype=torch.float32, seed=3)
    inp = syn.scan_inputs(w)
    cp = syn.conv_params(w, 4)
    g = {k: v.to(DEV) for k, v in inp.items()}
    c = {k: v.to(DEV) for k, v in cp.items()}
    st = _status()
    y, last, _ = mb.conv_scan_fwd(g["u"], c["conv_w"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"],
                                  g["delta_bias"], True, conv_b=c["conv_b"], dev_status=st)
    dw = syn.DecodeWorkload("dbg", batch=2, dim=256, dstate=16, steps=1, in_dtype=torch.float32)
    p = syn.decode_params(dw, varied_A=True)
    s = syn.decode_step_inputs(dw, 0)
    state = p["state0"].to(DEV).clone()
    yd = mb.state_update(state, s["x"].to(DEV), s["delta"].to(DEV), p["A"].to(DEV), s["B"].to(DEV),
                         s["C"].to(DEV), p["D"].to(DEV), s["z"].to(DEV), p["delta_bias"].to(DEV), True,
                         dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    yr, lr, _ = oracle.conv_scan(f64(inp["u"]), f64(cp["conv_w"]), f64(cp["conv_b"]), None, True,
                                 *(f64(inp[k]) for k in ("delta", "A", "B", "C", "D", "z", "delta_bias")))
    check(f64(y), yr, torch.float32, "debug conv y")
    ydr, hr = oracle.state_update(f64(p["state0"]), f64(s["x"]), f64(s["delta"]), f64(p["A"]), f64(s["B"]),
                                  f64(s["C"]), f64(p["D"]), f64(s["z"]), f64(p["delta_bias"]), True)
    check(f64(yd), ydr, torch.float32, "debug decode y")
    check(f64(state), hr, torch.float32, "debug decode state")


@pytest.mark.parametrize("L,dim", [(128, 40), (130, 40), (128, 10240)])
def test_training_forward_and_backward_clean(debug_lib, L, dim):
    # L = 128: 16-byte dB/dC atomics; L = 130: ragged last block, 4-byte atomics;
    # dim 10240 (2 rows): a wide saved-state instantiation of the forward (more
    # than 12 warps per CTA)
    w = syn.scaled(syn.M130, batch=2, dim=dim, seqlen=L, in_dtype=torch.float32, seed=L)
    inp = syn.scan_inputs(w)
    inp["A"] = syn.a_matrix_varied(w.dim, w.dstate, L)
    gen = torch.Generator().manual_seed(L)
    dout = torch.randn(w.batch, w.dim, L, generator=gen)
    dlast = torch.randn(w.batch, w.dim, w.dstate, generator=gen)
    g = {k: v.to(DEV) for k, v in inp.items()}
    st_fwd, st_bwd = _status(), _status()
    _, _, ckpt = mb.scan_fwd_train(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"], g["delta_bias"],
                                   True, dev_status=st_fwd)
    gr = mb.scan_bwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"], g["delta_bias"], True,
                     dout.to(DEV), dlast=dlast.to(DEV), ckpt=ckpt, dev_status=st_bwd)
    torch.cuda.synchronize()
    assert (int(st_fwd.item()), int(st_bwd.item())) == (0, 0)
    rr = oracle.scan_bwd(*(f64(inp[k]) for k in ("u", "delta", "A", "B", "C", "D", "z", "delta_bias")), True,
                         f64(dout), dlast=f64(dlast))
    for k in ("du", "ddelta", "dA", "dB", "dC", "dD", "dz", "ddelta_bias"):
        check(f64(gr[k]), rr[k], torch.float32, f"debug backward {k}")


def test_ssd_forward_and_decode_clean(debug_lib):
    w = syn.SsdWorkload("dbg", 2, 300, 4, 64, 128, 2, seed=7)
    inp = syn.ssd_inputs(w)
    s0 = 0.3 * torch.randn(2, 4, 64, 128, generator=torch.Generator().manual_seed(7))
    g = {k: v.to(DEV) for k, v in inp.items()}
    st = _status()
    y, fs = mb.ssd_fwd(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], g["dt_bias"], True,
                       initial_state=s0.to(DEV), dev_status=st)
    # two decode steps from the forward's final state: tokens 0 and 1 again
    state = fs.clone()
    yd = [mb.ssd_state_update(state, g["x"][:, t].contiguous(), g["dt"][:, t].contiguous(), g["A"],
                              g["B"][:, t].contiguous(), g["C"][:, t].contiguous(), g["D"], g["dt_bias"], True,
                              dev_status=st) for t in range(2)]
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    A64 = f64(inp["A"])
    yr, fr = oracle.ssd(f64(inp["x"]), f64(inp["dt"]), A64, f64(inp["B"]), f64(inp["C"]), f64(inp["D"]),
                        f64(inp["dt_bias"]), True, f64(s0))
    check_bf16(f64(y), yr, "debug ssd y")
    check_bf16(f64(fs), fr, "debug ssd final_state")
    ydr, sr = oracle.ssd(f64(inp["x"])[:, :2], f64(inp["dt"])[:, :2], A64, f64(inp["B"])[:, :2],
                         f64(inp["C"])[:, :2], f64(inp["D"]), f64(inp["dt_bias"]), True, fr)
    check_bf16(f64(torch.stack(yd, dim=1)), ydr, "debug ssd decode y")
    check_bf16(f64(state), sr, "debug ssd decode state")
