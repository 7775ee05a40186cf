"""GPU parity of mamba2_ssd_fwd (the Mamba-2 SSD layer, chunked on the tensor
cores) against the fp64 oracle's recurrence, through the C ABI. Inputs are
bf16 (the oracle is fed the same values), so the bf16 rule applies: relative
L2 <= 2e-3 and max |g - r| <= 1e-2 on y and on the final state."""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_40_b200 import binding as mb
from selective_state_space_40_b200 import synthetic as syn
from parity_util import check, check_bf16, check_out_bf16, f64

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    assert mb.mamba_device_check() == mb.MS_OK


def _case(b, L, H, G, seed):
    w = syn.SsdWorkload("t", b, L, H, 64, 128, G, seed=seed)
    return w, syn.ssd_inputs(w)


def run(inp, s0=None, use_D=True, use_bias=True, softplus=True, out_dtype=torch.float32):
    g = {k: v.to(DEV) for k, v in inp.items()}
    y, fs = mb.ssd_fwd(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"] if use_D else None,
                       g["dt_bias"] if use_bias else None, softplus,
                       initial_state=None if s0 is None else s0.to(DEV), out_dtype=out_dtype)
    torch.cuda.synchronize()
    yr, fr = oracle.ssd(f64(inp["x"]), f64(inp["dt"]), f64(inp["A"]), f64(inp["B"]), f64(inp["C"]),
                        f64(inp["D"]) if use_D else None, f64(inp["dt_bias"]) if use_bias else None, softplus,
                        None if s0 is None else f64(s0))
    return y, fs, yr, fr


@pytest.mark.parametrize("L", [1, 31, 32, 33, 100, 127, 128, 129, 256, 300, 700])
@pytest.mark.parametrize("G", [1, 2])
def test_lengths_and_groups(L, G):
    _, inp = _case(2, L, 4, G, 10 + L + G)
    y, fs, yr, fr = run(inp)
    check_bf16(f64(y), yr, f"ssd L={L} G={G} y")
    check_bf16(f64(fs), fr, f"ssd L={L} G={G} final_state")


@pytest.mark.parametrize("flags", [dict(use_D=False), dict(use_bias=False), dict(softplus=False)])
def test_options(flags):
    _, inp = _case(2, 70, 4, 1, 50)
    if flags.get("softplus") is False:
        inp["dt"] = (0.05 * torch.rand(inp["dt"].shape)).to(torch.bfloat16)
        inp["dt_bias"] = torch.zeros_like(inp["dt_bias"])
    y, fs, yr, fr = run(inp, **flags)
    check_bf16(f64(y), yr, f"{flags} y")
    check_bf16(f64(fs), fr, f"{flags} final_state")


def test_initial_state_and_split():
    """final_state carries the sequence across calls: [0, m) then [m, L) from
    its final state equals the whole sequence."""
    _, inp = _case(2, 150, 4, 2, 60)
    s0 = 0.5 * torch.randn(2, 4, 64, 128, generator=torch.Generator().manual_seed(1))
    y, fs, yr, fr = run(inp, s0=s0)
    check_bf16(f64(y), yr, "s0 y")
    check_bf16(f64(fs), fr, "s0 final_state")
    m = 77
    g = {k: v.to(DEV) for k, v in inp.items()}
    sl = lambda k, a, b: g[k][:, a:b].contiguous()  # noqa: E731
    y1, f1 = mb.ssd_fwd(sl("x", 0, m), sl("dt", 0, m), g["A"], sl("B", 0, m), sl("C", 0, m), g["D"], g["dt_bias"],
                        True, initial_state=s0.to(DEV))
    y2, f2 = mb.ssd_fwd(sl("x", m, 150), sl("dt", m, 150), g["A"], sl("B", m, 150), sl("C", m, 150), g["D"],
                        g["dt_bias"], True, initial_state=f1)
    torch.cuda.synchronize()
    check_bf16(f64(torch.cat([y1, y2], dim=1)), yr, "split y")
    check_bf16(f64(f2), fr, "split final_state")


@pytest.mark.parametrize("b,L,H,G", [(2, 400, 20, 2), (1, 260, 9, 1), (3, 129, 16, 4)])
def test_head_blocks_and_chunks(b, L, H, G):
    """Several chunks of 128 tokens and several blocks of heads per group (up
    to 4 heads per work item, a ragged last block), so chunk k's items take
    their entering state from chunk k - 1's items of the same heads."""
    _, inp = _case(b, L, H, G, 30 + L + H)
    inp["A"] = -torch.exp(torch.randn(H, generator=torch.Generator().manual_seed(L)))  # a decay per head
    s0 = 0.3 * torch.randn(b, H, 64, 128, generator=torch.Generator().manual_seed(H))
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    g = {k: v.to(DEV) for k, v in inp.items()}
    y, fs = mb.ssd_fwd(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], g["dt_bias"], True,
                       initial_state=s0.to(DEV), dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    yr, fr = oracle.ssd(f64(inp["x"]), f64(inp["dt"]), f64(inp["A"]), f64(inp["B"]), f64(inp["C"]),
                        f64(inp["D"]), f64(inp["dt_bias"]), True, f64(s0))
    check_bf16(f64(y), yr, f"b={b} L={L} H={H} G={G} y")
    check_bf16(f64(fs), fr, f"b={b} L={L} H={H} G={G} final_state")


@pytest.mark.parametrize("b,L,H,G,out_dtype", [(16, 1024, 7, 1, torch.float32), (8, 2048, 9, 1, torch.float32),
                                                (12, 1280, 12, 3, torch.float32), (16, 1000, 7, 1, torch.bfloat16)])
def test_many_items_per_cta(b, L, H, G, out_dtype):
    """More work items than SMs, so each persistent CTA walks several items:
    the next item's parameters, C tile, B tile and first x rows arrive while
    the current one computes, and the two warp groups cross item boundaries
    apart. Head blocks of 7 and 9 heads per group leave blocks of 3 or 1 head
    (one group with fewer heads, or none, in those items); a ragged last chunk
    and bf16 y in one case."""
    import os
    from concurrent.futures import ThreadPoolExecutor
    _, inp = _case(b, L, H, G, 100 + H)
    inp["A"] = -torch.exp(torch.randn(H, generator=torch.Generator().manual_seed(H)))
    s0 = 0.3 * torch.randn(b, H, 64, 128, generator=torch.Generator().manual_seed(L))
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    g = {k: v.to(DEV) for k, v in inp.items()}
    y, fs = mb.ssd_fwd(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], g["dt_bias"], True,
                       initial_state=s0.to(DEV), dev_status=status, out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert int(status.item()) == 0

    def part(r):
        return oracle.ssd(f64(inp["x"][r:r + 1]), f64(inp["dt"][r:r + 1]), f64(inp["A"]), f64(inp["B"][r:r + 1]),
                          f64(inp["C"][r:r + 1]), f64(inp["D"]), f64(inp["dt_bias"]), True, f64(s0[r:r + 1]))

    with ThreadPoolExecutor(max(1, min(16, os.cpu_count() or 1))) as pool:
        parts = list(pool.map(part, range(b)))
    yr = np.concatenate([p_[0] for p_ in parts])
    fr = np.concatenate([p_[1] for p_ in parts])
    if out_dtype == torch.bfloat16:
        check_out_bf16(f64(y), yr, f"b={b} L={L} H={H} G={G} bf16 y")
    else:
        check_bf16(f64(y), yr, f"b={b} L={L} H={H} G={G} y")
    check_bf16(f64(fs), fr, f"b={b} L={L} H={H} G={G} final_state")


def test_repeat_is_bitwise_deterministic():
    """Items go to CTAs by ticket and chunk states pass between them through
    the workspace, so which CTA computes an item changes from run to run; the
    arithmetic of each output does not, and two runs agree bit for bit."""
    _, inp = _case(8, 2048, 9, 1, 77)
    g = {k: v.to(DEV) for k, v in inp.items()}
    outs = [mb.ssd_fwd(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], g["dt_bias"], True) for _ in range(3)]
    torch.cuda.synchronize()
    for y, fs in outs[1:]:
        assert torch.equal(y, outs[0][0]) and torch.equal(fs, outs[0][1])


def test_state_in_place_and_in_workspace():
    """initial_state and final_state as one array (updated in place), and no
    final_state (the running state in the workspace): the same y."""
    _, inp = _case(2, 300, 8, 1, 40)
    s0 = 0.3 * torch.randn(2, 8, 64, 128, generator=torch.Generator().manual_seed(5))
    g = {k: v.to(DEV) for k, v in inp.items()}
    st = s0.to(DEV).clone()
    y1, f1 = mb.ssd_fwd(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], g["dt_bias"], True,
                        initial_state=st, final_state=st)
    y2, f2 = mb.ssd_fwd(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], g["dt_bias"], True,
                        initial_state=s0.to(DEV), return_final_state=False)
    torch.cuda.synchronize()
    assert f1.data_ptr() == st.data_ptr() and f2 is None
    assert torch.equal(y1, y2)
    yr, fr = oracle.ssd(f64(inp["x"]), f64(inp["dt"]), f64(inp["A"]), f64(inp["B"]), f64(inp["C"]),
                        f64(inp["D"]), f64(inp["dt_bias"]), True, f64(s0))
    check_bf16(f64(y1), yr, "in-place y")
    check_bf16(f64(st), fr, "in-place final_state")


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_output_rows_not_16_byte_aligned(out_dtype):
    """y as a view whose head rows are 66 elements apart: the kernel stores the
    rows directly instead of through the tensor map."""
    _, inp = _case(2, 200, 4, 1, 75)
    g = {k: v.to(DEV) for k, v in inp.items()}
    ybuf = torch.full((2, 200, 4, 66), float("nan"), dtype=out_dtype, device=DEV)
    y = ybuf[..., :64]
    mb.ssd_fwd(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], g["dt_bias"], True, y=y, return_final_state=False)
    torch.cuda.synchronize()
    assert torch.isnan(ybuf[..., 64:].float()).all()  # the gaps are untouched
    yr, _ = oracle.ssd(f64(inp["x"]), f64(inp["dt"]), f64(inp["A"]), f64(inp["B"]), f64(inp["C"]), f64(inp["D"]),
                       f64(inp["dt_bias"]), True)
    if out_dtype == torch.bfloat16:
        check_out_bf16(f64(y), yr, "strided bf16 y")
    else:
        check_bf16(f64(y), yr, "strided y")


def test_bf16_output():
    _, inp = _case(1, 96, 4, 1, 70)
    y, _, yr, _ = run(inp, out_dtype=torch.bfloat16)
    check_out_bf16(f64(y), yr, "ssd bf16 y")


def test_strided_projection_layout():
    """x, dt, B, C as views into one projection output row per token (as a
    fused input projection produces them), not separate dense tensors."""
    b, L, H, P, N = 2, 64, 4, 64, 128
    w, inp = _case(b, L, H, 1, 80)
    width = H * P + 2 * N + 8  # x | B | C | dt (H of the last 8) -- rows stay 16-byte aligned
    buf = torch.zeros(b, L, width, dtype=torch.bfloat16)
    buf[:, :, :H * P] = inp["x"].reshape(b, L, H * P)
    buf[:, :, H * P:H * P + N] = inp["B"][:, :, 0]
    buf[:, :, H * P + N:H * P + 2 * N] = inp["C"][:, :, 0]
    buf[:, :, H * P + 2 * N:H * P + 2 * N + H] = inp["dt"]
    gb = buf.to(DEV)
    x = gb[:, :, :H * P].unflatten(2, (H, P))
    Bv = gb[:, :, H * P:H * P + N].unsqueeze(2)
    Cv = gb[:, :, H * P + N:H * P + 2 * N].unsqueeze(2)
    dtv = gb[:, :, H * P + 2 * N:H * P + 2 * N + H]
    y, fs = mb.ssd_fwd(x, dtv, inp["A"].to(DEV), Bv, Cv, inp["D"].to(DEV), inp["dt_bias"].to(DEV), True)
    torch.cuda.synchronize()
    yr, fr = oracle.ssd(f64(inp["x"]), f64(inp["dt"]), f64(inp["A"]), f64(inp["B"]), f64(inp["C"]),
                        f64(inp["D"]), f64(inp["dt_bias"]), True)
    check_bf16(f64(y), yr, "strided y")
    check_bf16(f64(fs), fr, "strided final_state")


def test_empty_sequence_passes_state():
    _, inp = _case(1, 0, 4, 1, 90)
    s0 = torch.randn(1, 4, 64, 128)
    y, fs, _, _ = run(inp, s0=s0)
    assert y.numel() == 0 and torch.equal(fs.cpu(), s0)


@pytest.mark.slow
def test_full_2p7b_layer_every_output():
    """The 2.7B-class layer at full size in the benchmark's configuration:
    every y and the whole final state against the oracle, which runs over
    blocks of heads on the host's cores (ctypes calls release the GIL)."""
    import os
    from concurrent.futures import ThreadPoolExecutor
    w = syn.SSD_2P7B
    inp = syn.ssd_inputs(w)
    g = {k: v.to(DEV) for k, v in inp.items()}
    y, fs = mb.ssd_fwd(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], g["dt_bias"], True)
    torch.cuda.synchronize()
    y, fs = f64(y), f64(fs)
    hb = 10
    jobs = [(b, h0) for b in range(w.batch) for h0 in range(0, w.nheads, hb)]

    def part(job):
        b, h0 = job
        hs = slice(h0, h0 + hb)
        return oracle.ssd(f64(inp["x"][b:b + 1, :, hs]), f64(inp["dt"][b:b + 1, :, hs]), f64(inp["A"][hs]),
                          f64(inp["B"][b:b + 1]), f64(inp["C"][b:b + 1]), f64(inp["D"][hs]),
                          f64(inp["dt_bias"][hs]), True)

    yr = np.empty_like(y)
    fr = np.empty_like(fs)
    with ThreadPoolExecutor(max(1, min(32, os.cpu_count() or 1))) as pool:
        for (b, h0), (yp, fp) in zip(jobs, pool.map(part, jobs)):
            yr[b:b + 1, :, h0:h0 + hb] = yp
            fr[b:b + 1, h0:h0 + hb] = fp
    check_bf16(y, yr, "2.7B y (every element)")
    check_bf16(fs, fr, "2.7B final_state (every element)")


# ------------------------------------------------------------ decode step ----

def _decode_inputs(b, H, P, G, seed, dtype=torch.bfloat16):
    gen = torch.Generator().manual_seed(seed)
    x = torch.randn(b, H, P, generator=gen).to(dtype)
    dt = torch.randn(b, H, generator=gen).to(dtype)
    B = torch.randn(b, G, 128, generator=gen).to(dtype)
    C = torch.randn(b, G, 128, generator=gen).to(dtype)
    return x, dt, B, C


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("P,G", [(64, 1), (48, 2), (8, 4)])
def test_decode_steps_against_oracle(dtype, P, G):
    """Several one-token steps from a random state, each against the oracle's
    recurrence with one token (y every step, the state at the end)."""
    b, H = 3, 4
    w = syn.SsdWorkload("d", b, 1, H, P, 128, G)
    par = syn.ssd_inputs(w)
    state = 0.3 * torch.randn(b, H, P, 128, generator=torch.Generator().manual_seed(2))
    sg = state.to(DEV)
    sr = f64(state)
    for k in range(6):
        x, dt, B, C = _decode_inputs(b, H, P, G, 100 + k, dtype)
        y = mb.ssd_state_update(sg, x.to(DEV), dt.to(DEV), par["A"].to(DEV), B.to(DEV), C.to(DEV),
                                par["D"].to(DEV), par["dt_bias"].to(DEV), True)
        torch.cuda.synchronize()
        yr, sr = oracle.ssd(f64(x)[:, None], f64(dt)[:, None], f64(par["A"]), f64(B)[:, None], f64(C)[:, None],
                            f64(par["D"]), f64(par["dt_bias"]), True, sr)
        check(f64(y), yr[:, 0], dtype, f"ssd decode step {k} y")
    check(f64(sg), sr, dtype, "ssd decode final state")


def test_full_decode_b64_every_output():
    """The decode step at the benchmark's size (64 sequences of the 2.7B-class
    layer, state [64, 80, 64, 128] fp32, bf16 inputs): three steps from a
    random state, every y of every step and the whole final state against the
    oracle's recurrence."""
    b, H, P, N = 64, 80, 64, 128
    par = syn.ssd_inputs(syn.SsdWorkload("d", 1, 1, H, P, N, 1))
    state = 0.1 * torch.randn(b, H, P, N, generator=torch.Generator().manual_seed(11))
    sg = state.to(DEV)
    sr = f64(state)
    for k in range(3):
        x, dt, B, C = _decode_inputs(b, H, P, 1, 300 + k)
        y = mb.ssd_state_update(sg, x.to(DEV), dt.to(DEV), par["A"].to(DEV), B.to(DEV), C.to(DEV),
                                par["D"].to(DEV), par["dt_bias"].to(DEV), True)
        torch.cuda.synchronize()
        yr, sr = oracle.ssd(f64(x)[:, None], f64(dt)[:, None], f64(par["A"]), f64(B)[:, None], f64(C)[:, None],
                            f64(par["D"]), f64(par["dt_bias"]), True, sr)
        check(f64(y), yr[:, 0], torch.bfloat16, f"b64 decode step {k} y (every element)")
    check(f64(sg), sr, torch.bfloat16, "b64 decode final state (every element)")


def test_decode_steps_equal_chunked_forward():
    """L one-token steps from a state equal the chunked forward over the same
    L tokens (recurrent view == matrix view) on the GPU."""
    b, L, H, G = 2, 40, 4, 1
    w, inp = _case(b, L, H, G, 120)
    s0 = 0.2 * torch.randn(b, H, 64, 128, generator=torch.Generator().manual_seed(3))
    g = {k: v.to(DEV) for k, v in inp.items()}
    yf, sf = mb.ssd_fwd(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], g["dt_bias"], True,
                        initial_state=s0.to(DEV))
    st = s0.to(DEV).clone()
    ys = []
    for t in range(L):
        ys.append(mb.ssd_state_update(st, g["x"][:, t].contiguous(), g["dt"][:, t].contiguous(), g["A"],
                                      g["B"][:, t].contiguous(), g["C"][:, t].contiguous(), g["D"], g["dt_bias"], True))
    torch.cuda.synchronize()
    yd = torch.stack(ys, dim=1)
    check_bf16(f64(yd), f64(yf), "decode steps vs chunked y")
    check_bf16(f64(st), f64(sf), "decode steps vs chunked final state")


@pytest.mark.parametrize("batch,L,G,strided", [(1, 1, 1, False), (1, 128, 1, False), (2, 300, 2, False),
                                               (1, 2048, 1, False), (2, 200, 2, True)])
def test_chunk_cb_tcgen05_against_oracle(batch, L, G, strided):
    # mamba2_ssd_chunk_cb (tcgen05 tensor cores, fp32 accumulation of exact
    # bf16 products) against the oracle's per-chunk C B^T of the same values:
    # only the summation order differs.
    gen = torch.Generator().manual_seed(100 + L)
    if strided:
        # B and C as slices of one projection tensor [b, L, 2 G 128 + 64]
        proj = torch.randn(batch, L, 2 * G * 128 + 64, generator=gen).to(torch.bfloat16)
        B = proj[:, :, 64:64 + G * 128].unflatten(-1, (G, 128))
        C = proj[:, :, 64 + G * 128:].unflatten(-1, (G, 128))
    else:
        B = torch.randn(batch, L, G, 128, generator=gen).to(torch.bfloat16)
        C = torch.randn(batch, L, G, 128, generator=gen).to(torch.bfloat16)
    cb = mb.ssd_chunk_cb(B.to(DEV), C.to(DEV)).cpu().double().numpy()
    ref = oracle.ssd_chunk_cb(f64(B), f64(C))
    assert cb.shape == ref.shape
    # fp32 summation of 128 exact products in any order: error <= 127 u sum |C_n B_n|
    bound = 127 * 2.0 ** -24 * oracle.ssd_chunk_cb(np.abs(f64(B)), np.abs(f64(C)))
    assert np.all(np.abs(cb - ref) <= bound + 1e-30), float(np.max(np.abs(cb - ref) - bound))


def test_chunk_cb_tcgen05_zero_rows_and_repeat():
    # zero B rows give zero columns; two calls give identical results
    gen = torch.Generator().manual_seed(3)
    B = torch.randn(1, 96, 1, 128, generator=gen).to(torch.bfloat16)
    C = torch.randn(1, 96, 1, 128, generator=gen).to(torch.bfloat16)
    B[:, 40:48] = 0
    cb1 = mb.ssd_chunk_cb(B.to(DEV), C.to(DEV))
    cb2 = mb.ssd_chunk_cb(B.to(DEV), C.to(DEV))
    torch.cuda.synchronize()
    assert torch.equal(cb1, cb2)
    assert float(cb1[0, 0, 1, :, 8:16].abs().max()) == 0.0
