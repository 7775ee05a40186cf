"""mamba_scan_bwd_noalloc (collected last): the allocation-free backward,
whose recomputed saved states live in the library's fixed device scratch,
gives the results of mamba_scan_bwd with a caller workspace, on two calls in
a row (the second call reuses the same scratch), and each call's gradients
match the fp64 oracle's. Passes alone and after the other tests."""
import pytest
import torch

import oracle
from selective_state_space_40_b200 import binding as mb
from selective_state_space_40_b200 import synthetic as syn
from parity_util import check, check_fp32, f64

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    assert mb.mamba_device_check() == mb.MS_OK


@pytest.mark.parametrize("dtype,L", [(torch.float32, 300), (torch.bfloat16, 1000)])
def test_noalloc_matches_workspace_backward_twice(dtype, L):
    w = syn.scaled(syn.M130, batch=3, dim=96, seqlen=L, in_dtype=dtype, seed=900 + L)
    host = syn.scan_inputs(w)
    host["A"] = syn.a_matrix_varied(w.dim, w.dstate, 900 + L)
    inp = {k: v.to(DEV) for k, v in host.items()}
    gen = torch.Generator().manual_seed(5)
    dout = torch.randn(w.batch, w.dim, w.seqlen, generator=gen).to(DEV)
    dlast = torch.randn(w.batch, w.dim, w.dstate, generator=gen).to(DEV)
    h0 = (0.3 * torch.randn(w.batch, w.dim, w.dstate, generator=gen)).to(DEV)
    args = (inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"], inp["z"], inp["delta_bias"], True, dout)
    ref = mb.scan_bwd(*args, dlast=dlast, initial_state=h0, ckpt=None)  # caller workspace
    runs = [mb.scan_bwd_noalloc(*args, dlast=dlast, initial_state=h0) for _ in range(2)]
    torch.cuda.synchronize()
    for r in runs:
        for k in ("du", "ddelta", "dz", "dinitial_state"):  # written directly: identical
            assert torch.equal(r[k], ref[k]), k
        for k in ("dA", "dB", "dC", "dD", "ddelta_bias"):    # fp32 atomic sums: order may differ
            check_fp32(f64(r[k]), f64(ref[k]), f"noalloc {k}")
    # and directly against the oracle's gradients of the same inputs
    rr = oracle.scan_bwd(*(f64(host[k]) for k in ("u", "delta", "A", "B", "C", "D", "z", "delta_bias")), True,
                         f64(dout), h0=f64(h0), dlast=f64(dlast))
    for r in runs:
        for k in ("du", "ddelta", "dA", "dB", "dC", "dD", "dz", "ddelta_bias"):
            # sums over batch rows, channels or tokens: the bf16 rule's absolute bound scales with their rms
            check(f64(r[k]), rr[k], dtype, f"noalloc vs oracle {k}", scaled=k in ("dA", "dB", "dC", "dD", "ddelta_bias"))
        check(f64(r["dinitial_state"]), rr["dh0"], dtype, "noalloc vs oracle dinitial_state")


def test_noalloc_oversize_is_rejected_without_launch():
    dims = mb.ScanDims(2, 5120, 16, 131072, 5120 * 131072, 131072, 5120 * 131072, 131072,
                       5120 * 131072, 131072, 5120 * 131072, 131072, 16 * 131072, 131072, 16 * 131072, 131072,
                       mb.MS_BF16, mb.MS_F32)
    fake = 1 << 20
    rc = mb.mamba_scan_bwd_noalloc(fake, fake, fake, fake, fake, None, None, None, 1, None, fake, None,
                                   fake, fake, fake, fake, fake, None, None, None, None, dims, None, None)
    assert rc == mb.MS_ERR_SCRATCH
