"""Device failure detection without a GPU fault: a bounded wait that runs out
reports MS_ERR_TIMEOUT through the caller's device status word and the
context stays usable (a decode step right after still matches the oracle)."""
import pytest
import torch

import oracle
from selective_state_space_40_b200 import binding as mb
from selective_state_space_40_b200 import synthetic as syn
from parity_util import check_fp32, f64

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    assert mb.mamba_device_check() == mb.MS_OK


@pytest.mark.parametrize("rounds", [1, 64])
def test_bounded_wait_reports_timeout(rounds):
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    stream = torch.cuda.current_stream().cuda_stream
    assert mb.mamba_debug_bounded_wait(rounds, status.data_ptr(), stream) == mb.MS_OK
    torch.cuda.synchronize()
    assert int(status.item()) == mb.MS_ERR_TIMEOUT


def test_context_usable_after_timeout():
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    mb.mamba_debug_bounded_wait(8, status.data_ptr(), torch.cuda.current_stream().cuda_stream)
    w = syn.DecodeWorkload("after", batch=2, dim=256, dstate=16, steps=1, in_dtype=torch.float32)
    p = syn.decode_params(w)
    s = syn.decode_step_inputs(w, 0)
    state = p["state0"].to(DEV).clone()
    ok = torch.zeros(1, dtype=torch.int32, device=DEV)
    y = mb.state_update(state, s["x"].to(DEV), s["delta"].to(DEV), p["A"].to(DEV), s["B"].to(DEV), s["C"].to(DEV),
                        p["D"].to(DEV), s["z"].to(DEV), p["delta_bias"].to(DEV), True, dev_status=ok)
    torch.cuda.synchronize()
    assert int(status.item()) == mb.MS_ERR_TIMEOUT and int(ok.item()) == mb.MS_OK
    yr, hr = oracle.state_update(f64(p["state0"]), f64(s["x"]), f64(s["delta"]), f64(p["A"]), f64(s["B"]),
                                 f64(s["C"]), f64(p["D"]), f64(s["z"]), f64(p["delta_bias"]), True)
    check_fp32(f64(y), yr, "decode after a timeout y")
    check_fp32(f64(state), hr, "decode after a timeout state")
