"""The C-ABI library: builds, loads without a GPU, exports every function the
headers declare, and rejects bad arguments on the host (no GPU involved)."""
import ctypes
import glob
import os
import re

import pytest

from selective_state_space_40_b200 import binding as mb
from selective_state_space_40_b200 import build as mbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    mbuild.build()
    return mb.library()


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(mamba2?_\w+)\s*\(", text, flags=re.M):
            names.add(m.group(1))
    return sorted(names)


def test_header_declares_entry_points():
    names = declared_functions()
    for n in ("mamba_scan_fwd", "mamba_state_update", "mamba_scan_workspace_size",
              "mamba_status_string", "mamba_device_check", "mamba_scan_fwd_plan",
              "mamba_scan_choose_plan", "mamba_conv_scan_fwd", "mamba2_ssd_fwd", "mamba2_ssd_state_update",
              "mamba2_ssd_chunk_cb", "mamba2_ssd_chunk_cb_size"):
        assert n in names


@pytest.mark.parametrize("name", declared_functions())
def test_library_exports(lib, name):
    assert hasattr(lib, name), f"{name} declared in include/ but not exported"


def test_no_cpu_fallback_symbols(lib):
    # the product library never links the oracle
    for sym in ("oracle_scan_f64", "oracle_state_update_f64", "oracle_causal_conv_f64"):
        with pytest.raises(AttributeError):
            getattr(lib, sym)


def test_status_strings(lib):
    for code in range(0, 11):
        s = mb.mamba_status_string(code)
        assert isinstance(s, str) and s
    assert mb.mamba_status_string(0) == "ok"
    assert "unknown" in mb.mamba_status_string(12345)


def _dims(**kw):
    d = dict(batch=2, dim=8, dstate=16, seqlen=32, u_sb=256, u_sd=32, delta_sb=256, delta_sd=32,
             z_sb=256, z_sd=32, y_sb=256, y_sd=32, B_sb=512, B_sn=32, C_sb=512, C_sn=32,
             in_dtype=mb.MS_F32, out_dtype=mb.MS_F32)
    d.update(kw)
    return mb.ScanDims(**d)


FAKE = 1 << 20  # never dereferenced: every call below fails its host checks


def _scan(dims, u=FAKE, delta=FAKE, A=FAKE, B=FAKE, C=FAKE, y=FAKE, ws=None, ws_bytes=0, plan=None):
    return mb.mamba_scan_fwd(u, delta, A, B, C, None, None, None, 1, None, y, None, dims,
                             ws, ws_bytes, None, None, plan)


@pytest.mark.parametrize("kw,code", [
    (dict(in_dtype=7), mb.MS_ERR_DTYPE),
    (dict(out_dtype=-1), mb.MS_ERR_DTYPE),
    (dict(dstate=0), mb.MS_ERR_SHAPE),
    (dict(dstate=17), mb.MS_ERR_SHAPE),
    (dict(batch=-1), mb.MS_ERR_SHAPE),
    (dict(seqlen=-5), mb.MS_ERR_SHAPE),
    (dict(u_sd=-1), mb.MS_ERR_STRIDE),
    (dict(B_sn=-2), mb.MS_ERR_STRIDE),
    (dict(u_sb=1 << 61, batch=1 << 4), mb.MS_ERR_SHAPE),
])
def test_scan_rejects_bad_dims(lib, kw, code):
    assert _scan(_dims(**kw)) == code


def test_scan_rejects_null_and_misaligned(lib):
    assert mb.library().mamba_scan_fwd(*([None] * 8), 1, None, None, None, None, None, 0, None, None) \
        == mb.MS_ERR_NULL
    assert _scan(_dims(), u=None) == mb.MS_ERR_NULL
    assert _scan(_dims(), y=None) == mb.MS_ERR_NULL
    assert _scan(_dims(), A=None) == mb.MS_ERR_NULL
    assert _scan(_dims(), u=FAKE + 2) == mb.MS_ERR_ALIGN       # fp32 needs 4-byte alignment
    assert _scan(_dims(in_dtype=mb.MS_BF16), u=FAKE + 1) == mb.MS_ERR_ALIGN
    assert _scan(_dims(), A=FAKE + 1) == mb.MS_ERR_ALIGN


def test_scan_rejects_bad_plan_and_workspace(lib):
    assert _scan(_dims(), plan=mb.ScanPlan(3, 1, 0)) == mb.MS_ERR_SHAPE
    assert _scan(_dims(), plan=mb.ScanPlan(4, 3, 0)) == mb.MS_ERR_SHAPE
    assert _scan(_dims(), plan=mb.ScanPlan(8, 2, 0)) == mb.MS_ERR_SHAPE
    assert _scan(_dims(), plan=mb.ScanPlan(4, 1, 5)) == mb.MS_ERR_SHAPE
    assert _scan(_dims(), plan=mb.ScanPlan(4, 1, 0, 2)) == mb.MS_ERR_SHAPE      # no such engine
    assert _scan(_dims(), plan=mb.ScanPlan(8, 1, 0, mb.MS_ENGINE_TMEM)) == mb.MS_ERR_SHAPE
    assert _scan(_dims(), plan=mb.ScanPlan(4, 2, 0, mb.MS_ENGINE_TMEM)) == mb.MS_ERR_SHAPE
    # the tensor-memory engine needs seqlen % 8 == 0 (and a device): refused before any launch
    assert _scan(_dims(seqlen=30, u_sb=240, u_sd=30, delta_sb=240, delta_sd=30, z_sb=240, z_sd=30, y_sb=240,
                       y_sd=30, B_sb=480, B_sn=30, C_sb=480, C_sn=30),
                 plan=mb.ScanPlan(4, 1, 0, mb.MS_ENGINE_TMEM)) == mb.MS_ERR_SHAPE
    assert _scan(_dims(), ws=None, ws_bytes=64) == mb.MS_ERR_WORKSPACE


def test_empty_scan_is_a_noop(lib):
    # nothing to compute: no launch, so this is safe without a GPU
    assert _scan(_dims(batch=0)) == mb.MS_OK
    assert _scan(_dims(dim=0), u=None, y=None) == mb.MS_OK
    assert mb.mamba_scan_workspace_size(_dims()) == 0


def test_choose_plan(lib):
    rc, plan = mb.mamba_scan_choose_plan(_dims(batch=8, dim=1536, seqlen=2048, in_dtype=mb.MS_BF16))
    assert rc == mb.MS_OK and plan.lanes_per_channel in (1, 2, 4, 8) and plan.poly8 in (0, 2, 4, 8)
    assert plan.chunks_per_lane in (1, 2)
    # 130M-class shape: the tensor-memory engine (by sizes and strides)
    d130 = _dims(batch=8, dim=1536, seqlen=2048, in_dtype=mb.MS_BF16, u_sb=1536 * 2048, u_sd=2048,
                 delta_sb=1536 * 2048, delta_sd=2048, z_sb=1536 * 2048, z_sd=2048, y_sb=1536 * 2048, y_sd=2048,
                 B_sb=16 * 2048, B_sn=2048, C_sb=16 * 2048, C_sn=2048)
    rc, plan = mb.mamba_scan_choose_plan(d130)
    assert rc == mb.MS_OK and plan.engine == mb.MS_ENGINE_TMEM and plan.lanes_per_channel == 4
    # seqlen not a multiple of 8: the register engine
    rc, plan = mb.mamba_scan_choose_plan(_dims(seqlen=30, u_sd=30, delta_sd=30, z_sd=30, y_sd=30, B_sn=30, C_sn=30))
    assert rc == mb.MS_OK and plan.engine == mb.MS_ENGINE_REGISTER
    rc, _ = mb.mamba_scan_choose_plan(_dims(dstate=40))
    assert rc == mb.MS_ERR_SHAPE


def _conv(dims, width=4, silu=1, uout_sb=256, uout_sd=32, w=FAKE, b=None, x0=None, u_out=None,
          x=FAKE, y=FAKE, plan=None):
    cd = mb.ConvDims(width, uout_sb, uout_sd, silu)
    return mb.mamba_conv_scan_fwd(x, w, b, x0, u_out, cd, FAKE, FAKE, FAKE, FAKE, None, None, None, 1,
                                  None, y, None, dims, plan, None, None)


def test_conv_scan_rejects_bad_arguments(lib):
    assert _conv(_dims(), width=0) == mb.MS_ERR_SHAPE
    assert _conv(_dims(), width=5) == mb.MS_ERR_SHAPE
    assert _conv(_dims(), uout_sd=-1) == mb.MS_ERR_STRIDE
    assert _conv(_dims(), w=None) == mb.MS_ERR_NULL
    assert _conv(_dims(), x=None) == mb.MS_ERR_NULL
    assert _conv(_dims(), w=FAKE + 2) == mb.MS_ERR_ALIGN
    assert _conv(_dims(), b=FAKE + 1) == mb.MS_ERR_ALIGN
    assert _conv(_dims(in_dtype=mb.MS_BF16), x0=FAKE + 1) == mb.MS_ERR_ALIGN
    assert _conv(_dims(), u_out=FAKE + 2) == mb.MS_ERR_ALIGN
    assert _conv(_dims(), u_out=FAKE, uout_sb=1 << 61, uout_sd=1) == mb.MS_ERR_SHAPE
    assert _conv(_dims(in_dtype=9)) == mb.MS_ERR_DTYPE
    # the conv front-end runs one chunk per lane, exponentials all MUFU or all polynomial
    assert _conv(_dims(), plan=mb.ScanPlan(4, 2, 0)) == mb.MS_ERR_SHAPE
    assert _conv(_dims(), plan=mb.ScanPlan(4, 1, 2)) == mb.MS_ERR_SHAPE
    assert _conv(_dims(), plan=mb.ScanPlan(3, 1, 0)) == mb.MS_ERR_SHAPE
    assert _conv(_dims(), plan=mb.ScanPlan(4, 1, 0, mb.MS_ENGINE_TMEM)) == mb.MS_ERR_SHAPE
    cd = mb.ConvDims(4, 0, 0, 1)
    assert mb.library().mamba_conv_scan_fwd(FAKE, FAKE, None, None, None, None, FAKE, FAKE, FAKE, FAKE,
                                            None, None, None, 1, None, FAKE, None, ctypes.byref(_dims()),
                                            None, None, None) == mb.MS_ERR_NULL
    del cd


def test_conv_scan_empty_is_a_noop(lib):
    assert _conv(_dims(batch=0)) == mb.MS_OK
    assert _conv(_dims(dim=0), w=None, x=None, y=None) == mb.MS_OK


def _bwd(dims, ckpt=FAKE, dout=FAKE, du=FAKE, ddelta=FAKE, dA=FAKE, dB=FAKE, dC=FAKE, ws=None, ws_bytes=0):
    return mb.mamba_scan_bwd(FAKE, FAKE, FAKE, FAKE, FAKE, None, None, None, 1, None, ckpt, dout, None,
                             du, ddelta, dA, dB, dC, None, None, None, None, dims, ws, ws_bytes, None, None)


def test_scan_bwd_rejects_bad_arguments(lib):
    assert _bwd(_dims(dstate=17)) == mb.MS_ERR_SHAPE
    assert _bwd(_dims(in_dtype=5)) == mb.MS_ERR_DTYPE
    assert _bwd(_dims(), dout=None) == mb.MS_ERR_NULL
    assert _bwd(_dims(), dA=None) == mb.MS_ERR_NULL
    assert _bwd(_dims(), dB=None) == mb.MS_ERR_NULL
    assert _bwd(_dims(), du=FAKE + 2) == mb.MS_ERR_ALIGN
    assert _bwd(_dims(), ckpt=FAKE + 1) == mb.MS_ERR_ALIGN
    # no saved states and no workspace for recomputing them
    assert _bwd(_dims(), ckpt=None) == mb.MS_ERR_WORKSPACE
    assert _bwd(_dims(), ckpt=None, ws=FAKE, ws_bytes=16) == mb.MS_ERR_WORKSPACE
    assert _bwd(_dims(batch=0)) == mb.MS_OK


def test_ckpt_sizes(lib):
    d = _dims(batch=2, dim=8, dstate=16, seqlen=130)
    assert mb.mamba_scan_ckpt_size(d) == 2 * 8 * 3 * 16 * 4
    assert mb.mamba_scan_bwd_workspace_size(d) == mb.mamba_scan_ckpt_size(d)
    assert mb.mamba_scan_ckpt_size(_dims(seqlen=0)) == 0
    rc = mb.mamba_scan_fwd_train(FAKE, FAKE, FAKE, FAKE, FAKE, None, None, None, 1, None, FAKE, None, None,
                                 _dims(), None, None)
    assert rc == mb.MS_ERR_NULL  # training forward without its saved-state array


def test_bwd_noalloc_rejects_oversize_and_bad_arguments(lib):
    def call(dims, dout=FAKE):
        return mb.mamba_scan_bwd_noalloc(FAKE, FAKE, FAKE, FAKE, FAKE, None, None, None, 1, None, dout, None,
                                         FAKE, FAKE, FAKE, FAKE, FAKE, None, None, None, None, dims, None, None)
    # 4 x 5120 x 65536 tokens needs 1024 blocks of saved states: 1.3 GB > the fixed 96 MiB
    big = _dims(batch=4, dim=5120, seqlen=65536, u_sb=5120 * 65536, u_sd=65536, delta_sb=5120 * 65536,
                delta_sd=65536, z_sb=5120 * 65536, z_sd=65536, y_sb=5120 * 65536, y_sd=65536,
                B_sb=16 * 65536, B_sn=65536, C_sb=16 * 65536, C_sn=65536)
    assert mb.mamba_scan_bwd_workspace_size(big) > mb.MS_BWD_NOALLOC_MAX_BYTES
    assert call(big) == mb.MS_ERR_SCRATCH
    assert "fixed buffer" in mb.mamba_status_string(mb.MS_ERR_SCRATCH)
    assert call(_dims(dstate=0)) == mb.MS_ERR_SHAPE
    assert call(_dims(), dout=None) == mb.MS_ERR_NULL
    assert call(_dims(batch=0)) == mb.MS_OK


def _sdims(**kw):
    d = dict(batch=2, seqlen=64, nheads=4, headdim=64, dstate=128, ngroups=1, x_sb=64 * 256, x_sl=256, x_sh=64,
             dt_sb=256, dt_sl=4, B_sb=64 * 128, B_sl=128, B_sg=128, C_sb=64 * 128, C_sl=128, C_sg=128,
             y_sb=64 * 256, y_sl=256, y_sh=64, in_dtype=mb.MS_BF16, out_dtype=mb.MS_F32)
    d.update(kw)
    return mb.SsdDims(**d)


def test_ssd_rejects_bad_arguments(lib):
    def call(dims, x=FAKE, y=FAKE, B=FAKE, ws=None, ws_bytes=0):
        return mb.mamba2_ssd_fwd(x, FAKE, FAKE, B, FAKE, None, None, 1, None, y, None, dims, ws, ws_bytes, None,
                                 None)
    assert call(_sdims(headdim=32)) == mb.MS_ERR_SHAPE
    assert call(_sdims(dstate=64)) == mb.MS_ERR_SHAPE
    assert call(_sdims(nheads=5, ngroups=2)) == mb.MS_ERR_SHAPE
    assert call(_sdims(in_dtype=mb.MS_F32)) == mb.MS_ERR_DTYPE
    assert call(_sdims(out_dtype=4)) == mb.MS_ERR_DTYPE
    assert call(_sdims(x_sl=-1)) == mb.MS_ERR_STRIDE
    assert call(_sdims(), x=None) == mb.MS_ERR_NULL
    assert call(_sdims(), x=FAKE + 2) == mb.MS_ERR_ALIGN      # rows need 16-byte alignment
    assert call(_sdims(B_sl=132)) == mb.MS_ERR_ALIGN         # row stride not a multiple of 8 elements
    assert call(_sdims(), y=FAKE + 4) == mb.MS_ERR_ALIGN      # fp32 pairs need 8-byte alignment
    assert call(_sdims(batch=0)) == mb.MS_OK
    # the chunk hand-off needs the workspace: flags, counter and (no final_state) the running state
    need = mb.mamba2_ssd_workspace_size(_sdims())
    assert need >= 2 * 4 * 64 * 128 * 4 + (2 * 4 + 1) * 4
    assert call(_sdims()) == mb.MS_ERR_WORKSPACE
    assert call(_sdims(), ws=FAKE, ws_bytes=need - 1) == mb.MS_ERR_WORKSPACE
    assert call(_sdims(), ws=FAKE + 8, ws_bytes=need) == mb.MS_ERR_ALIGN


def test_ssd_chunk_cb_rejects_bad_arguments(lib):
    def call(dims, B=FAKE, C=FAKE, cb=FAKE):
        return mb.mamba2_ssd_chunk_cb(B, C, cb, dims, None, None)
    assert call(_sdims(dstate=64)) == mb.MS_ERR_SHAPE
    assert call(_sdims(ngroups=0)) == mb.MS_ERR_SHAPE
    assert call(_sdims(in_dtype=mb.MS_F32)) == mb.MS_ERR_DTYPE
    assert call(_sdims(C_sl=-1)) == mb.MS_ERR_STRIDE
    assert call(_sdims(), cb=None) == mb.MS_ERR_NULL
    assert call(_sdims(), B=FAKE + 2) == mb.MS_ERR_ALIGN
    assert call(_sdims(C_sl=132)) == mb.MS_ERR_ALIGN
    assert call(_sdims(), cb=FAKE + 8) == mb.MS_ERR_ALIGN
    assert call(_sdims(batch=0)) == mb.MS_OK
    assert call(_sdims(seqlen=0)) == mb.MS_OK
    # batch 2, 1 group, 64 tokens = 2 chunks of 32 x 32 fp32
    assert mb.mamba2_ssd_chunk_cb_size(_sdims()) == 2 * 1 * 2 * 32 * 32 * 4
    assert mb.mamba2_ssd_chunk_cb_size(_sdims(seqlen=65, ngroups=2)) == 2 * 2 * 3 * 32 * 32 * 4


def test_ssd_update_rejects_bad_arguments(lib):
    def dims(**kw):
        d = dict(batch=2, nheads=4, headdim=64, dstate=128, ngroups=1, x_sb=256, x_sh=64, dt_sb=4, B_sb=128,
                 B_sg=128, C_sb=128, C_sg=128, y_sb=256, y_sh=64, state_sb=4 * 64 * 128, state_sh=64 * 128,
                 in_dtype=mb.MS_BF16, out_dtype=mb.MS_F32)
        d.update(kw)
        return mb.SsdUpdateDims(**d)

    def call(dm, state=FAKE):
        return mb.mamba2_ssd_state_update(state, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, 1, FAKE, dm, None, None)
    assert call(dims(dstate=64)) == mb.MS_ERR_SHAPE
    assert call(dims(nheads=3, ngroups=2)) == mb.MS_ERR_SHAPE
    assert call(dims(in_dtype=3)) == mb.MS_ERR_DTYPE
    assert call(dims(x_sh=-1)) == mb.MS_ERR_STRIDE
    assert call(dims(), state=None) == mb.MS_ERR_NULL
    assert call(dims(), state=FAKE + 4) == mb.MS_ERR_ALIGN
    assert call(dims(state_sh=64 * 128 + 2)) == mb.MS_ERR_ALIGN
    assert call(dims(batch=0)) == mb.MS_OK


def test_debug_bounded_wait_argument_checks(lib):
    assert mb.mamba_debug_bounded_wait(16, None, None) == mb.MS_ERR_NULL
    assert mb.mamba_debug_bounded_wait(0, FAKE, None) == mb.MS_ERR_SHAPE
    assert mb.mamba_debug_bounded_wait((1 << 20) + 1, FAKE, None) == mb.MS_ERR_SHAPE
    assert mb.mamba_debug_bounded_wait(16, FAKE + 2, None) == mb.MS_ERR_ALIGN


def _udims(**kw):
    d = dict(batch=4, dim=8, dstate=16, x_sb=8, delta_sb=8, z_sb=8, y_sb=8, B_sb=16, C_sb=16,
             state_sb=128, state_sd=16, in_dtype=mb.MS_BF16, out_dtype=mb.MS_F32)
    d.update(kw)
    return mb.UpdateDims(**d)


@pytest.mark.parametrize("kw,code", [
    (dict(in_dtype=3), mb.MS_ERR_DTYPE),
    (dict(dstate=0), mb.MS_ERR_SHAPE),
    (dict(dstate=32), mb.MS_ERR_SHAPE),
    (dict(state_sd=-16), mb.MS_ERR_STRIDE),
])
def test_update_rejects_bad_dims(lib, kw, code):
    rc = mb.mamba_state_update(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, None, 1, FAKE,
                               _udims(**kw), None, None)
    assert rc == code


def test_update_rejects_null_and_misaligned(lib):
    assert mb.mamba_state_update(None, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, None, 1, FAKE,
                                 _udims(), None, None) == mb.MS_ERR_NULL
    assert mb.mamba_state_update(FAKE + 2, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, None, 1, FAKE,
                                 _udims(), None, None) == mb.MS_ERR_ALIGN
    assert mb.mamba_state_update(FAKE, FAKE + 1, FAKE, FAKE, FAKE, FAKE, None, None, None, 1, FAKE,
                                 _udims(), None, None) == mb.MS_ERR_ALIGN


def test_device_check_without_gpu(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present; this checks the no-device answer")
    assert mb.mamba_device_check() == mb.MS_ERR_CUDA


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(mb, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(mb, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        mb.library()


def _long_dims(batch=1, dim=2048, L=131072, N=16):
    return _dims(batch=batch, dim=dim, dstate=N, seqlen=L, u_sb=dim * L, u_sd=L, delta_sb=dim * L, delta_sd=L,
                 z_sb=dim * L, z_sd=L, y_sb=dim * L, y_sd=L, B_sb=N * L, B_sn=L, C_sb=N * L, C_sn=L)


def test_sequence_split_workspace(lib):
    # few channels and a long sequence: the sequence is split and the call
    # needs a workspace for the segments' end states, Delta sums, initial and
    # last states (16-byte aligned regions); no split otherwise
    ws = mb.mamba_scan_workspace_size(_long_dims())
    assert ws > 0 and ws % 16 == 0
    dim, N = 2048, 16
    S = None
    for s in range(2, 257):   # the workspace is a whole-region formula in S
        if ((s - 1) * dim * N + (s - 1) * dim + 2 * s * dim * N) * 4 == ws:
            S = s
    assert S is not None and 131072 % S == 0 and (131072 // S) % 64 == 0
    assert mb.mamba_scan_workspace_size(_long_dims(L=4096)) == 0            # short: no split
    assert mb.mamba_scan_workspace_size(_long_dims(batch=8, dim=1536)) == 0  # many channels: no split
    # a split call without its workspace is refused before any launch
    assert _scan(_long_dims(), ws=None, ws_bytes=0) == mb.MS_ERR_WORKSPACE
    assert _scan(_long_dims(), ws=FAKE, ws_bytes=ws - 16) == mb.MS_ERR_WORKSPACE
