"""Thin ctypes binding of libmambascan.so (declared in include/mambascan.h).

The raw functions keep the C names and take plain integers (device addresses,
sizes, a stream handle). ``scan_fwd`` and ``state_update`` are conveniences
that read the addresses, strides and dtypes off torch CUDA tensors; they do
argument marshalling only, every step of the computation runs in the CUDA
library. A missing library raises: there is no CPU fallback.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
from typing import Optional, Tuple

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmambascan.so")

MS_F32, MS_BF16 = 0, 1
MS_OK, MS_ERR_NULL, MS_ERR_DTYPE, MS_ERR_SHAPE, MS_ERR_STRIDE = 0, 1, 2, 3, 4
MS_ERR_ALIGN, MS_ERR_WORKSPACE, MS_ERR_CUDA, MS_ERR_TIMEOUT, MS_ERR_DEVICE = 5, 6, 7, 8, 9
MS_ERR_SCRATCH, MS_ERR_BOUNDS = 10, 11
MS_BWD_NOALLOC_MAX_BYTES = 96 << 20
MS_MAX_DSTATE = 16
MS_ENGINE_REGISTER, MS_ENGINE_TMEM = 0, 1


class ScanDims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in (
        "batch", "dim", "dstate", "seqlen", "u_sb", "u_sd", "delta_sb", "delta_sd",
        "z_sb", "z_sd", "y_sb", "y_sd", "B_sb", "B_sn", "C_sb", "C_sn")] + [
        ("in_dtype", ctypes.c_int32), ("out_dtype", ctypes.c_int32)]


class UpdateDims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in (
        "batch", "dim", "dstate", "x_sb", "delta_sb", "z_sb", "y_sb", "B_sb", "C_sb",
        "state_sb", "state_sd")] + [("in_dtype", ctypes.c_int32), ("out_dtype", ctypes.c_int32)]


class ScanPlan(ctypes.Structure):
    _fields_ = [("lanes_per_channel", ctypes.c_int32), ("chunks_per_lane", ctypes.c_int32),
                ("poly8", ctypes.c_int32), ("engine", ctypes.c_int32)]


class ConvDims(ctypes.Structure):
    _fields_ = [("width", ctypes.c_int64), ("uout_sb", ctypes.c_int64), ("uout_sd", ctypes.c_int64),
                ("silu", ctypes.c_int32)]


class SsdDims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in (
        "batch", "seqlen", "nheads", "headdim", "dstate", "ngroups", "x_sb", "x_sl", "x_sh", "dt_sb", "dt_sl",
        "B_sb", "B_sl", "B_sg", "C_sb", "C_sl", "C_sg", "y_sb", "y_sl", "y_sh")] + [
        ("in_dtype", ctypes.c_int32), ("out_dtype", ctypes.c_int32)]


class SsdUpdateDims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in (
        "batch", "nheads", "headdim", "dstate", "ngroups", "x_sb", "x_sh", "dt_sb", "B_sb", "B_sg", "C_sb", "C_sg",
        "y_sb", "y_sh", "state_sb", "state_sh")] + [("in_dtype", ctypes.c_int32), ("out_dtype", ctypes.c_int32)]


class MambaScanError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: status {code} ({mamba_status_string(code)})")
        self.code = code


_lib = None
_loaded = {}
_vp = ctypes.c_void_p


def library() -> ctypes.CDLL:
    """Load libmambascan.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        _lib = _load(LIB_PATH)
    return _lib


@contextlib.contextmanager
def use_library(path: str):
    """Route every call of this module to another build of the library (the
    MS_DEBUG build, in the tests) inside the `with` block."""
    global _lib
    saved = library()
    _lib = _load(path)
    try:
        yield _lib
    finally:
        _lib = saved


def _load(path: str) -> ctypes.CDLL:
    if path not in _loaded:
        if not os.path.exists(path):
            raise RuntimeError(
                f"{path} is missing: build it with `python -m selective_state_space_40_b200.build`")
        lib = ctypes.CDLL(path)
        lib.mamba_scan_workspace_size.argtypes = [ctypes.POINTER(ScanDims)]
        lib.mamba_scan_workspace_size.restype = ctypes.c_size_t
        scan_args = [_vp] * 8 + [ctypes.c_int, _vp, _vp, _vp, ctypes.POINTER(ScanDims), _vp,
                                 ctypes.c_size_t, _vp, _vp]
        lib.mamba_scan_fwd.argtypes = scan_args
        lib.mamba_scan_fwd.restype = ctypes.c_int
        lib.mamba_scan_fwd_plan.argtypes = scan_args + [ctypes.POINTER(ScanPlan)]
        lib.mamba_scan_fwd_plan.restype = ctypes.c_int
        lib.mamba_scan_choose_plan.argtypes = [ctypes.POINTER(ScanDims), ctypes.POINTER(ScanPlan)]
        lib.mamba_scan_choose_plan.restype = ctypes.c_int
        lib.mamba_conv_scan_fwd.argtypes = ([_vp] * 5 + [ctypes.POINTER(ConvDims)] + [_vp] * 7 +
                                            [ctypes.c_int, _vp, _vp, _vp, ctypes.POINTER(ScanDims),
                                             ctypes.POINTER(ScanPlan), _vp, _vp])
        lib.mamba_conv_scan_fwd.restype = ctypes.c_int
        lib.mamba_scan_ckpt_size.argtypes = [ctypes.POINTER(ScanDims)]
        lib.mamba_scan_ckpt_size.restype = ctypes.c_size_t
        lib.mamba_scan_bwd_workspace_size.argtypes = [ctypes.POINTER(ScanDims)]
        lib.mamba_scan_bwd_workspace_size.restype = ctypes.c_size_t
        lib.mamba_scan_fwd_train.argtypes = [_vp] * 8 + [ctypes.c_int, _vp, _vp, _vp, _vp,
                                                         ctypes.POINTER(ScanDims), _vp, _vp]
        lib.mamba_scan_fwd_train.restype = ctypes.c_int
        lib.mamba_scan_bwd.argtypes = ([_vp] * 8 + [ctypes.c_int] + [_vp] * 13 +
                                       [ctypes.POINTER(ScanDims), _vp, ctypes.c_size_t, _vp, _vp])
        lib.mamba_scan_bwd.restype = ctypes.c_int
        lib.mamba_scan_bwd_noalloc.argtypes = ([_vp] * 8 + [ctypes.c_int] + [_vp] * 12 +
                                               [ctypes.POINTER(ScanDims), _vp, _vp])
        lib.mamba_scan_bwd_noalloc.restype = ctypes.c_int
        lib.mamba2_ssd_fwd.argtypes = [_vp] * 7 + [ctypes.c_int, _vp, _vp, _vp, ctypes.POINTER(SsdDims), _vp,
                                                   ctypes.c_size_t, _vp, _vp]
        lib.mamba2_ssd_fwd.restype = ctypes.c_int
        lib.mamba2_ssd_workspace_size.argtypes = [ctypes.POINTER(SsdDims)]
        lib.mamba2_ssd_workspace_size.restype = ctypes.c_size_t
        lib.mamba2_ssd_chunk_cb_size.argtypes = [ctypes.POINTER(SsdDims)]
        lib.mamba2_ssd_chunk_cb_size.restype = ctypes.c_size_t
        lib.mamba2_ssd_chunk_cb.argtypes = [_vp, _vp, _vp, ctypes.POINTER(SsdDims), _vp, _vp]
        lib.mamba2_ssd_chunk_cb.restype = ctypes.c_int
        lib.mamba2_ssd_state_update.argtypes = [_vp] * 8 + [ctypes.c_int, _vp, ctypes.POINTER(SsdUpdateDims),
                                                            _vp, _vp]
        lib.mamba2_ssd_state_update.restype = ctypes.c_int
        lib.mamba_state_update.argtypes = [_vp] * 9 + [ctypes.c_int, _vp, ctypes.POINTER(UpdateDims),
                                                       _vp, _vp]
        lib.mamba_state_update.restype = ctypes.c_int
        lib.mamba_status_string.argtypes = [ctypes.c_int]
        lib.mamba_status_string.restype = ctypes.c_char_p
        lib.mamba_debug_bounded_wait.argtypes = [ctypes.c_uint32, _vp, _vp]
        lib.mamba_debug_bounded_wait.restype = ctypes.c_int
        lib.mamba_device_check.argtypes = []
        lib.mamba_device_check.restype = ctypes.c_int
        lib.mamba_debug_bounds_probe.argtypes = [ctypes.c_int32, _vp, _vp]
        lib.mamba_debug_bounds_probe.restype = ctypes.c_int
        lib.mamba_debug_build.argtypes = []
        lib.mamba_debug_build.restype = ctypes.c_int
        _loaded[path] = lib
    return _loaded[path]


# ------------------------------------------------------------ raw C entry ----

def mamba_status_string(code: int) -> str:
    return library().mamba_status_string(int(code)).decode()


def mamba_device_check() -> int:
    return library().mamba_device_check()


def mamba_debug_build() -> int:
    return library().mamba_debug_build()


def mamba_debug_bounds_probe(index: int, dev_status, stream) -> int:
    return library().mamba_debug_bounds_probe(int(index), dev_status, stream)


def mamba_debug_bounded_wait(rounds: int, dev_status, stream) -> int:
    return library().mamba_debug_bounded_wait(int(rounds), dev_status, stream)


def mamba_scan_workspace_size(dims: ScanDims) -> int:
    return library().mamba_scan_workspace_size(ctypes.byref(dims))


def mamba_scan_choose_plan(dims: ScanDims) -> Tuple[int, ScanPlan]:
    plan = ScanPlan()
    rc = library().mamba_scan_choose_plan(ctypes.byref(dims), ctypes.byref(plan))
    return rc, plan


def mamba_scan_fwd(u, delta, A, B, C, D, z, delta_bias, softplus_flag, initial_state, y, last_state,
                   dims: ScanDims, workspace, workspace_bytes, dev_status, stream,
                   plan: Optional[ScanPlan] = None) -> int:
    lib = library()
    args = (u, delta, A, B, C, D, z, delta_bias, int(softplus_flag), initial_state, y, last_state,
            ctypes.byref(dims), workspace, int(workspace_bytes), dev_status, stream)
    if plan is None:
        return lib.mamba_scan_fwd(*args)
    return lib.mamba_scan_fwd_plan(*args, ctypes.byref(plan))


def mamba_scan_ckpt_size(dims: ScanDims) -> int:
    return library().mamba_scan_ckpt_size(ctypes.byref(dims))


def mamba_scan_bwd_workspace_size(dims: ScanDims) -> int:
    return library().mamba_scan_bwd_workspace_size(ctypes.byref(dims))


def mamba_scan_fwd_train(u, delta, A, B, C, D, z, delta_bias, softplus_flag, initial_state, y, last_state,
                         ckpt, dims: ScanDims, dev_status, stream) -> int:
    return library().mamba_scan_fwd_train(u, delta, A, B, C, D, z, delta_bias, int(softplus_flag),
                                          initial_state, y, last_state, ckpt, ctypes.byref(dims),
                                          dev_status, stream)


def mamba_scan_bwd(u, delta, A, B, C, D, z, delta_bias, softplus_flag, initial_state, ckpt, dout, dlast,
                   du, ddelta, dA, dB, dC, dD, dz, ddelta_bias, dinitial_state, dims: ScanDims,
                   workspace, workspace_bytes, dev_status, stream) -> int:
    return library().mamba_scan_bwd(u, delta, A, B, C, D, z, delta_bias, int(softplus_flag), initial_state,
                                    ckpt, dout, dlast, du, ddelta, dA, dB, dC, dD, dz, ddelta_bias,
                                    dinitial_state, ctypes.byref(dims), workspace, int(workspace_bytes),
                                    dev_status, stream)


def mamba_scan_bwd_noalloc(u, delta, A, B, C, D, z, delta_bias, softplus_flag, initial_state, dout, dlast,
                           du, ddelta, dA, dB, dC, dD, dz, ddelta_bias, dinitial_state, dims: ScanDims,
                           dev_status, stream) -> int:
    return library().mamba_scan_bwd_noalloc(u, delta, A, B, C, D, z, delta_bias, int(softplus_flag),
                                            initial_state, dout, dlast, du, ddelta, dA, dB, dC, dD, dz,
                                            ddelta_bias, dinitial_state, ctypes.byref(dims), dev_status, stream)


def mamba2_ssd_chunk_cb_size(dims: SsdDims) -> int:
    return library().mamba2_ssd_chunk_cb_size(ctypes.byref(dims))


def mamba2_ssd_chunk_cb(B, C, cb, dims: SsdDims, dev_status=None, stream=None) -> int:
    return library().mamba2_ssd_chunk_cb(B, C, cb, ctypes.byref(dims), dev_status, stream)


def mamba2_ssd_workspace_size(dims: SsdDims) -> int:
    return int(library().mamba2_ssd_workspace_size(ctypes.byref(dims)))


def mamba2_ssd_fwd(x, dt, A, B, C, D, dt_bias, softplus_flag, initial_state, y, final_state, dims: SsdDims,
                   workspace, workspace_bytes, dev_status, stream) -> int:
    return library().mamba2_ssd_fwd(x, dt, A, B, C, D, dt_bias, int(softplus_flag), initial_state, y, final_state,
                                    ctypes.byref(dims), workspace, workspace_bytes, dev_status, stream)


def mamba2_ssd_state_update(state, x, dt, A, B, C, D, dt_bias, softplus_flag, y, dims: SsdUpdateDims,
                            dev_status, stream) -> int:
    return library().mamba2_ssd_state_update(state, x, dt, A, B, C, D, dt_bias, int(softplus_flag), y,
                                             ctypes.byref(dims), dev_status, stream)


def mamba_conv_scan_fwd(x, conv_w, conv_b, conv_x0, u_out, cdims: ConvDims, delta, A, B, C, D, z,
                        delta_bias, softplus_flag, initial_state, y, last_state, dims: ScanDims,
                        plan: Optional[ScanPlan], dev_status, stream) -> int:
    return library().mamba_conv_scan_fwd(
        x, conv_w, conv_b, conv_x0, u_out, ctypes.byref(cdims), delta, A, B, C, D, z, delta_bias,
        int(softplus_flag), initial_state, y, last_state, ctypes.byref(dims),
        None if plan is None else ctypes.byref(plan), dev_status, stream)


def mamba_state_update(state, x, delta, A, B, C, D, z, delta_bias, softplus_flag, y,
                       dims: UpdateDims, dev_status, stream) -> int:
    return library().mamba_state_update(state, x, delta, A, B, C, D, z, delta_bias,
                                        int(softplus_flag), y, ctypes.byref(dims), dev_status, stream)


# ----------------------------------------------------- torch conveniences ----

def _torch():
    import torch
    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.float32:
        return MS_F32
    if t.dtype == torch.bfloat16:
        return MS_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream_handle(stream) -> Optional[int]:
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _inner_contiguous(t, name):
    if t is not None and t.numel() > 0 and t.stride(-1) != 1:
        raise ValueError(f"{name} must have unit stride along its last dimension")


def _check_f32(**tensors):
    """Parameters and states cross the C ABI as dense fp32 arrays."""
    torch = _torch()
    for n, t in tensors.items():
        if t is not None and (t.dtype != torch.float32 or not t.is_contiguous()):
            raise ValueError(f"{n} must be a contiguous fp32 tensor")


def scan_dims_for(u, delta, B, C, z, y) -> ScanDims:
    """ScanDims read off tensors u/delta/z/y [b, d, L] and B/C [b, N, L]."""
    for t, n in ((u, "u"), (delta, "delta"), (B, "B"), (C, "C"), (z, "z"), (y, "y")):
        _inner_contiguous(t, n)
    batch, dim, L = u.shape
    N = B.shape[1]
    zz = z if z is not None else u
    return ScanDims(batch, dim, N, L, u.stride(0), u.stride(1), delta.stride(0), delta.stride(1),
                    zz.stride(0), zz.stride(1), y.stride(0), y.stride(1), B.stride(0), B.stride(1),
                    C.stride(0), C.stride(1), _dtype_code(u), _dtype_code(y))


def scan_fwd(u, delta, A, B, C, D=None, z=None, delta_bias=None, softplus: bool = True,
             initial_state=None, out_dtype=None, y=None, last_state=None,
             return_last_state: bool = True, stream=None, plan: Optional[Tuple[int, int, int]] = None,
             dev_status=None, workspace=None):
    """Selective scan forward on torch CUDA tensors (see include/mambascan.h).
    ``workspace`` (optional, uint8 CUDA tensor of at least
    ``mamba_scan_workspace_size`` bytes) is allocated per call when omitted.
    Returns (y, last_state or None)."""
    torch = _torch()
    if out_dtype is None:
        out_dtype = torch.float32
    batch, dim, L = u.shape
    N = A.shape[1]
    if y is None:
        y = torch.empty((batch, dim, L), dtype=out_dtype, device=u.device)
    if last_state is None and return_last_state:
        last_state = torch.empty((batch, dim, N), dtype=torch.float32, device=u.device)
    for t, n in ((A, "A"), (D, "D"), (delta_bias, "delta_bias"), (initial_state, "initial_state"),
                 (last_state, "last_state")):
        if t is not None and (t.dtype != torch.float32 or not t.is_contiguous()):
            raise ValueError(f"{n} must be a contiguous fp32 tensor")
    dims = scan_dims_for(u, delta, B, C, z, y)
    ws_bytes = mamba_scan_workspace_size(dims)
    if workspace is not None:
        ws, ws_bytes = workspace, workspace.numel() * workspace.element_size()
    else:
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=u.device) if ws_bytes else None
    pl = ScanPlan(*plan) if plan is not None else None
    rc = mamba_scan_fwd(_ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
                        _ptr(delta_bias), softplus, _ptr(initial_state), _ptr(y), _ptr(last_state),
                        dims, _ptr(ws), ws_bytes, _ptr(dev_status), _stream_handle(stream), pl)
    if rc != MS_OK:
        raise MambaScanError(rc, "mamba_scan_fwd")
    return y, last_state


def conv_scan_fwd(x, conv_w, delta, A, B, C, D=None, z=None, delta_bias=None, softplus: bool = True,
                  conv_b=None, conv_x0=None, conv_silu: bool = True, return_u: bool = False,
                  initial_state=None, out_dtype=None, y=None, last_state=None, u_out=None,
                  return_last_state: bool = True, stream=None,
                  plan: Optional[Tuple[int, int, int]] = None, dev_status=None):
    """Scan with the causal conv front-end on torch CUDA tensors (see
    include/mambascan.h, mamba_conv_scan_fwd): x [b, d, L] is the conv input,
    conv_w [d, W] fp32. Returns (y, last_state or None, u or None)."""
    torch = _torch()
    if out_dtype is None:
        out_dtype = torch.float32
    batch, dim, L = x.shape
    N = A.shape[1]
    if y is None:
        y = torch.empty((batch, dim, L), dtype=out_dtype, device=x.device)
    if last_state is None and return_last_state:
        last_state = torch.empty((batch, dim, N), dtype=torch.float32, device=x.device)
    if u_out is None and return_u:
        u_out = torch.empty((batch, dim, L), dtype=x.dtype, device=x.device)
    for t, n in ((A, "A"), (D, "D"), (delta_bias, "delta_bias"), (initial_state, "initial_state"),
                 (last_state, "last_state"), (conv_w, "conv_w"), (conv_b, "conv_b")):
        if t is not None and (t.dtype != torch.float32 or not t.is_contiguous()):
            raise ValueError(f"{n} must be a contiguous fp32 tensor")
    if conv_x0 is not None and (conv_x0.dtype != x.dtype or not conv_x0.is_contiguous()):
        raise ValueError("conv_x0 must be contiguous with the dtype of x")
    if u_out is not None and u_out.dtype != x.dtype:
        raise ValueError("u_out must have the dtype of x")
    _inner_contiguous(u_out, "u_out")
    dims = scan_dims_for(x, delta, B, C, z, y)
    uo = u_out if u_out is not None else x
    cdims = ConvDims(conv_w.shape[1], uo.stride(0), uo.stride(1), int(bool(conv_silu)))
    pl = ScanPlan(*plan) if plan is not None else None
    rc = mamba_conv_scan_fwd(_ptr(x), _ptr(conv_w), _ptr(conv_b), _ptr(conv_x0), _ptr(u_out), cdims,
                             _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(delta_bias),
                             softplus, _ptr(initial_state), _ptr(y), _ptr(last_state), dims, pl,
                             _ptr(dev_status), _stream_handle(stream))
    if rc != MS_OK:
        raise MambaScanError(rc, "mamba_conv_scan_fwd")
    return y, last_state, u_out


def scan_fwd_train(u, delta, A, B, C, D=None, z=None, delta_bias=None, softplus: bool = True,
                   initial_state=None, out_dtype=None, stream=None, dev_status=None):
    """Training forward: (y, last_state, ckpt), ckpt the saved states the
    backward recomputes from (fp32 [b, d, ceil(L/64), N])."""
    torch = _torch()
    if out_dtype is None:
        out_dtype = torch.float32
    batch, dim, L = u.shape
    N = A.shape[1]
    _check_f32(A=A, D=D, delta_bias=delta_bias, initial_state=initial_state)
    y = torch.empty((batch, dim, L), dtype=out_dtype, device=u.device)
    last = torch.empty((batch, dim, N), dtype=torch.float32, device=u.device)
    ckpt = torch.empty((batch, dim, (L + 63) // 64, N), dtype=torch.float32, device=u.device)
    dims = scan_dims_for(u, delta, B, C, z, y)
    rc = mamba_scan_fwd_train(_ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
                              _ptr(delta_bias), softplus, _ptr(initial_state), _ptr(y), _ptr(last), _ptr(ckpt),
                              dims, _ptr(dev_status), _stream_handle(stream))
    if rc != MS_OK:
        raise MambaScanError(rc, "mamba_scan_fwd_train")
    return y, last, ckpt


def scan_bwd(u, delta, A, B, C, D, z, delta_bias, softplus: bool, dout, dlast=None, initial_state=None,
             ckpt=None, want_dinitial: bool = True, stream=None, dev_status=None, workspace=None):
    """Gradients of the scan on torch CUDA tensors. dout has y's shape and
    dtype. Returns a dict du, ddelta, dA, dB, dC, dD, dz, ddelta_bias,
    dinitial_state (fp32; None where the input is None)."""
    torch = _torch()
    batch, dim, L = u.shape
    N = A.shape[1]
    dev = u.device
    _check_f32(A=A, D=D, delta_bias=delta_bias, initial_state=initial_state, ckpt=ckpt, dlast=dlast)
    f32 = dict(dtype=torch.float32, device=dev)
    g = {"du": torch.empty((batch, dim, L), **f32), "ddelta": torch.empty((batch, dim, L), **f32),
         "dA": torch.empty((dim, N), **f32), "dB": torch.empty((batch, N, L), **f32),
         "dC": torch.empty((batch, N, L), **f32),
         "dD": torch.empty(dim, **f32) if D is not None else None,
         "dz": torch.empty((batch, dim, L), **f32) if z is not None else None,
         "ddelta_bias": torch.empty(dim, **f32) if delta_bias is not None else None,
         "dinitial_state": torch.empty((batch, dim, N), **f32) if want_dinitial else None}
    dims = scan_dims_for(u, delta, B, C, z, dout)
    ws_bytes = 0 if ckpt is not None else mamba_scan_bwd_workspace_size(dims)
    if workspace is not None:
        ws, ws_bytes = workspace, workspace.numel() * workspace.element_size()
    else:
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev) if ws_bytes else None
    rc = mamba_scan_bwd(_ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(delta_bias),
                        softplus, _ptr(initial_state), _ptr(ckpt), _ptr(dout), _ptr(dlast), _ptr(g["du"]),
                        _ptr(g["ddelta"]), _ptr(g["dA"]), _ptr(g["dB"]), _ptr(g["dC"]), _ptr(g["dD"]),
                        _ptr(g["dz"]), _ptr(g["ddelta_bias"]), _ptr(g["dinitial_state"]), dims, _ptr(ws),
                        ws_bytes, _ptr(dev_status), _stream_handle(stream))
    if rc != MS_OK:
        raise MambaScanError(rc, "mamba_scan_bwd")
    return g


def scan_bwd_noalloc(u, delta, A, B, C, D, z, delta_bias, softplus: bool, dout, dlast=None,
                     initial_state=None, stream=None, dev_status=None):
    """scan_bwd through mamba_scan_bwd_noalloc (no saved states, no
    workspace: the library's fixed scratch). Output tensors are created here
    by torch; the library call itself allocates nothing."""
    torch = _torch()
    batch, dim, L = u.shape
    N = A.shape[1]
    _check_f32(A=A, D=D, delta_bias=delta_bias, initial_state=initial_state, dlast=dlast)
    f32 = dict(dtype=torch.float32, device=u.device)
    g = {"du": torch.empty((batch, dim, L), **f32), "ddelta": torch.empty((batch, dim, L), **f32),
         "dA": torch.empty((dim, N), **f32), "dB": torch.empty((batch, N, L), **f32),
         "dC": torch.empty((batch, N, L), **f32),
         "dD": torch.empty(dim, **f32) if D is not None else None,
         "dz": torch.empty((batch, dim, L), **f32) if z is not None else None,
         "ddelta_bias": torch.empty(dim, **f32) if delta_bias is not None else None,
         "dinitial_state": torch.empty((batch, dim, N), **f32)}
    dims = scan_dims_for(u, delta, B, C, z, dout)
    rc = mamba_scan_bwd_noalloc(_ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
                                _ptr(delta_bias), softplus, _ptr(initial_state), _ptr(dout), _ptr(dlast),
                                _ptr(g["du"]), _ptr(g["ddelta"]), _ptr(g["dA"]), _ptr(g["dB"]), _ptr(g["dC"]),
                                _ptr(g["dD"]), _ptr(g["dz"]), _ptr(g["ddelta_bias"]), _ptr(g["dinitial_state"]),
                                dims, _ptr(dev_status), _stream_handle(stream))
    if rc != MS_OK:
        raise MambaScanError(rc, "mamba_scan_bwd_noalloc")
    return g


def ssd_fwd(x, dt, A, B, C, D=None, dt_bias=None, softplus: bool = True, initial_state=None,
            out_dtype=None, return_final_state: bool = True, y=None, stream=None, dev_status=None,
            final_state=None, workspace=None):
    """Mamba-2 SSD layer forward on torch CUDA tensors: x [b, L, H, P], dt
    [b, L, H], B/C [b, L, G, N] (bf16), A/D/dt_bias [H] fp32. Returns (y,
    final_state [b, H, P, N] or None). ``final_state`` (fp32, dense) may be
    given to be written in place (it may be ``initial_state`` itself);
    ``workspace`` (uint8 CUDA tensor of at least ``mamba2_ssd_workspace_size``
    bytes) is allocated per call when omitted."""
    torch = _torch()
    if out_dtype is None:
        out_dtype = torch.float32
    batch, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    _check_f32(A=A, D=D, dt_bias=dt_bias, initial_state=initial_state)
    for t, n in ((x, "x"), (dt, "dt"), (B, "B"), (C, "C")):
        _inner_contiguous(t, n)
    if y is None:
        y = torch.empty((batch, L, H, P), dtype=out_dtype, device=x.device)
    fs = final_state
    if fs is None and return_final_state:
        fs = torch.empty((batch, H, P, N), dtype=torch.float32, device=x.device)
    if fs is not None:
        _check_f32(final_state=fs)
    dims = SsdDims(batch, L, H, P, N, G, x.stride(0), x.stride(1), x.stride(2), dt.stride(0), dt.stride(1),
                   B.stride(0), B.stride(1), B.stride(2), C.stride(0), C.stride(1), C.stride(2),
                   y.stride(0), y.stride(1), y.stride(2), _dtype_code(x), _dtype_code(y))
    ws_bytes = mamba2_ssd_workspace_size(dims)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=x.device)
    rc = mamba2_ssd_fwd(_ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(dt_bias), softplus,
                        _ptr(initial_state), _ptr(y), _ptr(fs), dims, _ptr(workspace),
                        workspace.numel() * workspace.element_size(), _ptr(dev_status), _stream_handle(stream))
    if rc != MS_OK:
        raise MambaScanError(rc, "mamba2_ssd_fwd")
    return y, fs


def ssd_chunk_cb(B, C, cb=None, stream=None, dev_status=None):
    """Per-chunk products C_t . B_s (chunks of 32 tokens) of B/C [b, L, G,
    128] bf16 CUDA tensors, through mamba2_ssd_chunk_cb (tcgen05 tensor
    cores). Returns cb [b, G, ceil(L / 32), 32, 32] fp32."""
    torch = _torch()
    batch, L, G, N = B.shape
    for t, n in ((B, "B"), (C, "C")):
        _inner_contiguous(t, n)
    if cb is None:
        cb = torch.empty((batch, G, (L + 31) // 32, 32, 32), dtype=torch.float32, device=B.device)
    dims = SsdDims(batch, L, 1, 64, N, G, 0, 0, 0, 0, 0, B.stride(0), B.stride(1), B.stride(2), C.stride(0),
                   C.stride(1), C.stride(2), 0, 0, 0, _dtype_code(B), MS_F32)
    rc = mamba2_ssd_chunk_cb(_ptr(B), _ptr(C), _ptr(cb), dims, _ptr(dev_status), _stream_handle(stream))
    if rc != MS_OK:
        raise MambaScanError(rc, "mamba2_ssd_chunk_cb")
    return cb


def ssd_state_update(state, x, dt, A, B, C, D=None, dt_bias=None, softplus: bool = True, out_dtype=None,
                     y=None, stream=None, dev_status=None):
    """One Mamba-2 decode step on torch CUDA tensors: state [b, H, P, 128]
    fp32 (updated in place), x [b, H, P], dt [b, H], B/C [b, G, 128].
    Returns y [b, H, P]."""
    torch = _torch()
    if out_dtype is None:
        out_dtype = torch.float32
    batch, H, P = x.shape
    G, N = B.shape[1], B.shape[2]
    _check_f32(A=A, D=D, dt_bias=dt_bias)
    if state.dtype != torch.float32 or state.stride(-1) != 1 or state.stride(-2) != N:
        raise ValueError("state must be fp32 with dense [headdim, dstate] blocks")
    for t, n in ((x, "x"), (dt, "dt"), (B, "B"), (C, "C")):
        _inner_contiguous(t, n)
    if y is None:
        y = torch.empty((batch, H, P), dtype=out_dtype, device=x.device)
    dims = SsdUpdateDims(batch, H, P, N, G, x.stride(0), x.stride(1), dt.stride(0), B.stride(0), B.stride(1),
                         C.stride(0), C.stride(1), y.stride(0), y.stride(1), state.stride(0), state.stride(1),
                         _dtype_code(x), _dtype_code(y))
    rc = mamba2_ssd_state_update(_ptr(state), _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(dt_bias),
                                 softplus, _ptr(y), dims, _ptr(dev_status), _stream_handle(stream))
    if rc != MS_OK:
        raise MambaScanError(rc, "mamba2_ssd_state_update")
    return y


def update_dims_for(state, x, delta, B, C, z, y) -> UpdateDims:
    for t, n in ((x, "x"), (delta, "delta"), (B, "B"), (C, "C"), (z, "z"), (y, "y"), (state, "state")):
        _inner_contiguous(t, n)
    batch, dim, N = state.shape
    zz = z if z is not None else x
    return UpdateDims(batch, dim, N, x.stride(0), delta.stride(0), zz.stride(0), y.stride(0),
                      B.stride(0), C.stride(0), state.stride(0), state.stride(1),
                      _dtype_code(x), _dtype_code(y))


def state_update(state, x, delta, A, B, C, D=None, z=None, delta_bias=None, softplus: bool = True,
                 out_dtype=None, y=None, stream=None, dev_status=None):
    """One decode step on torch CUDA tensors; ``state`` [b, d, N] fp32 is
    updated in place. Returns y [b, d]."""
    torch = _torch()
    if out_dtype is None:
        out_dtype = torch.float32
    if state.dtype != torch.float32:
        raise ValueError("state must be fp32")
    _check_f32(A=A, D=D, delta_bias=delta_bias)
    batch, dim, N = state.shape
    if y is None:
        y = torch.empty((batch, dim), dtype=out_dtype, device=state.device)
    dims = update_dims_for(state, x, delta, B, C, z, y)
    rc = mamba_state_update(_ptr(state), _ptr(x), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                            _ptr(z), _ptr(delta_bias), softplus, _ptr(y), dims, _ptr(dev_status),
                            _stream_handle(stream))
    if rc != MS_OK:
        raise MambaScanError(rc, "mamba_state_update")
    return y
