"""ctypes wrapper around the fp64 C oracle (``mamba_oracle.c``).

TEST INFRASTRUCTURE ONLY (tests, smoke check, benchmark CPU-baseline leg).

Every array is converted to a dense float64 numpy array before the call; bf16
inputs must already be widened by the caller from the very bf16 values the GPU
reads (bf16 -> fp32 -> fp64 is exact), so both sides see identical inputs.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import tempfile
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mamba_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

_dp = ctypes.POINTER(ctypes.c_double)


def build_oracle(out_path: str = _LIB, mutant: int = 0, force: bool = False) -> str:
    """Compile the oracle with gcc -O2 (no fast-math). ``mutant`` != 0 plants
    the numbered mistake (tests only) and must go to a separate path."""
    if mutant and os.path.abspath(out_path) == os.path.abspath(_LIB):
        raise ValueError("a mutant oracle must not overwrite the real one")
    if not force and os.path.exists(out_path) and os.path.getmtime(out_path) >= os.path.getmtime(_SRC):
        return out_path
    tmp = out_path + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
           f"-DORACLE_MUTANT={int(mutant)}", _SRC, "-o", tmp, "-lm", "-lpthread"]
    subprocess.run(cmd, check=True, capture_output=True)
    os.replace(tmp, out_path)
    return out_path


def _declare(lib: ctypes.CDLL) -> ctypes.CDLL:
    i64 = ctypes.c_int64
    lib.oracle_softplus.argtypes = [ctypes.c_double]
    lib.oracle_softplus.restype = ctypes.c_double
    lib.oracle_silu.argtypes = [ctypes.c_double]
    lib.oracle_silu.restype = ctypes.c_double
    lib.oracle_scan_f64.argtypes = [i64, i64, i64, i64] + [_dp] * 8 + [ctypes.c_int, _dp, _dp, _dp]
    lib.oracle_scan_f64.restype = ctypes.c_int
    lib.oracle_scan_f64_mt.argtypes = [ctypes.c_int, i64, i64, i64, i64] + [_dp] * 8 + [ctypes.c_int, _dp, _dp, _dp]
    lib.oracle_scan_f64_mt.restype = ctypes.c_int
    lib.oracle_state_update_f64.argtypes = [i64, i64, i64] + [_dp] * 9 + [ctypes.c_int, _dp]
    lib.oracle_state_update_f64.restype = ctypes.c_int
    lib.oracle_causal_conv_f64.argtypes = [i64, i64, i64, i64] + [_dp] * 4 + [ctypes.c_int, _dp]
    lib.oracle_causal_conv_f64.restype = ctypes.c_int
    lib.oracle_scan_bwd_f64.argtypes = [i64, i64, i64, i64] + [_dp] * 8 + [ctypes.c_int] + [_dp] * 12
    lib.oracle_scan_bwd_f64.restype = ctypes.c_int
    lib.oracle_ssd_f64.argtypes = [i64] * 6 + [_dp] * 7 + [ctypes.c_int, _dp, _dp, _dp]
    lib.oracle_ssd_f64.restype = ctypes.c_int
    return lib


_cache: dict = {}


def load_oracle(path: Optional[str] = None) -> ctypes.CDLL:
    """Load (building first if needed) the oracle library; ``path`` selects a
    separately built variant (e.g. a mutant in a temporary directory)."""
    if path is None:
        path = build_oracle()
    if path not in _cache:
        _cache[path] = _declare(ctypes.CDLL(path))
    return _cache[path]


def _f64(a) -> Optional[np.ndarray]:
    if a is None:
        return None
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(_dp)


def softplus(x: float, lib=None) -> float:
    return (lib or load_oracle()).oracle_softplus(float(x))


def silu(x: float, lib=None) -> float:
    return (lib or load_oracle()).oracle_silu(float(x))


def _scan_args(u, delta, A, B, C, D, z, delta_bias, h0):
    u, delta, A, B, C = (_f64(a) for a in (u, delta, A, B, C))
    D, z, delta_bias, h0 = (_f64(a) for a in (D, z, delta_bias, h0))
    batch, dim, L = u.shape
    N = A.shape[1]
    assert delta.shape == u.shape and A.shape == (dim, N)
    assert B.shape == (batch, N, L) and C.shape == (batch, N, L)
    assert D is None or D.shape == (dim,)
    assert z is None or z.shape == u.shape
    assert delta_bias is None or delta_bias.shape == (dim,)
    assert h0 is None or h0.shape == (batch, dim, N)
    return u, delta, A, B, C, D, z, delta_bias, h0, batch, dim, N, L


def scan(u, delta, A, B, C, D=None, z=None, delta_bias=None, softplus_flag=True,
         h0=None, lib=None, nthreads: int = 1):
    """Selective scan in fp64. Shapes: u/delta/z [batch, dim, L]; A [dim, N];
    B/C [batch, N, L]; D/delta_bias [dim]; h0 [batch, dim, N] (zero if None).
    Returns (y [batch, dim, L], last_state [batch, dim, N])."""
    lib = lib or load_oracle()
    u, delta, A, B, C, D, z, delta_bias, h0, batch, dim, N, L = _scan_args(
        u, delta, A, B, C, D, z, delta_bias, h0)
    y = np.full((batch, dim, L), np.nan, dtype=np.float64)
    last = np.full((batch, dim, N), np.nan, dtype=np.float64)
    args = (batch, dim, N, L, _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
            _ptr(z), _ptr(delta_bias), int(bool(softplus_flag)), _ptr(h0), _ptr(y), _ptr(last))
    if nthreads > 1:
        rc = lib.oracle_scan_f64_mt(int(nthreads), *args)
    else:
        rc = lib.oracle_scan_f64(*args)
    if rc != 0:
        raise ValueError(f"oracle_scan_f64 rejected its arguments (rc={rc})")
    return y, last


def scan_mt(nthreads: int, *args, **kw):
    """``scan`` with the (batch, dim) channels split over ``nthreads`` threads."""
    return scan(*args, nthreads=nthreads, **kw)


def state_update(state, x, delta, A, B, C, D=None, z=None, delta_bias=None,
                 softplus_flag=True, lib=None):
    """One decode step in fp64. state [batch, dim, N] (not modified; the new
    state is returned); x/delta/z [batch, dim]; B/C [batch, N].
    Returns (y [batch, dim], new_state [batch, dim, N])."""
    lib = lib or load_oracle()
    st = np.array(state, dtype=np.float64, copy=True, order="C")
    x, delta, A, B, C = (_f64(a) for a in (x, delta, A, B, C))
    D, z, delta_bias = (_f64(a) for a in (D, z, delta_bias))
    batch, dim, N = st.shape
    assert x.shape == (batch, dim) and delta.shape == (batch, dim)
    assert A.shape == (dim, N) and B.shape == (batch, N) and C.shape == (batch, N)
    y = np.empty((batch, dim), dtype=np.float64)
    rc = lib.oracle_state_update_f64(batch, dim, N, _ptr(st), _ptr(x), _ptr(delta), _ptr(A),
                                     _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(delta_bias),
                                     int(bool(softplus_flag)), _ptr(y))
    if rc != 0:
        raise ValueError(f"oracle_state_update_f64 rejected its arguments (rc={rc})")
    return y, st


def scan_bwd(u, delta, A, B, C, D, z, delta_bias, softplus_flag, dout, h0=None, dlast=None, lib=None):
    """Gradients of the selective scan in fp64 for dL/dy = dout (and
    dL/dlast_state = dlast). Returns a dict du, ddelta, dA, dB, dC, dD, dz,
    ddelta_bias, dh0 (dD/dz/ddelta_bias None when D/z/delta_bias are None)."""
    lib = lib or load_oracle()
    u, delta, A, B, C, D, z, delta_bias, h0, batch, dim, N, L = _scan_args(
        u, delta, A, B, C, D, z, delta_bias, h0)
    dout, dlast = _f64(dout), _f64(dlast)
    assert dout.shape == u.shape and (dlast is None or dlast.shape == (batch, dim, N))
    g = {"du": np.full(u.shape, np.nan), "ddelta": np.full(u.shape, np.nan),
         "dA": np.zeros((dim, N)), "dB": np.zeros((batch, N, L)), "dC": np.zeros((batch, N, L)),
         "dD": None if D is None else np.zeros(dim), "dz": None if z is None else np.full(u.shape, np.nan),
         "ddelta_bias": None if delta_bias is None else np.zeros(dim),
         "dh0": np.full((batch, dim, N), np.nan)}
    rc = lib.oracle_scan_bwd_f64(batch, dim, N, L, _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                                 _ptr(z), _ptr(delta_bias), int(bool(softplus_flag)), _ptr(h0), _ptr(dout),
                                 _ptr(dlast), _ptr(g["du"]), _ptr(g["ddelta"]), _ptr(g["dA"]), _ptr(g["dB"]),
                                 _ptr(g["dC"]), _ptr(g["dD"]), _ptr(g["dz"]), _ptr(g["ddelta_bias"]),
                                 _ptr(g["dh0"]))
    if rc != 0:
        raise ValueError(f"oracle_scan_bwd_f64 rejected its arguments (rc={rc})")
    return g


def ssd(x, dt, A, B, C, D=None, dt_bias=None, softplus_flag=True, s0=None, lib=None):
    """Mamba-2 SSD layer, recurrent view, fp64. x [b, L, H, P]; dt [b, L, H];
    A, D, dt_bias [H]; B, C [b, L, G, N]; s0 [b, H, P, N] (zero if None).
    Returns (y [b, L, H, P], s_last [b, H, P, N])."""
    lib = lib or load_oracle()
    x, dt, A, B, C, D, dt_bias, s0 = (_f64(a) for a in (x, dt, A, B, C, D, dt_bias, s0))
    batch, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    assert dt.shape == (batch, L, H) and A.shape == (H,) and B.shape == (batch, L, G, N) and C.shape == B.shape
    assert s0 is None or s0.shape == (batch, H, P, N)
    y = np.full(x.shape, np.nan)
    last = np.full((batch, H, P, N), np.nan)
    rc = lib.oracle_ssd_f64(batch, L, H, P, N, G, _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                            _ptr(dt_bias), int(bool(softplus_flag)), _ptr(s0), _ptr(y), _ptr(last))
    if rc != 0:
        raise ValueError(f"oracle_ssd_f64 rejected its arguments (rc={rc})")
    return y, last


def ssd_chunk_cb(B, C, chunk: int = 32):
    """The intra-chunk products of the SSD matrix view ('Mamba-1/2/3
    Markdown図解' blog, section 3: inside a chunk the output is built from
    C_t . B_s of the chunk's tokens), fp64, by definition: for chunk k and
    i, j < chunk, cb[b, g, k, i, j] = sum_n C[b, k*chunk+i, g, n] *
    B[b, k*chunk+j, g, n], tokens at or past L counting as zero (one matrix
    product per chunk). B, C [b, L, G, N]; returns [b, G, ceil(L / chunk),
    chunk, chunk]."""
    B, C = _f64(B), _f64(C)
    batch, L, G, N = B.shape
    assert C.shape == B.shape
    nch = (L + chunk - 1) // chunk
    out = np.zeros((batch, G, nch, chunk, chunk))
    for k in range(nch):
        t0, t1 = k * chunk, min(L, (k + 1) * chunk)
        for b in range(batch):
            for g in range(G):
                out[b, g, k, : t1 - t0, : t1 - t0] = C[b, t0:t1, g, :] @ B[b, t0:t1, g, :].T
    return out


def causal_conv(x, w, bias=None, x0=None, silu_flag=True, lib=None):
    """Causal depthwise convolution + silu of the block's input path, fp64.
    x [batch, dim, L]; w [dim, W]; bias [dim]; x0 [batch, dim, W-1] (the W-1
    tokens before token 0; zero if None). Returns u [batch, dim, L]."""
    lib = lib or load_oracle()
    x, w, bias, x0 = (_f64(a) for a in (x, w, bias, x0))
    batch, dim, L = x.shape
    W = w.shape[1]
    assert w.shape == (dim, W) and (bias is None or bias.shape == (dim,))
    assert x0 is None or x0.shape == (batch, dim, W - 1)
    u = np.full((batch, dim, L), np.nan, dtype=np.float64)
    rc = lib.oracle_causal_conv_f64(batch, dim, L, W, _ptr(x), _ptr(w), _ptr(bias), _ptr(x0),
                                    int(bool(silu_flag)), _ptr(u))
    if rc != 0:
        raise ValueError(f"oracle_causal_conv_f64 rejected its arguments (rc={rc})")
    return u


def conv_scan(x, conv_w, conv_b, conv_x0, conv_silu, delta, A, B, C, D=None, z=None,
              delta_bias=None, softplus_flag=True, h0=None, lib=None, nthreads: int = 1):
    """The scan fed by the block's causal conv front-end: u = causal_conv(x),
    then the selective scan of u. Returns (y, last_state, u)."""
    lib = lib or load_oracle()
    u = causal_conv(x, conv_w, conv_b, conv_x0, conv_silu, lib=lib)
    y, last = scan(u, delta, A, B, C, D, z, delta_bias, softplus_flag, h0, lib=lib, nthreads=nthreads)
    return y, last, u


def mutant_library(mutant: int, directory: Optional[str] = None) -> ctypes.CDLL:
    """Build and load the oracle with planted mistake number ``mutant`` (tests)."""
    directory = directory or tempfile.mkdtemp(prefix="oracle_mutant_")
    path = os.path.join(directory, f"liboracle_mutant{mutant}.so")
    build_oracle(path, mutant=mutant, force=True)
    return load_oracle(path)
