"""Pins of the fp64 oracle to facts that do not come from the oracle itself.

Each pin is an independent formulation of something the Mamba pages (or plain
mathematics) fix, written without the oracle's code:

* time-invariant case == one long convolution ('Mamba (deep learning)' wiki
  page, state-space paragraph: constant A, B, C, Delta make the model an LTI
  convolution), kernel K_k = sum_n C_n A_bar_n^k Delta B_n, by direct O(L^2) sum;
* d_state = 1 closed form with cumulative step sums S_t (A_bar = exp(Delta*A),
  same paragraph, composed over tokens);
* zero input: the state only decays, h_k = h_0 * exp(A * sum_j Delta_j);
* brute force: h_T = sum_s (prod_{r>s} A_bar_r) B_bar_s u_s with explicit
  products, against the recurrence of the 'Mamba-1/2/3 Markdown図解' blog,
  section 1;
* decode == scan (blog, section 2: train/prefill by scan and one-token
  generation by recurrent update are the same model) and split/resume (only
  the state is carried between tokens);
* degenerate cases: B = 0, and Delta = 0 (A_bar = 1);
* softplus / silu special values and library routines (numpy logaddexp,
  scipy expit);
* the hand-worked cases in tests/golden/hand_worked.json;
* the gradients of the scan (reverse mode) against central finite differences
  of the forward oracle along random directions, for every input (u, delta,
  A, B, C, D, z, delta_bias, h0) with a loss on both y and last_state;
* the Mamba-2 SSD layer (blog, section 3: one model, a recurrent view and a
  matrix view): the matrix view written out directly, y_t = sum_{s<=t}
  (C_t . B_s) exp(A sum_{r=s+1..t} Delta_r) Delta_s x_s (+ initial state
  and D terms), O(L^2); the reduction of a scalar-per-head transition to the
  Mamba-1 oracle (every (head, p) a Mamba-1 channel whose A row is A_h); and
  split/resume (the state is what passes between chunks);
* the block's causal conv front-end (blog, section 2, block diagram: a short
  causal convolution per channel, then silu, feeds the SSM) against numpy's
  full convolution with the history prepended, one-hot filters as explicit
  token shifts, and split/resume of conv + scan with the conv history and the
  state carried.

``test_oracle_mutants.py`` plants known mistakes in the oracle and checks
that at least one of these pins fails for each.
"""
import json
import math
import os

import numpy as np
import pytest
from scipy.special import expit

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
TOL = 1e-12


def _rel(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    scale = max(np.max(np.abs(b)), 1e-300)
    return float(np.max(np.abs(a - b)) / scale)


def _softplus_ref(x):
    return np.logaddexp(0.0, x)


def _silu_ref(z):
    return z * expit(z)


# ---------------------------------------------------------------- pins ----

def pin_softplus_silu(lib):
    errs = []
    errs.append(abs(oracle.softplus(0.0, lib) - math.log(2.0)))
    for x in (-30.0, -3.5, -0.25, 0.7, 4.0, 19.0, 40.0):
        errs.append(abs(oracle.softplus(x, lib) - oracle.softplus(-x, lib) - x) / max(1.0, abs(x)))
        errs.append(abs(oracle.softplus(x, lib) - _softplus_ref(x)) / _softplus_ref(x))
        errs.append(abs(oracle.silu(x, lib) - oracle.silu(-x, lib) - x) / max(1.0, abs(x)))
        errs.append(abs(oracle.silu(x, lib) - _silu_ref(x)) / max(abs(_silu_ref(x)), 1e-300))
    errs.append(abs(oracle.silu(0.0, lib)))
    return max(errs)


def pin_lti_convolution(lib):
    rng = np.random.default_rng(11)
    b, d, N, L = 2, 3, 5, 40
    A = -rng.uniform(0.2, 3.0, size=(d, N))
    Bc = rng.standard_normal((b, N))
    Cc = rng.standard_normal((b, N))
    dt = rng.uniform(0.05, 0.5, size=(b, d))
    u = rng.standard_normal((b, d, L))
    z = rng.standard_normal((b, d, L))
    D = rng.standard_normal(d)
    delta = np.repeat(dt[:, :, None], L, axis=2)
    B = np.repeat(Bc[:, :, None], L, axis=2)
    C = np.repeat(Cc[:, :, None], L, axis=2)
    worst = 0.0
    for with_gate in (False, True):
        y, _ = oracle.scan(u, delta, A, B, C, D if with_gate else None, z if with_gate else None,
                           np.zeros(d), False, lib=lib)
        ref = np.empty_like(y)
        for bi in range(b):
            for di in range(d):
                k = np.arange(L)
                K = np.zeros(L)
                for n in range(N):
                    K += Cc[bi, n] * np.exp(dt[bi, di] * A[di, n]) ** k * dt[bi, di] * Bc[bi, n]
                conv = np.convolve(u[bi, di], K)[:L]
                if with_gate:
                    conv = (conv + D[di] * u[bi, di]) * _silu_ref(z[bi, di])
                ref[bi, di] = conv
        worst = max(worst, _rel(y, ref))
    return worst


def pin_n1_closed_form(lib):
    rng = np.random.default_rng(12)
    b, d, L = 2, 3, 50
    A = -rng.uniform(0.3, 2.0, size=(d, 1))
    u = rng.standard_normal((b, d, L))
    raw = rng.standard_normal((b, d, L))
    z = rng.standard_normal((b, d, L))
    B = rng.standard_normal((b, 1, L))
    C = rng.standard_normal((b, 1, L))
    D = rng.standard_normal(d)
    bias = rng.uniform(-2.0, 0.5, size=d)
    y, last = oracle.scan(u, raw, A, B, C, D, z, bias, True, lib=lib)
    ref = np.empty_like(y)
    ref_last = np.empty_like(last)
    for bi in range(b):
        for di in range(d):
            dt = _softplus_ref(raw[bi, di] + bias[di])
            S = np.cumsum(dt)
            for t in range(L):
                s = np.arange(t + 1)
                h = np.sum(np.exp(A[di, 0] * (S[t] - S[s])) * dt[s] * B[bi, 0, s] * u[bi, di, s])
                ref[bi, di, t] = (C[bi, 0, t] * h + D[di] * u[bi, di, t]) * _silu_ref(z[bi, di, t])
                if t == L - 1:
                    ref_last[bi, di, 0] = h
    return max(_rel(y, ref), _rel(last, ref_last))


def pin_zero_input_decay(lib):
    rng = np.random.default_rng(13)
    b, d, N, K = 2, 4, 6, 25
    A = -rng.uniform(0.1, 4.0, size=(d, N))
    h0 = rng.standard_normal((b, d, N))
    D = rng.standard_normal(d)
    bias = rng.uniform(-3.0, 0.0, size=d)
    h = h0.copy()
    S = np.zeros((b, d))
    worst = 0.0
    for k in range(K):
        raw = rng.standard_normal((b, d))
        z = rng.standard_normal((b, d))
        B = rng.standard_normal((b, N))
        C = rng.standard_normal((b, N))
        y, h = oracle.state_update(h, np.zeros((b, d)), raw, A, B, C, D, z, bias, True, lib=lib)
        S += _softplus_ref(raw + bias)
        h_ref = h0 * np.exp(A[None, :, :] * S[:, :, None])
        y_ref = np.einsum("bn,bdn->bd", C, h_ref) * _silu_ref(z)
        worst = max(worst, _rel(h, h_ref), _rel(y, y_ref))
    return worst


def pin_brute_force_products(lib):
    rng = np.random.default_rng(14)
    b, d, N, L = 1, 2, 3, 12
    A = -rng.uniform(0.1, 2.5, size=(d, N))
    u = rng.standard_normal((b, d, L))
    raw = rng.standard_normal((b, d, L))
    z = rng.standard_normal((b, d, L))
    B = rng.standard_normal((b, N, L))
    C = rng.standard_normal((b, N, L))
    D = rng.standard_normal(d)
    bias = rng.uniform(-1.0, 1.0, size=d)
    y, last = oracle.scan(u, raw, A, B, C, D, z, bias, True, lib=lib)
    ref = np.zeros_like(y)
    ref_last = np.zeros_like(last)
    for di in range(d):
        dt = [math.log1p(math.exp(raw[0, di, t] + bias[di])) for t in range(L)]
        for T in range(L):
            acc = 0.0
            for n in range(N):
                hT = 0.0
                for s in range(T + 1):
                    prod = 1.0
                    for r in range(s + 1, T + 1):
                        prod *= math.exp(dt[r] * A[di, n])
                    hT += prod * dt[s] * B[0, n, s] * u[0, di, s]
                acc += C[0, n, T] * hT
                if T == L - 1:
                    ref_last[0, di, n] = hT
            zz = z[0, di, T]
            ref[0, di, T] = (acc + D[di] * u[0, di, T]) * zz / (1.0 + math.exp(-zz))
    return max(_rel(y, ref), _rel(last, ref_last))


def pin_scan_equals_decode(lib):
    rng = np.random.default_rng(15)
    b, d, N, L = 2, 3, 4, 30
    A = -rng.uniform(0.1, 3.0, size=(d, N))
    u = rng.standard_normal((b, d, L))
    raw = rng.standard_normal((b, d, L))
    z = rng.standard_normal((b, d, L))
    B = rng.standard_normal((b, N, L))
    C = rng.standard_normal((b, N, L))
    D = rng.standard_normal(d)
    bias = rng.uniform(-2.0, 0.0, size=d)
    y, last = oracle.scan(u, raw, A, B, C, D, z, bias, True, lib=lib)
    h = np.zeros((b, d, N))
    ys = []
    for t in range(L):
        yt, h = oracle.state_update(h, u[:, :, t], raw[:, :, t], A, B[:, :, t], C[:, :, t], D,
                                    z[:, :, t], bias, True, lib=lib)
        ys.append(yt)
    return max(_rel(np.stack(ys, axis=2), y), _rel(h, last))


def pin_split_resume(lib):
    rng = np.random.default_rng(16)
    b, d, N, L, m = 2, 3, 4, 40, 17
    A = -rng.uniform(0.1, 3.0, size=(d, N))
    u = rng.standard_normal((b, d, L))
    raw = rng.standard_normal((b, d, L))
    z = rng.standard_normal((b, d, L))
    B = rng.standard_normal((b, N, L))
    C = rng.standard_normal((b, N, L))
    D = rng.standard_normal(d)
    bias = rng.uniform(-2.0, 0.0, size=d)
    y, last = oracle.scan(u, raw, A, B, C, D, z, bias, True, lib=lib)
    y1, h1 = oracle.scan(u[:, :, :m], raw[:, :, :m], A, B[:, :, :m], C[:, :, :m], D, z[:, :, :m],
                         bias, True, lib=lib)
    y2, h2 = oracle.scan(u[:, :, m:], raw[:, :, m:], A, B[:, :, m:], C[:, :, m:], D, z[:, :, m:],
                         bias, True, h0=h1, lib=lib)
    return max(_rel(np.concatenate([y1, y2], axis=2), y), _rel(h2, last))


def pin_degenerate(lib):
    rng = np.random.default_rng(17)
    b, d, N, L = 2, 3, 4, 20
    A = -rng.uniform(0.1, 3.0, size=(d, N))
    u = rng.standard_normal((b, d, L))
    raw = rng.standard_normal((b, d, L))
    z = rng.standard_normal((b, d, L))
    C = rng.standard_normal((b, N, L))
    D = rng.standard_normal(d)
    bias = rng.uniform(-2.0, 0.0, size=d)
    # B = 0: nothing is written into the state.
    y, last = oracle.scan(u, raw, A, np.zeros((b, N, L)), C, D, z, bias, True, lib=lib)
    e1 = max(_rel(y, D[None, :, None] * u * _silu_ref(z)), float(np.max(np.abs(last))))
    # Delta = 0 (softplus off, raw = -bias): A_bar = 1 and the input term is 0,
    # so the state keeps h0 and y_t = C_t . h0 + D u_t, gated.
    h0 = rng.standard_normal((b, d, N))
    Bn = rng.standard_normal((b, N, L))
    raw0 = np.repeat(-bias[None, :, None], b, axis=0).repeat(L, axis=2)
    y, last = oracle.scan(u, raw0, A, Bn, C, D, z, bias, False, h0=h0, lib=lib)
    y_ref = (np.einsum("bnt,bdn->bdt", C, h0) + D[None, :, None] * u) * _silu_ref(z)
    e2 = max(_rel(y, y_ref), _rel(last, h0))
    return max(e1, e2)


def pin_hand_worked(lib):
    with open(os.path.join(HERE, "golden", "hand_worked.json")) as f:
        cases = json.load(f)["cases"]
    worst = 0.0
    for c in cases:
        arr = {k: (None if c[k] is None else np.array(c[k], dtype=np.float64))
               for k in ("u", "delta", "A", "B", "C", "D", "z", "delta_bias")}
        y, last = oracle.scan(arr["u"], arr["delta"], arr["A"], arr["B"], arr["C"], arr["D"],
                              arr["z"], arr["delta_bias"], c["softplus"], lib=lib)
        if "y_over_ln2" in c:
            y_ref = np.array(c["y_over_ln2"]) * math.log(2.0)
        else:
            y_ref = np.array(c["y_over_ln3"]) * math.log(3.0)
        last_ref = np.array(c["last_state_over_ln2"]) * math.log(2.0)
        worst = max(worst, float(np.max(np.abs(y - y_ref))), float(np.max(np.abs(last - last_ref))))
    return worst


def _conv_ref(x, w, bias, x0, silu_flag):
    """u_t = act(bias + sum_k w_k x_{t-(W-1)+k}) from numpy's full convolution
    of the history-prepended row with the reversed filter."""
    b, d, L = x.shape
    W = w.shape[1]
    u = np.empty((b, d, L))
    for bi in range(b):
        for di in range(d):
            hist = np.zeros(W - 1) if x0 is None else x0[bi, di]
            full = np.convolve(np.concatenate([hist, x[bi, di]]), w[di, ::-1])
            v = full[W - 1:W - 1 + L] + (0.0 if bias is None else bias[di])
            u[bi, di] = _silu_ref(v) if silu_flag else v
    return u


def pin_conv_numpy(lib):
    rng = np.random.default_rng(18)
    worst = 0.0
    for W in (1, 2, 3, 4):
        b, d, L = 2, 3, 29
        x = rng.standard_normal((b, d, L))
        w = rng.standard_normal((d, W))
        bias = rng.standard_normal(d)
        x0 = rng.standard_normal((b, d, W - 1))
        for silu_flag in (False, True):
            for hist in (None, x0):
                u = oracle.causal_conv(x, w, bias, hist, silu_flag, lib=lib)
                worst = max(worst, _rel(u, _conv_ref(x, w, bias, hist, silu_flag)))
    return worst


def pin_conv_shift(lib):
    rng = np.random.default_rng(19)
    b, d, L, W = 1, 2, 15, 4
    x = rng.standard_normal((b, d, L))
    x0 = rng.standard_normal((b, d, W - 1))
    ext = np.concatenate([x0, x], axis=2)  # ext[..., s + W - 1] = x_s
    worst = 0.0
    for k in range(W):
        w = np.zeros((d, W))
        w[:, k] = 1.0
        u = oracle.causal_conv(x, w, None, x0, False, lib=lib)
        # tap k alone picks token t - (W-1) + k
        ref = np.stack([ext[:, :, t + k] for t in range(L)], axis=2)
        worst = max(worst, float(np.max(np.abs(u - ref))))
    return worst


def pin_conv_scan_split(lib):
    rng = np.random.default_rng(20)
    b, d, N, L, m, W = 2, 3, 4, 36, 13, 4
    A = -rng.uniform(0.1, 3.0, size=(d, N))
    x = rng.standard_normal((b, d, L))
    w = rng.standard_normal((d, W))
    cb = rng.standard_normal(d)
    raw = rng.standard_normal((b, d, L))
    z = rng.standard_normal((b, d, L))
    B = rng.standard_normal((b, N, L))
    C = rng.standard_normal((b, N, L))
    D = rng.standard_normal(d)
    bias = rng.uniform(-2.0, 0.0, size=d)
    y, last, u = oracle.conv_scan(x, w, cb, None, True, raw, A, B, C, D, z, bias, True, lib=lib)
    y1, h1, u1 = oracle.conv_scan(x[:, :, :m], w, cb, None, True, raw[:, :, :m], A, B[:, :, :m],
                                  C[:, :, :m], D, z[:, :, :m], bias, True, lib=lib)
    y2, h2, u2 = oracle.conv_scan(x[:, :, m:], w, cb, x[:, :, m - W + 1:m], True, raw[:, :, m:], A,
                                  B[:, :, m:], C[:, :, m:], D, z[:, :, m:], bias, True, h0=h1, lib=lib)
    return max(_rel(np.concatenate([y1, y2], axis=2), y), _rel(h2, last),
               _rel(np.concatenate([u1, u2], axis=2), u))


def pin_backward_finite_differences(lib):
    """Every gradient of oracle.scan_bwd against (L(x + eV) - L(x - eV)) / 2e
    with L = <dout, y> + <dlast, last_state>; returns the worst relative
    mismatch (central differences in fp64 reach ~1e-9 here)."""
    rng = np.random.default_rng(22)
    b, d, N, L = 2, 3, 4, 9
    x = dict(u=rng.standard_normal((b, d, L)), delta=rng.standard_normal((b, d, L)),
             A=-rng.uniform(0.2, 2.0, (d, N)), B=rng.standard_normal((b, N, L)),
             C=rng.standard_normal((b, N, L)), D=rng.standard_normal(d), z=rng.standard_normal((b, d, L)),
             delta_bias=rng.uniform(-1.5, 0.5, d), h0=rng.standard_normal((b, d, N)))
    dout = rng.standard_normal((b, d, L))
    dlast = rng.standard_normal((b, d, N))

    def loss(v):
        y, last = oracle.scan(v["u"], v["delta"], v["A"], v["B"], v["C"], v["D"], v["z"], v["delta_bias"],
                              True, h0=v["h0"], lib=lib)
        return float(np.sum(y * dout) + np.sum(last * dlast))

    g = oracle.scan_bwd(x["u"], x["delta"], x["A"], x["B"], x["C"], x["D"], x["z"], x["delta_bias"], True,
                        dout, h0=x["h0"], dlast=dlast, lib=lib)
    names = dict(u="du", delta="ddelta", A="dA", B="dB", C="dC", D="dD", z="dz", delta_bias="ddelta_bias",
                 h0="dh0")
    eps = 1e-5
    worst = 0.0
    for k, gk in names.items():
        for _ in range(2):
            V = rng.standard_normal(x[k].shape)
            xp = dict(x); xp[k] = x[k] + eps * V
            xm = dict(x); xm[k] = x[k] - eps * V
            fd = (loss(xp) - loss(xm)) / (2 * eps)
            an = float(np.sum(g[gk] * V))
            worst = max(worst, abs(fd - an) / max(abs(an), 1e-3))
    return worst


def _ssd_case(rng, b=2, L=23, H=4, P=3, N=5, G=2):
    return dict(x=rng.standard_normal((b, L, H, P)), dt=rng.standard_normal((b, L, H)),
                A=-rng.uniform(0.3, 2.5, H), B=rng.standard_normal((b, L, G, N)),
                C=rng.standard_normal((b, L, G, N)), D=rng.standard_normal(H), dt_bias=rng.uniform(-2.0, 0.0, H),
                s0=rng.standard_normal((b, H, P, N)))


def pin_ssd_matrix_view(lib):
    rng = np.random.default_rng(23)
    c = _ssd_case(rng)
    y, last = oracle.ssd(c["x"], c["dt"], c["A"], c["B"], c["C"], c["D"], c["dt_bias"], True, c["s0"], lib=lib)
    b, L, H, P = c["x"].shape
    G = c["B"].shape[2]
    ref = np.zeros_like(y)
    ref_last = np.zeros_like(last)
    for bi in range(b):
        for h in range(H):
            g = h // (H // G)
            dlt = _softplus_ref(c["dt"][bi, :, h] + c["dt_bias"][h])
            S = np.concatenate([[0.0], np.cumsum(dlt)])  # S[t+1] = sum_{r<=t} Delta_r
            for t in range(L):
                acc = np.exp(c["A"][h] * S[t + 1]) * (c["s0"][bi, h] @ c["C"][bi, t, g])  # initial state
                for s_ in range(t + 1):
                    w = (c["C"][bi, t, g] @ c["B"][bi, s_, g]) * np.exp(c["A"][h] * (S[t + 1] - S[s_ + 1])) * dlt[s_]
                    acc = acc + w * c["x"][bi, s_, h]
                ref[bi, t, h] = acc + c["D"][h] * c["x"][bi, t, h]
            st = np.exp(c["A"][h] * S[L]) * c["s0"][bi, h]
            for s_ in range(L):
                st = st + np.exp(c["A"][h] * (S[L] - S[s_ + 1])) * dlt[s_] * np.outer(c["x"][bi, s_, h], c["B"][bi, s_, g])
            ref_last[bi, h] = st
    return max(_rel(y, ref), _rel(last, ref_last))


def pin_ssd_is_mamba1_with_scalar_heads(lib):
    rng = np.random.default_rng(24)
    c = _ssd_case(rng)
    y, last = oracle.ssd(c["x"], c["dt"], c["A"], c["B"], c["C"], c["D"], c["dt_bias"], True, c["s0"], lib=lib)
    b, L, H, P = c["x"].shape
    G, N = c["B"].shape[2], c["B"].shape[3]
    worst = 0.0
    for h in range(H):
        g = h // (H // G)
        u = np.transpose(c["x"][:, :, h, :], (0, 2, 1))               # [b, P, L]
        delta = np.repeat(c["dt"][:, None, :, h], P, axis=1)           # [b, P, L]
        A1 = np.full((P, N), c["A"][h])
        B1 = np.transpose(c["B"][:, :, g, :], (0, 2, 1))               # [b, N, L]
        C1 = np.transpose(c["C"][:, :, g, :], (0, 2, 1))
        y1, l1 = oracle.scan(u, delta, A1, B1, C1, np.full(P, c["D"][h]), None, np.full(P, c["dt_bias"][h]),
                             True, h0=c["s0"][:, h], lib=lib)
        worst = max(worst, _rel(np.transpose(y[:, :, h, :], (0, 2, 1)), y1), _rel(last[:, h], l1))
    return worst


def pin_ssd_split_resume(lib):
    rng = np.random.default_rng(25)
    c = _ssd_case(rng, L=40)
    m = 17
    y, last = oracle.ssd(c["x"], c["dt"], c["A"], c["B"], c["C"], c["D"], c["dt_bias"], True, c["s0"], lib=lib)
    sl = lambda k, a, z: c[k][:, a:z]  # noqa: E731
    y1, l1 = oracle.ssd(sl("x", 0, m), sl("dt", 0, m), c["A"], sl("B", 0, m), sl("C", 0, m), c["D"], c["dt_bias"],
                        True, c["s0"], lib=lib)
    y2, l2 = oracle.ssd(sl("x", m, 40), sl("dt", m, 40), c["A"], sl("B", m, 40), sl("C", m, 40), c["D"],
                        c["dt_bias"], True, l1, lib=lib)
    return max(_rel(np.concatenate([y1, y2], axis=1), y), _rel(l2, last))



def pin_ssd_chunk_cb_is_intra_chunk_product(lib):
    # No decay (A = 0), Delta = 1 (no softplus, dt = 1, no bias), no D skip and
    # a zero state entering each chunk: the recurrence's output inside a chunk
    # is then exactly sum_{s <= t} (C_t . B_s) x_s, i.e. the lower triangle of
    # the chunk's cb block times x. Chunk 0 of a 40-token run, and chunk 1 as
    # a run of its own tokens from a zero state.
    rng = np.random.default_rng(26)
    b, L, H, P, N, G = 2, 40, 2, 3, 5, 2
    x = rng.standard_normal((b, L, H, P))
    B = rng.standard_normal((b, L, G, N))
    C = rng.standard_normal((b, L, G, N))
    cb = oracle.ssd_chunk_cb(B, C)
    worst = 0.0
    for k, (t0, t1) in enumerate(((0, 32), (32, 40))):
        n = t1 - t0
        y, _ = oracle.ssd(x[:, t0:t1], np.ones((b, n, H)), np.zeros(H), B[:, t0:t1], C[:, t0:t1], None, None,
                          False, None, lib=lib)
        for bi in range(b):
            for h in range(H):
                g = h // (H // G)
                ref = np.tril(cb[bi, g, k, :n, :n]) @ x[bi, t0:t1, h]
                worst = max(worst, _rel(y[bi, :, h], ref))
    # rows and columns past the sequence are zero
    worst = max(worst, float(np.abs(cb[:, :, 1, 8:, :]).max()), float(np.abs(cb[:, :, 1, :, 8:]).max()))
    return worst

PINS = {
    "softplus_silu": pin_softplus_silu,
    "lti_convolution": pin_lti_convolution,
    "n1_closed_form": pin_n1_closed_form,
    "zero_input_decay": pin_zero_input_decay,
    "brute_force_products": pin_brute_force_products,
    "scan_equals_decode": pin_scan_equals_decode,
    "split_resume": pin_split_resume,
    "degenerate": pin_degenerate,
    "hand_worked": pin_hand_worked,
    "conv_numpy": pin_conv_numpy,
    "conv_shift": pin_conv_shift,
    "conv_scan_split": pin_conv_scan_split,
    "backward_finite_differences": pin_backward_finite_differences,
    "ssd_matrix_view": pin_ssd_matrix_view,
    "ssd_is_mamba1_with_scalar_heads": pin_ssd_is_mamba1_with_scalar_heads,
    "ssd_split_resume": pin_ssd_split_resume,
    "ssd_chunk_cb_is_intra_chunk_product": pin_ssd_chunk_cb_is_intra_chunk_product,
}

# Pins that compare against a numerical approximation carry their own bound.
PIN_TOL = {"backward_finite_differences": 1e-7}


def pin_tol(name):
    return PIN_TOL.get(name, TOL)


@pytest.mark.parametrize("name", sorted(PINS))
def test_pin(name, oracle_lib):
    err = PINS[name](oracle_lib)
    assert err <= pin_tol(name), f"pin {name}: error {err:.3e} > {pin_tol(name):.0e}"


def test_multithreaded_oracle_is_identical(oracle_lib):
    rng = np.random.default_rng(21)
    b, d, N, L = 3, 7, 5, 33
    args = (rng.standard_normal((b, d, L)), rng.standard_normal((b, d, L)),
            -rng.uniform(0.1, 3, (d, N)), rng.standard_normal((b, N, L)),
            rng.standard_normal((b, N, L)), rng.standard_normal(d),
            rng.standard_normal((b, d, L)), rng.uniform(-2, 0, d))
    y1, h1 = oracle.scan(*args, lib=oracle_lib)
    y4, h4 = oracle.scan_mt(4, *args, lib=oracle_lib)
    assert np.array_equal(y1, y4) and np.array_equal(h1, h4)


def test_oracle_rejects_bad_sizes(oracle_lib):
    dp = None
    assert oracle_lib.oracle_scan_f64(1, 1, 0, 4, *([dp] * 8), 1, dp, dp, dp) == -1
    assert oracle_lib.oracle_scan_f64(1, 1, 4, 4, *([dp] * 8), 1, dp, dp, dp) == -1
