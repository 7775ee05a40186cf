"""Comparison rules shared by the GPU parity tests.

Tolerances (stated here, used everywhere):
* fp32 inputs, fp32 y: every element |g - r| <= 1e-4 * max(|r|, rms(r)), with
  rms over the compared tensor (a pure relative bound is undefined where the
  gated output crosses 0).
* bf16 inputs (the oracle is fed the same bf16 values, widened exactly):
  relative L2 ||g - r|| / ||r|| <= 2e-3 and max |g - r| <= 1e-2, on y and on
  the state separately.
* bf16 y: each element within one bf16 ulp of the oracle value (or within
  1e-4 * rms for values near 0), on top of the rule for the inputs' dtype
  applied to the fp32 reference.
"""
import numpy as np
import torch

FP32_REL = 1e-4
BF16_REL_L2 = 2e-3
BF16_MAX_ABS = 1e-2


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").to(torch.float64).numpy()


def check_fp32(g, r, what=""):
    g = np.asarray(g, dtype=np.float64)
    r = np.asarray(r, dtype=np.float64)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    rms = float(np.sqrt(np.mean(r * r))) if r.size else 0.0
    bound = FP32_REL * np.maximum(np.abs(r), rms)
    err = np.abs(g - r)
    worst = float(np.max(err / np.maximum(bound, 1e-300))) if r.size else 0.0
    assert np.all(err <= bound), f"{what}: max err/bound {worst:.3f} (max abs err {err.max():.3e}, rms {rms:.3e})"
    return worst


def check_bf16(g, r, what=""):
    g = np.asarray(g, dtype=np.float64)
    r = np.asarray(r, dtype=np.float64)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    nr = float(np.linalg.norm(r))
    rel = float(np.linalg.norm(g - r) / nr) if nr > 0 else float(np.linalg.norm(g))
    mx = float(np.max(np.abs(g - r))) if r.size else 0.0
    assert rel <= BF16_REL_L2 and mx <= BF16_MAX_ABS, f"{what}: rel L2 {rel:.3e}, max abs {mx:.3e}"
    return rel, mx


def check_out_bf16(g, r, what=""):
    """g: bf16 output widened; r: fp64 oracle."""
    g = np.asarray(g, dtype=np.float64)
    r = np.asarray(r, dtype=np.float64)
    rms = float(np.sqrt(np.mean(r * r))) if r.size else 0.0
    mag = np.maximum(np.abs(r), 1e-30)
    ulp = np.exp2(np.floor(np.log2(mag)) - 7)
    bound = np.maximum(ulp, FP32_REL * rms)
    err = np.abs(g - r)
    assert np.all(err <= bound), f"{what}: max err/bound {float(np.max(err / bound)):.3f}"


def check(g, r, in_dtype, what=""):
    if in_dtype == torch.bfloat16:
        return check_bf16(g, r, what)
    return check_fp32(g, r, what)
