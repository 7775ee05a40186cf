"""Comparison rules shared by the GPU parity tests.

Tolerances (stated here, used everywhere):
* fp32 inputs, fp32 y: every element |g - r| <= 1e-4 * max(|r|, rms(r)), with
  rms over the compared tensor (a pure relative bound is undefined where the
  gated output crosses 0).
* bf16 inputs (the oracle is fed the same bf16 values, widened exactly):
  relative L2 ||g - r|| / ||r|| <= 2e-3 and max |g - r| <= 1e-2, on y and on
  the state separately.
* inputs far from unit scale (the tail cases: steps up to ~55, gates up to
  40, so outputs reach ~1e5): the same two rules, with the bf16 rule's
  absolute bound scaled by max(1, rms(r)); the relative bounds are unchanged.
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


def check_bf16(g, r, what="", scaled=False):
    g = np.asarray(g, dtype=np.float64)
    r = np.asarray(r, dtype=np.float64)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    nr = float(np.linalg.norm(r))
    rel = float(np.linalg.norm(g - r) / nr) if nr > 0 else float(np.linalg.norm(g))
    mx = float(np.max(np.abs(g - r))) if r.size else 0.0
    bound = BF16_MAX_ABS
    if scaled and r.size:
        bound *= max(1.0, float(np.sqrt(np.mean(r * r))))
    assert rel <= BF16_REL_L2 and mx <= bound, f"{what}: rel L2 {rel:.3e}, max abs {mx:.3e} (bound {bound:.3e})"
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


def check(g, r, in_dtype, what="", scaled=False):
    if in_dtype == torch.bfloat16:
        return check_bf16(g, r, what, scaled=scaled)
    return check_fp32(g, r, what)


class StreamCheck:
    """The rule of ``check`` applied to a tensor compared in pieces (every
    element, without holding the whole reference at once).

    fp32 rule: an element passes when err <= 1e-4 |r| or err <= 1e-4 rms(r);
    so the pieces keep the largest error among elements failing the first
    test, and at the end that error must be within 1e-4 of the global rms.
    bf16 rule: sums of squared differences and of squared references, and
    the largest absolute difference.
    """

    def __init__(self, in_dtype, what=""):
        self.bf16 = in_dtype == torch.bfloat16
        self.what = what
        self.n = 0
        self.sum_r2 = 0.0
        self.sum_d2 = 0.0
        self.max_abs = 0.0
        self.max_unexplained = 0.0

    def add(self, g, r):
        g = np.asarray(g, dtype=np.float64)
        r = np.asarray(r, dtype=np.float64)
        assert g.shape == r.shape, f"{self.what}: shape {g.shape} vs {r.shape}"
        assert np.all(np.isfinite(g)), f"{self.what}: non-finite output"
        err = np.abs(g - r)
        self.n += r.size
        self.sum_r2 += float(np.sum(r * r))
        self.sum_d2 += float(np.sum(err * err))
        if err.size:
            self.max_abs = max(self.max_abs, float(err.max()))
            bad = err > FP32_REL * np.abs(r)
            if bad.any():
                self.max_unexplained = max(self.max_unexplained, float(err[bad].max()))

    def finish(self):
        if self.bf16:
            nr = np.sqrt(self.sum_r2)
            rel = float(np.sqrt(self.sum_d2) / nr) if nr > 0 else float(np.sqrt(self.sum_d2))
            assert rel <= BF16_REL_L2 and self.max_abs <= BF16_MAX_ABS, \
                f"{self.what}: rel L2 {rel:.3e}, max abs {self.max_abs:.3e} over {self.n} elements"
            return rel, self.max_abs
        rms = float(np.sqrt(self.sum_r2 / self.n)) if self.n else 0.0
        assert self.max_unexplained <= FP32_REL * rms, \
            f"{self.what}: error {self.max_unexplained:.3e} above 1e-4 |r| and 1e-4 rms ({rms:.3e})"
        return self.max_unexplained / max(FP32_REL * rms, 1e-300)
