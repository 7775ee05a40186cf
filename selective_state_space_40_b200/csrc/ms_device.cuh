// ms_device.cuh -- device helpers shared by the scan and state-update kernels:
// element loads, packed fp32x2 arithmetic (sm_100 `fma/mul/add .f32x2`), the
// exponential on the MUFU pipe and on the FMA pipe, softplus and silu.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace ms {

// ------------------------------------------------------ debug bounds checks --
// In the debug build (-DMS_DEBUG, libmambascan_debug.so) MS_CHECK(status, ok)
// evaluates `ok`; when it is false it ORs MS_ERR_BOUNDS (11) into the
// caller's device status word (when given) and yields false, and the guarded
// access is skipped: an index out of range is recorded, never performed. In
// the product build the check compiles to `true` (no cost).
constexpr int kErrBounds = 11;
__device__ __forceinline__ bool debug_check(int *status, bool ok) {
    if (!ok && status != nullptr) atomicOr(status, kErrBounds);
    return ok;
}
#ifdef MS_DEBUG
#define MS_CHECK(status, cond) ::ms::debug_check((status), (cond))
#else
#define MS_CHECK(status, cond) true
#endif

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// ---------------------------------------------------------------- elements --
__device__ __forceinline__ float bf16_bits_to_f32(uint32_t bits16) {
    return __uint_as_float(bits16 << 16);
}
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T> struct Elem;
template <> struct Elem<float> {
    static constexpr int kBytes = 4;
    __device__ __forceinline__ static float load(const float *p) { return __ldg(p); }
    __device__ __forceinline__ static void store(float *p, float v) { *p = v; }
};
template <> struct Elem<__nv_bfloat16> {
    static constexpr int kBytes = 2;
    __device__ __forceinline__ static float load(const __nv_bfloat16 *p) {
        return bf16_bits_to_f32(__ldg(reinterpret_cast<const unsigned short *>(p)));
    }
    __device__ __forceinline__ static void store(__nv_bfloat16 *p, float v) { *p = __float2bfloat16_rn(v); }
};

// ------------------------------------------------------- packed fp32 pairs --
// A pair of fp32 values in one 64-bit register pair; sm_100 executes the
// .f32x2 forms with one instruction for both lanes of the pair.
typedef unsigned long long f2;

__device__ __forceinline__ f2 f2_make(float lo, float hi) {
    f2 r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_split(f2 v, float &lo, float &hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ f2 f2_fma(f2 a, f2 b, f2 c) {
    f2 d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ f2 f2_mul(f2 a, f2 b) {
    f2 d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ f2 f2_add(f2 a, f2 b) {
    f2 d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ f2 f2_sub(f2 a, f2 b) {
    f2 d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ f2 f2_splat(float v) { return f2_make(v, v); }

// 16 bytes of shared memory straight into two fp32 pairs.
__device__ __forceinline__ void lds_f2x2(const float *p, f2 &a, f2 &b) {
    const unsigned addr = static_cast<unsigned>(__cvta_generic_to_shared(p));
    asm volatile("ld.shared.v2.b64 {%0, %1}, [%2];" : "=l"(a), "=l"(b) : "r"(addr));
}
// 8 bytes of shared memory straight into one fp32 pair.
__device__ __forceinline__ f2 lds_f2(const float *p) {
    const unsigned addr = static_cast<unsigned>(__cvta_generic_to_shared(p));
    f2 a;
    asm volatile("ld.shared.b64 %0, [%1];" : "=l"(a) : "r"(addr));
    return a;
}

// ------------------------------------------------------------ exponentials --
// 2^x on the MUFU pipe (16 per clock per SM on B200).
__device__ __forceinline__ float exp2_mufu(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float log2_mufu(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float rcp_mufu(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// 2^x on the FMA pipe: x = r + f with r = round(x) and |f| <= 1/2, then
// 2^f = 1 + f*q(f), q a degree-5 polynomial fitted here (linear program on a
// dense grid) for the least maximum relative error of q against (2^f - 1)/f;
// fp32 evaluation error <= 6.9e-8 relative, mean signed error ~1e-10. The last
// step is one rounded fma(f, q, 1), so for small |x| the result is 1 + (an
// accurate x*ln2 + ...) rounded to nearest: no systematic bias where the state
// decays slowly. 2^r is applied by adding r to the exponent field.
// Valid for x in [-125, 125]; callers clamp.
struct Exp2Poly {
    static constexpr float c0 = 0.6931471824645996f;
    static constexpr float c1 = 0.24022649228572845f;
    static constexpr float c2 = 0.05550345778465271f;
    static constexpr float c3 = 0.00961834006011486f;
    static constexpr float c4 = 0.0013397816801443696f;
    static constexpr float c5 = 0.00015364137652795762f;
    static constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
};

__device__ __forceinline__ float exp2_poly(float x) {
    x = fminf(fmaxf(x, -125.0f), 125.0f);
    const float t = x + Exp2Poly::kRound;  // r sits in the low mantissa bits
    const float r = t - Exp2Poly::kRound;
    const float f = x - r;
    float q = Exp2Poly::c5;
    q = fmaf(q, f, Exp2Poly::c4);
    q = fmaf(q, f, Exp2Poly::c3);
    q = fmaf(q, f, Exp2Poly::c2);
    q = fmaf(q, f, Exp2Poly::c1);
    q = fmaf(q, f, Exp2Poly::c0);
    const float p = fmaf(q, f, 1.0f);
    return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}

// Packed form of exp2_poly for a pair of arguments.
__device__ __forceinline__ f2 exp2_poly2(f2 x2) {
    float xa, xb;
    f2_split(x2, xa, xb);
    xa = fminf(fmaxf(xa, -125.0f), 125.0f);
    xb = fminf(fmaxf(xb, -125.0f), 125.0f);
    x2 = f2_make(xa, xb);
    const f2 t = f2_add(x2, f2_splat(Exp2Poly::kRound));
    const f2 r = f2_sub(t, f2_splat(Exp2Poly::kRound));
    const f2 f = f2_sub(x2, r);
    f2 q = f2_fma(f2_splat(Exp2Poly::c5), f, f2_splat(Exp2Poly::c4));
    q = f2_fma(q, f, f2_splat(Exp2Poly::c3));
    q = f2_fma(q, f, f2_splat(Exp2Poly::c2));
    q = f2_fma(q, f, f2_splat(Exp2Poly::c1));
    q = f2_fma(q, f, f2_splat(Exp2Poly::c0));
    const f2 p = f2_fma(q, f, f2_splat(1.0f));
    float pa, pb, ta, tb;
    f2_split(p, pa, pb);
    f2_split(t, ta, tb);
    pa = __int_as_float(__float_as_int(pa) + (__float_as_int(ta) << 23));
    pb = __int_as_float(__float_as_int(pb) + (__float_as_int(tb) << 23));
    return f2_make(pa, pb);
}

// exp2(y) - 1 for a pair with |y| <= 1/(2 ln 2) (|y ln 2| <= 1/2), by the
// Taylor series of expm1 in y ln 2 to degree 8: coefficient k is
// (ln 2)^k / k!; the first omitted term is below 5.4e-9, relative to the
// result under 1.4e-8. Used as A_bar - 1, so that h + (A_bar - 1) h keeps the
// low bits of a decay factor close to 1 that 1 + (A_bar - 1) would round off.
struct Expm1Series {
    static constexpr float c1 = 0.693147180559945f;
    static constexpr float c2 = 0.240226506959101f;
    static constexpr float c3 = 0.0555041086648216f;
    static constexpr float c4 = 0.00961812910762848f;
    static constexpr float c5 = 0.00133335581464284f;
    static constexpr float c6 = 0.000154035303933816f;
    static constexpr float c7 = 1.52527338040598e-05f;
    static constexpr float c8 = 1.32154867901443e-06f;
    static constexpr float kMaxArg = 0.721347520444482f;  // 1 / (2 ln 2)
};
__device__ __forceinline__ f2 exp2m1_series2(f2 y) {
    f2 q = f2_fma(y, f2_splat(Expm1Series::c8), f2_splat(Expm1Series::c7));
    q = f2_fma(q, y, f2_splat(Expm1Series::c6));
    q = f2_fma(q, y, f2_splat(Expm1Series::c5));
    q = f2_fma(q, y, f2_splat(Expm1Series::c4));
    q = f2_fma(q, y, f2_splat(Expm1Series::c3));
    q = f2_fma(q, y, f2_splat(Expm1Series::c2));
    q = f2_fma(q, y, f2_splat(Expm1Series::c1));
    return f2_mul(q, y);
}

__device__ __forceinline__ f2 exp2_mufu2(f2 x2) {
    float xa, xb;
    f2_split(x2, xa, xb);
    return f2_make(exp2_mufu(xa), exp2_mufu(xb));
}

template <bool kPoly>
__device__ __forceinline__ f2 exp2_pair(f2 x2) {
    if constexpr (kPoly) return exp2_poly2(x2);
    else return exp2_mufu2(x2);
}

// -------------------------------------------------------- softplus / silu --
// Default (MS_FMA_NONLIN 0): the exponential, the logarithm (softplus above its
// series range) and the reciprocal (silu) on the MUFU pipe. MS_FMA_NONLIN 1
// keeps only the exponential on MUFU and evaluates log1p and the reciprocal
// on the FMA pipe; timed side by side on one B200 that variant was slower in
// every kernel that uses them (selective scan 8.6 %, with the conv front-end
// 15 %, backward 3 %), so it stays as a compile-time option only.
#ifndef MS_FMA_NONLIN
#define MS_FMA_NONLIN 0
#endif

// log1p(e) / e on [0, 1]: the degree-9 polynomial through the Chebyshev
// nodes of the interval (fitted here in fp64, rounded to fp32). Evaluated in
// fp32, e * p(e) is within 1.6e-7 relative of log1p(e) on the whole interval,
// so no separate form is needed near 0 or near 1.
struct Log1pOverX {
    static constexpr float c0 = 1.0f;
    static constexpr float c1 = -0.49999892711639404f;
    static constexpr float c2 = 0.33329710364341736f;
    static constexpr float c3 = -0.24951615929603577f;
    static constexpr float c4 = 0.1966327428817749f;
    static constexpr float c5 = -0.1526966691017151f;
    static constexpr float c6 = 0.10543623566627502f;
    static constexpr float c7 = -0.056373611092567444f;
    static constexpr float c8 = 0.019542526453733444f;
    static constexpr float c9 = -0.0031760570127516985f;
};

// softplus(v) = max(v, 0) + log1p(e), e = exp(-|v|) in (0, 1] (given): accurate
// at both tails (large |v|: e -> 0 and the polynomial's relative accuracy holds).
__device__ __forceinline__ float softplus_e(float v, float e) {
#if MS_FMA_NONLIN
    float p = fmaf(Log1pOverX::c9, e, Log1pOverX::c8);
    p = fmaf(p, e, Log1pOverX::c7);
    p = fmaf(p, e, Log1pOverX::c6);
    p = fmaf(p, e, Log1pOverX::c5);
    p = fmaf(p, e, Log1pOverX::c4);
    p = fmaf(p, e, Log1pOverX::c3);
    p = fmaf(p, e, Log1pOverX::c2);
    p = fmaf(p, e, Log1pOverX::c1);
    p = fmaf(p, e, Log1pOverX::c0);
    return fmaxf(v, 0.0f) + e * p;
#else
    float s = fmaf(e, -1.0f / 6.0f, 0.2f);
    s = fmaf(e, s, -0.25f);
    s = fmaf(e, s, 1.0f / 3.0f);
    s = fmaf(e, s, -0.5f);
    s = fmaf(e, s, 1.0f);
    const float series = e * s;
    const float logform = log2_mufu(1.0f + e) * kLn2;
    return fmaxf(v, 0.0f) + (e < 0.0625f ? series : logform);
#endif
}
__device__ __forceinline__ float softplus_f(float v) { return softplus_e(v, exp2_mufu(-fabsf(v) * kLog2e)); }

// 1 / d for d in [1, 2] by Newton's iteration for the reciprocal: the linear
// seed 24/17 - 8/17 d (relative error at most 1/17 on the interval), then
// three steps r <- r + r (1 - d r), each squaring the relative error
// (fp32 result within 9e-8 relative).
__device__ __forceinline__ float rcp_1to2(float d) {
    float r = fmaf(-8.0f / 17.0f, d, 24.0f / 17.0f);
#pragma unroll
    for (int i = 0; i < 3; ++i) r = fmaf(r, fmaf(-d, r, 1.0f), r);
    return r;
}

// silu(z) = z sigma(z); sigma from e = exp(-|z|) in (0, 1]: 1 / (1 + e) for
// z >= 0, e / (1 + e) below, so the reciprocal always sees d in [1, 2].
__device__ __forceinline__ float silu_f(float z) {
#if MS_FMA_NONLIN
    const float e = exp2_mufu(-fabsf(z) * kLog2e);
    const float r = rcp_1to2(1.0f + e);
    return z * (z >= 0.0f ? r : e * r);
#else
    return z * rcp_mufu(1.0f + exp2_mufu(-z * kLog2e));
#endif
}

}  // namespace ms
