// ssd_update.cu -- Mamba-2 SSD layer, one-token state update (decode) on sm_100a.
//
// 'Mamba-1/2/3 Markdown図解' blog, section 3: decoding runs the recurrent view
// of the SSD model, one state update per token. For batch row b and head h
// (state S [P x N] fp32, group g of B and C):
//   Delta = softplus(dt + dt_bias),  S = exp(Delta A_h) S + Delta x B^T,
//   y = S C + D x
// The state is read and written once (the step's traffic); one CTA of 8
// warps per (b, h): lane l owns columns n in [4l, 4l+4) (one 16-byte access
// per row), warps stride over the rows p, and each row's readout C . S is a
// warp sum.

#include <cstdint>

#include "ms_device.cuh"
#include "ms_internal.h"

namespace ms {

namespace {

constexpr int kUW = 8;  // warps per CTA

template <typename T>
__device__ __forceinline__ float ldv(const T *p) {
    if constexpr (sizeof(T) == 4) return __ldg(reinterpret_cast<const float *>(p));
    else return bf16_bits_to_f32(__ldg(reinterpret_cast<const unsigned short *>(p)));
}

template <typename TIn, typename TOut>
__global__ void __launch_bounds__(kUW * 32) ssd_update_kernel(const SsdUpdArgs a) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t b = blockIdx.x / a.H, h = blockIdx.x % a.H;
    const int64_t g = h / (a.H / a.G);
    const int P = a.P;
    constexpr int N = 128;
    const float v = ldv(static_cast<const TIn *>(a.dt) + b * a.dt_sb + h) + (a.dt_bias ? __ldg(a.dt_bias + h) : 0.0f);
    const float dl = a.softplus ? softplus_f(v) : v;
    const float decay = exp2_mufu(dl * __ldg(a.A + h) * kLog2e);
    const float Dh = a.D ? __ldg(a.D + h) : 0.0f;
    const TIn *Bp = static_cast<const TIn *>(a.B) + b * a.B_sb + g * a.B_sg + 4 * lane;
    const TIn *Cp = static_cast<const TIn *>(a.C) + b * a.C_sb + g * a.C_sg + 4 * lane;
    float Bv[4], Cv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        Bv[i] = dl * ldv(Bp + i);
        Cv[i] = ldv(Cp + i);
    }
    const TIn *xr = static_cast<const TIn *>(a.x) + b * a.x_sb + h * a.x_sh;
    TOut *yr = static_cast<TOut *>(a.y) + b * a.y_sb + h * a.y_sh;
    float *st = a.state + b * a.st_sb + h * a.st_sh + 4 * lane;
#pragma unroll 4
    for (int p = warp; p < P; p += kUW) {
        float4 s = *reinterpret_cast<const float4 *>(st + (int64_t)p * N);
        const float xv = ldv(xr + p);
        s.x = fmaf(decay, s.x, xv * Bv[0]);
        s.y = fmaf(decay, s.y, xv * Bv[1]);
        s.z = fmaf(decay, s.z, xv * Bv[2]);
        s.w = fmaf(decay, s.w, xv * Bv[3]);
        *reinterpret_cast<float4 *>(st + (int64_t)p * N) = s;
        float part = Cv[0] * s.x + Cv[1] * s.y + Cv[2] * s.z + Cv[3] * s.w;
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
        if (lane == 0) Elem<TOut>::store(yr + p, part + Dh * xv);
    }
}

template <typename TIn, typename TOut>
cudaError_t launch_t(const SsdUpdArgs &a, cudaStream_t stream) {
    const int64_t blocks = a.batch * a.H;
    if (blocks <= 0) return cudaSuccess;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    ssd_update_kernel<TIn, TOut><<<(unsigned)blocks, kUW * 32, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_ssd_update(const SsdUpdArgs &a, bool in_bf16, bool out_bf16, cudaStream_t stream) {
    if (in_bf16) return out_bf16 ? launch_t<__nv_bfloat16, __nv_bfloat16>(a, stream)
                                 : launch_t<__nv_bfloat16, float>(a, stream);
    return out_bf16 ? launch_t<float, __nv_bfloat16>(a, stream) : launch_t<float, float>(a, stream);
}

}  // namespace ms
