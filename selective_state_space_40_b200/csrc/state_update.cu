// state_update.cu -- single-token selective state update (decode) on sm_100a.
//
// Generation takes the recurrence one token at a time from the stored state
// ('Mamba-1/2/3 Markdown図解' blog, section 2: one-token generation is the
// recurrent update of the same model; section 1 for the step itself). Per
// (b, d): h <- exp(Delta A) * h + Delta B x ; y = (C . h + D x) * silu(z),
// with Delta = softplus(delta + bias).
//
// The fp32 state (64 bytes per channel at d_state 16) dominates the traffic:
// it is read and written once per step, so the kernel is an HBM stream. Four
// lanes share a channel, each owning four consecutive states (one 16-byte
// vector), so a warp moves 8 channels x 64 contiguous bytes per access; the
// readout is summed over the four lanes with two xor-shuffles. The
// exponentials use the MUFU unit: the arithmetic per channel must stay well
// below the time its 128 state bytes take to stream.

#include "ms_device.cuh"
#include "ms_internal.h"

namespace ms {

namespace {

constexpr int kThreads = 256;

template <typename TIn>
__device__ __forceinline__ void load4(const TIn *p, bool vec, int valid, float (&v)[4]) {
    if (vec && valid == 4) {
        if constexpr (sizeof(TIn) == 4) {
            const float4 q = __ldg(reinterpret_cast<const float4 *>(p));
            v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
        } else {
            const uint2 q = __ldg(reinterpret_cast<const uint2 *>(p));
            v[0] = bf16_lo(q.x); v[1] = bf16_hi(q.x); v[2] = bf16_lo(q.y); v[3] = bf16_hi(q.y);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = i < valid ? Elem<TIn>::load(p + i) : 0.0f;
    }
}

// grid: x covers the channels of one batch row (4 lanes each), y = batch row
template <typename TIn, typename TOut>
__global__ void __launch_bounds__(kThreads)
state_update_kernel(const UpdateArgs a) {
    const int64_t b = blockIdx.y;
    const int tid = blockIdx.x * kThreads + threadIdx.x;
    const int q = tid & 3;
    const int64_t d = tid >> 2;
    const bool act = d < a.dim;
    const int64_t dd = act ? d : 0;
    const int N = a.N;
    const int n0 = 4 * q;
    const int nv = act ? (N - n0 < 0 ? 0 : (N - n0 > 4 ? 4 : N - n0)) : 0;  // states this lane owns

    float h[4], A[4], Bv[4], Cv[4];
    float *st = a.state + b * a.st_sb + dd * a.st_sd + n0;
    if (a.vec_state && nv == 4) {
        const float4 v = __ldcs(reinterpret_cast<const float4 *>(st));
        h[0] = v.x; h[1] = v.y; h[2] = v.z; h[3] = v.w;
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) h[i] = i < nv ? __ldcs(st + i) : 0.0f;
    }
    float x = 0.f, raw = 0.f, zv = 0.f;
    if (act) {
        x = Elem<TIn>::load(static_cast<const TIn *>(a.x) + b * a.x_sb + dd);
        raw = Elem<TIn>::load(static_cast<const TIn *>(a.delta) + b * a.dl_sb + dd);
        if (a.z) zv = Elem<TIn>::load(static_cast<const TIn *>(a.z) + b * a.z_sb + dd);
    }
    load4<float>(a.A + dd * N + n0, a.vec_A != 0, nv, A);
    load4<TIn>(static_cast<const TIn *>(a.B) + b * a.B_sb + n0, a.vec_bc != 0, nv, Bv);
    load4<TIn>(static_cast<const TIn *>(a.C) + b * a.C_sb + n0, a.vec_bc != 0, nv, Cv);
    const float bias = (a.bias && act) ? __ldg(a.bias + dd) : 0.0f;
    const float Dd = (a.D && act) ? __ldg(a.D + dd) : 0.0f;

    const float v = raw + bias;
    const float dt = a.softplus ? softplus_f(v) : v;
    const float dx = dt * x;
    const float dtl = dt * kLog2e;
    float acc = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float abar = exp2_mufu(dtl * A[i]);
        h[i] = fmaf(abar, h[i], dx * Bv[i]);
        acc = fmaf(Cv[i], h[i], acc);
    }
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    acc += __shfl_xor_sync(0xffffffffu, acc, 2);

    if (a.vec_state && nv == 4) {
        __stcs(reinterpret_cast<float4 *>(st), make_float4(h[0], h[1], h[2], h[3]));
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i)
            if (i < nv) __stcs(st + i, h[i]);
    }
    if (act && q == 0) {
        float yv = acc + Dd * x;
        if (a.z) yv *= silu_f(zv);
        Elem<TOut>::store(static_cast<TOut *>(a.y) + b * a.y_sb + dd, yv);
    }
}

template <typename TIn, typename TOut>
cudaError_t launch_t(const UpdateArgs &a, cudaStream_t stream) {
    if (a.batch <= 0 || a.dim <= 0) return cudaSuccess;
    const int64_t bx = (a.dim * 4 + kThreads - 1) / kThreads;
    if (bx > 0x7fffffffLL / kThreads || a.batch > 65535) return cudaErrorInvalidConfiguration;
    state_update_kernel<TIn, TOut><<<dim3((unsigned)bx, (unsigned)a.batch), kThreads, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_state_update(const UpdateArgs &a, bool in_bf16, bool out_bf16, cudaStream_t stream) {
    if (in_bf16) {
        return out_bf16 ? launch_t<__nv_bfloat16, __nv_bfloat16>(a, stream)
                        : launch_t<__nv_bfloat16, float>(a, stream);
    }
    return out_bf16 ? launch_t<float, __nv_bfloat16>(a, stream) : launch_t<float, float>(a, stream);
}

}  // namespace ms
