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
// vector); the readout is summed over the quad with xor-shuffles. The
// exponentials use the MUFU unit: the arithmetic per channel must stay well
// below the time its 128 state bytes take to stream.

#include "ms_device.cuh"
#include "ms_internal.h"

namespace ms {

namespace {

// Threads per block and channels per lane quad (state vectors in flight per
// lane). Compile-time constants; the defaults are the measured best on B200.
#ifndef MS_DECODE_THREADS
#define MS_DECODE_THREADS 256
#endif
#ifndef MS_DECODE_U
#define MS_DECODE_U 1
#endif
constexpr int kThreads = MS_DECODE_THREADS;

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

// grid: x covers the channels of one batch row, y = batch row. Lane i of a
// warp is quad lane q = i % 4 (states 4q..4q+3) of channel slot s = i / 4;
// the warp owns 8U consecutive channels and lane (s, q) serves channels
// s, s + 8, ..., s + 8(U-1) of them, so for each u the warp's 16-byte state
// accesses cover 512 contiguous bytes, and each lane has U vectors in flight.
template <typename TIn, typename TOut, int U>
__global__ void __launch_bounds__(kThreads)
state_update_kernel(const UpdateArgs a) {
    const int64_t b = blockIdx.y;
    const int lane = threadIdx.x & 31;
    const int q = lane & 3;
    const int64_t dwarp = ((int64_t)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5)) * (8 * U);
    const int N = a.N;
    const int n0 = 4 * q;

    float h[U][4], A[U][4], Bv[4], Cv[4];
    float x[U], raw[U], zv[U], bias[U], Dd[U];
    bool act[U];
    int64_t dd[U];
    int nvs[U];
    const int nq = N - n0 < 0 ? 0 : (N - n0 > 4 ? 4 : N - n0);  // states of this quad lane
    // B and C depend only on the batch row: load once.
    load4<TIn>(static_cast<const TIn *>(a.B) + b * a.B_sb + n0, a.vec_bc != 0, nq, Bv);
    load4<TIn>(static_cast<const TIn *>(a.C) + b * a.C_sb + n0, a.vec_bc != 0, nq, Cv);
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int64_t d = dwarp + (lane >> 2) + 8 * u;
        act[u] = d < a.dim;
        dd[u] = act[u] ? d : 0;
        nvs[u] = act[u] ? nq : 0;
        const float *st = a.state + b * a.st_sb + dd[u] * a.st_sd + n0;
        if (a.vec_state && nvs[u] == 4) {
            const float4 t = __ldcs(reinterpret_cast<const float4 *>(st));
            h[u][0] = t.x; h[u][1] = t.y; h[u][2] = t.z; h[u][3] = t.w;
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) h[u][i] = i < nvs[u] ? __ldcs(st + i) : 0.0f;
        }
        x[u] = raw[u] = zv[u] = 0.0f;
        if (act[u]) {
            x[u] = Elem<TIn>::load(static_cast<const TIn *>(a.x) + b * a.x_sb + dd[u]);
            raw[u] = Elem<TIn>::load(static_cast<const TIn *>(a.delta) + b * a.dl_sb + dd[u]);
            if (a.z) zv[u] = Elem<TIn>::load(static_cast<const TIn *>(a.z) + b * a.z_sb + dd[u]);
        }
        load4<float>(a.A + dd[u] * N + n0, a.vec_A != 0, nvs[u], A[u]);
        bias[u] = (a.bias && act[u]) ? __ldg(a.bias + dd[u]) : 0.0f;
        Dd[u] = (a.D && act[u]) ? __ldg(a.D + dd[u]) : 0.0f;
    }

#pragma unroll
    for (int u = 0; u < U; ++u) {
        const float v = raw[u] + bias[u];
        const float dt = a.softplus ? softplus_f(v) : v;
        const float dx = dt * x[u];
        const float dtl = dt * kLog2e;
        float acc = 0.0f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float abar = exp2_mufu(dtl * A[u][i]);
            h[u][i] = fmaf(abar, h[u][i], dx * Bv[i]);
            acc = fmaf(Cv[i], h[u][i], acc);
        }
        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
        acc += __shfl_xor_sync(0xffffffffu, acc, 2);

        float *st = a.state + b * a.st_sb + dd[u] * a.st_sd + n0;
        if (a.vec_state && nvs[u] == 4) {
            __stcs(reinterpret_cast<float4 *>(st), make_float4(h[u][0], h[u][1], h[u][2], h[u][3]));
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i)
                if (i < nvs[u]) __stcs(st + i, h[u][i]);
        }
        if (act[u] && q == 0) {
            float yv = acc + Dd[u] * x[u];
            if (a.z) yv *= silu_f(zv[u]);
            Elem<TOut>::store(static_cast<TOut *>(a.y) + b * a.y_sb + dd[u], yv);
        }
    }
}

template <typename TIn, typename TOut>
cudaError_t launch_t(const UpdateArgs &a, cudaStream_t stream) {
    constexpr int U = MS_DECODE_U;
    if (a.batch <= 0 || a.dim <= 0) return cudaSuccess;
    if (a.batch > 65535) return cudaErrorInvalidConfiguration;
    const int64_t per_block = (int64_t)(kThreads / 32) * 8 * U;  // channels per block
    const int64_t bx = (a.dim + per_block - 1) / per_block;
    state_update_kernel<TIn, TOut, U><<<dim3((unsigned)bx, (unsigned)a.batch), kThreads, 0, stream>>>(a);
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
