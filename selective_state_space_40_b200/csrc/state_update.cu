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
// readout is summed over the four lanes with two xor-shuffles. Every
// exponential uses the FMA-pipe polynomial (unbiased near 1, and the pipes are
// idle here anyway).

#include "ms_device.cuh"
#include "ms_internal.h"

namespace ms {

namespace {

constexpr int kThreads = 256;

template <typename TIn, typename TOut>
__global__ void __launch_bounds__(kThreads)
state_update_kernel(const UpdateArgs a) {
    const int64_t gtid = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    const int64_t ch = gtid >> 2;  // flattened (b, d)
    const int q = (int)(gtid & 3);
    const int64_t nch = a.batch * a.dim;
    const bool active = ch < nch;
    const int64_t cc = active ? ch : 0;
    const int64_t b = cc / a.dim, d = cc % a.dim;
    const int N = a.N;
    const int n0 = 4 * q;
    const bool mine = active && n0 < N;  // this lane owns at least one real state

    float *st = a.state + b * a.st_sb + d * a.st_sd + n0;
    float h[4] = {0.f, 0.f, 0.f, 0.f};
    float A2[4], Bv[4], Cv[4];
    const TIn *Bb = static_cast<const TIn *>(a.B) + b * a.B_sb;
    const TIn *Cb = static_cast<const TIn *>(a.C) + b * a.C_sb;
    if (mine && a.vec_state && n0 + 4 <= N) {
        const float4 v = __ldcs(reinterpret_cast<const float4 *>(st));
        h[0] = v.x; h[1] = v.y; h[2] = v.z; h[3] = v.w;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const bool real = mine && n0 + i < N;
        if (real && !(a.vec_state && n0 + 4 <= N)) h[i] = __ldcs(st + i);
        A2[i] = real ? __ldg(a.A + d * N + n0 + i) * kLog2e : 0.0f;
        Bv[i] = real ? Elem<TIn>::load(Bb + n0 + i) : 0.0f;
        Cv[i] = real ? Elem<TIn>::load(Cb + n0 + i) : 0.0f;
    }
    float x = 0.f, raw = 0.f, zv = 0.f;
    if (active) {
        x = Elem<TIn>::load(static_cast<const TIn *>(a.x) + b * a.x_sb + d);
        raw = Elem<TIn>::load(static_cast<const TIn *>(a.delta) + b * a.dl_sb + d);
        if (a.z) zv = Elem<TIn>::load(static_cast<const TIn *>(a.z) + b * a.z_sb + d);
    }
    const float bias = (a.bias && active) ? __ldg(a.bias + d) : 0.0f;
    const float Dd = (a.D && active) ? __ldg(a.D + d) : 0.0f;
    const float v = raw + bias;
    const float dt = a.softplus ? softplus_f(v) : v;
    const float dx = dt * x;

    float acc = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float abar = exp2_poly(dt * A2[i]);
        h[i] = fmaf(abar, h[i], dx * Bv[i]);
        acc = fmaf(Cv[i], h[i], acc);
    }
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    acc += __shfl_xor_sync(0xffffffffu, acc, 2);

    if (mine) {
        if (a.vec_state && n0 + 4 <= N) {
            __stcs(reinterpret_cast<float4 *>(st), make_float4(h[0], h[1], h[2], h[3]));
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i)
                if (n0 + i < N) __stcs(st + i, h[i]);
        }
    }
    if (active && q == 0) {
        float yv = acc + Dd * x;
        if (a.z) yv *= silu_f(zv);
        Elem<TOut>::store(static_cast<TOut *>(a.y) + b * a.y_sb + d, yv);
    }
}

template <typename TIn, typename TOut>
cudaError_t launch_t(const UpdateArgs &a, cudaStream_t stream) {
    const int64_t threads = a.batch * a.dim * 4;
    if (threads <= 0) return cudaSuccess;
    const int64_t blocks = (threads + kThreads - 1) / kThreads;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    state_update_kernel<TIn, TOut><<<(unsigned)blocks, kThreads, 0, stream>>>(a);
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
