// scan_fwd.cu -- selective scan forward on sm_100a.
//
// Per (batch b, channel d): Delta_t = softplus(delta_t + bias_d), A_bar =
// exp(Delta_t A[d,n]) ('Mamba (deep learning)' wiki page, state-space
// paragraph), h_t = A_bar h_{t-1} + Delta_t B_t u_t and y_t = C_t . h_t
// ('Mamba-1/2/3 Markdown図解' blog, section 1), plus D u_t inside the silu(z_t)
// gate (blog, section 2: the SSM output is gated by a second branch).
//
// Work decomposition. A warp owns C_W = 32 / S_W channels of one batch row and
// splits each tile of S_W*T tokens into S_W segments of T tokens: lane
// (segment s, channel c). The state stays in registers for the whole
// sequence and is never written to HBM except as last_state (blog, section 2:
// the fused scan keeps intermediate state on chip). d_state is padded to 16 and
// processed as 8 pairs with packed f32x2 arithmetic.
//   S_W = 1: each lane runs the plain recurrence over its T tokens.
//   S_W > 1: for each state pair a lane first folds its segment from a zero
//     state into (P, H) = (prod A_bar, local end state), keeping A_bar and the
//     input term of its T tokens in registers; a warp-shuffle inclusive scan
//     over the segments with (P1,H1) o (P2,H2) = (P1 P2, P2 H1 + H2) gives each
//     segment its incoming state from the tile carry; the lane then replays its
//     T tokens from that state to produce y. No exponential is computed twice.
// B and C of the tile (shared by every channel of the batch row) are staged
// once per CTA in shared memory as fp32 pairs; the next tile's u/delta/z and
// B/C are prefetched into registers while the current tile computes.
// exp(x) = 2^(x log2 e): state pairs below `poly_pairs` use the FMA-pipe
// polynomial (unbiased, relieves the MUFU pipe), the others ex2.approx.

#include "ms_device.cuh"
#include "ms_internal.h"

namespace ms {

namespace {

constexpr int kPairs = 8;  // d_state padded to 16 = 8 pairs

template <int SW, int T, int NW>
struct Geom {
    static constexpr int kCW = 32 / SW;             // channels per warp
    static constexpr int kTT = SW * T;              // tokens per tile
    static constexpr int kSegStride = T + 2;        // float2 units (padding: no bank conflicts)
    static constexpr int kPairStride = SW * kSegStride;
    static constexpr int kBuf = kPairs * kPairStride;  // float2 per B (or C) buffer
    static constexpr int kChannels = NW * kCW;      // channels per CTA
    static constexpr int kThreads = NW * 32;
    static constexpr int kBcItems = (kPairs * kTT + kThreads - 1) / kThreads;
};

// T consecutive elements of one row, kept in their storage format.
template <typename TIn, int T>
struct Chunk {
    static constexpr int kWords = T * (int)sizeof(TIn) / 4;
    uint32_t w[kWords];

    __device__ __forceinline__ float get(int j) const {
        if constexpr (sizeof(TIn) == 4) {
            return __uint_as_float(w[j]);
        } else {
            return (j & 1) ? bf16_hi(w[j >> 1]) : bf16_lo(w[j >> 1]);
        }
    }

    __device__ __forceinline__ void clear() {
#pragma unroll
        for (int i = 0; i < kWords; ++i) w[i] = 0u;
    }

    // Load tokens [t, t+T) of `row` (t + j >= L reads as 0).
    __device__ __forceinline__ void load(const TIn *row, int64_t t, int64_t L, bool vec) {
        if (vec && t + T <= L) {
            const uint4 *p = reinterpret_cast<const uint4 *>(row + t);
#pragma unroll
            for (int i = 0; i < kWords / 4; ++i) {
                uint4 v = __ldcs(p + i);
                w[4 * i + 0] = v.x;
                w[4 * i + 1] = v.y;
                w[4 * i + 2] = v.z;
                w[4 * i + 3] = v.w;
            }
        } else {
            clear();
#pragma unroll
            for (int j = 0; j < T; ++j) {
                if (t + j < L) {
                    if constexpr (sizeof(TIn) == 4) {
                        w[j] = __float_as_uint(__ldcs(reinterpret_cast<const float *>(row) + t + j));
                    } else {
                        uint32_t bits = __ldcs(reinterpret_cast<const unsigned short *>(row) + t + j);
                        w[j >> 1] |= (j & 1) ? (bits << 16) : bits;
                    }
                }
            }
        }
    }
};

template <typename TOut, int T>
__device__ __forceinline__ void store_y(TOut *row, int64_t t, int64_t L, bool vec, const float (&v)[T]) {
    if (vec && t + T <= L) {
        if constexpr (sizeof(TOut) == 4) {
            float4 *p = reinterpret_cast<float4 *>(row + t);
#pragma unroll
            for (int i = 0; i < T / 4; ++i)
                __stcs(p + i, make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]));
        } else {
            uint4 *p = reinterpret_cast<uint4 *>(row + t);
#pragma unroll
            for (int i = 0; i < T / 8; ++i) {
                uint32_t w[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    __nv_bfloat162 h2 = __floats2bfloat162_rn(v[8 * i + 2 * k], v[8 * i + 2 * k + 1]);
                    w[k] = *reinterpret_cast<uint32_t *>(&h2);
                }
                __stcs(p + i, make_uint4(w[0], w[1], w[2], w[3]));
            }
        }
    } else {
#pragma unroll
        for (int j = 0; j < T; ++j)
            if (t + j < L) Elem<TOut>::store(row + t + j, v[j]);
    }
}

__device__ __forceinline__ f2 shfl_up_f2(f2 v, int delta) {
    return __shfl_up_sync(0xffffffffu, v, delta);
}
__device__ __forceinline__ f2 shfl_idx_f2(f2 v, int src) {
    return __shfl_sync(0xffffffffu, v, src);
}

template <typename TIn, typename TOut, int SW, int T, int NW, int NPOLY>
__global__ void __launch_bounds__(NW * 32)
scan_fwd_kernel(const ScanArgs a) {
    using G = Geom<SW, T, NW>;
    __shared__ __align__(16) float2 sB[2][G::kBuf];
    __shared__ __align__(16) float2 sC[2][G::kBuf];

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int seg = lane / G::kCW;
    const int cw = lane % G::kCW;

    const int64_t dblocks = (a.dim + G::kChannels - 1) / G::kChannels;
    const int64_t b = blockIdx.x / dblocks;
    const int64_t d = (blockIdx.x % dblocks) * G::kChannels + warp * G::kCW + cw;
    const bool active = d < a.dim;
    const int64_t dd = active ? d : 0;
    const int N = a.N;
    const int64_t L = a.L;

    // Per-channel parameters: A (scaled by log2 e) as pairs, D, bias, state.
    f2 A2[kPairs], carry[kPairs];
#pragma unroll
    for (int p = 0; p < kPairs; ++p) {
        const int n0 = 2 * p, n1 = 2 * p + 1;
        const float a0 = n0 < N ? __ldg(a.A + dd * N + n0) * kLog2e : 0.0f;
        const float a1 = n1 < N ? __ldg(a.A + dd * N + n1) * kLog2e : 0.0f;
        A2[p] = f2_make(a0, a1);
        float h0 = 0.0f, h1 = 0.0f;
        if (a.h0 != nullptr && active) {
            const float *hs = a.h0 + (b * a.dim + d) * N;
            if (n0 < N) h0 = __ldg(hs + n0);
            if (n1 < N) h1 = __ldg(hs + n1);
        }
        carry[p] = f2_make(h0, h1);
    }
    const float Dd = a.D ? __ldg(a.D + dd) : 0.0f;
    const float bias = a.bias ? __ldg(a.bias + dd) : 0.0f;
    const bool has_z = a.z != nullptr;
    const bool sp = a.softplus != 0;

    const TIn *u_row = static_cast<const TIn *>(a.u) + b * a.u_sb + dd * a.u_sd;
    const TIn *d_row = static_cast<const TIn *>(a.delta) + b * a.dl_sb + dd * a.dl_sd;
    const TIn *z_row = has_z ? static_cast<const TIn *>(a.z) + b * a.z_sb + dd * a.z_sd : u_row;
    TOut *y_row = static_cast<TOut *>(a.y) + b * a.y_sb + dd * a.y_sd;
    const TIn *B_b = static_cast<const TIn *>(a.B) + b * a.B_sb;
    const TIn *C_b = static_cast<const TIn *>(a.C) + b * a.C_sb;
    const bool vin = a.vec_in != 0;
    const bool vout = a.vec_out != 0;

    const int64_t ntiles = (L + G::kTT - 1) / G::kTT;

    // Register prefetch buffers for the next tile.
    Chunk<TIn, T> nu, nd, nz;
    float bcv[G::kBcItems][4];

    auto load_tokens = [&](int64_t t0) {
        const int64_t ts = t0 + seg * T;
        if (active) {
            nu.load(u_row, ts, L, vin);
            nd.load(d_row, ts, L, vin);
            if (has_z) nz.load(z_row, ts, L, vin);
            else nz.clear();
        } else {
            nu.clear();
            nd.clear();
            nz.clear();
        }
    };
    auto load_bc = [&](int64_t t0) {
#pragma unroll
        for (int i = 0; i < G::kBcItems; ++i) {
            const int e = threadIdx.x + i * G::kThreads;
            const int p = e / G::kTT, tt = e % G::kTT;
            const int64_t t = t0 + tt;
            float v0 = 0.f, v1 = 0.f, v2 = 0.f, v3 = 0.f;
            if (e < kPairs * G::kTT && t < L) {
                const int n0 = 2 * p, n1 = 2 * p + 1;
                if (n0 < N) {
                    v0 = Elem<TIn>::load(B_b + n0 * a.B_sn + t);
                    v2 = Elem<TIn>::load(C_b + n0 * a.C_sn + t);
                }
                if (n1 < N) {
                    v1 = Elem<TIn>::load(B_b + n1 * a.B_sn + t);
                    v3 = Elem<TIn>::load(C_b + n1 * a.C_sn + t);
                }
            }
            bcv[i][0] = v0;
            bcv[i][1] = v1;
            bcv[i][2] = v2;
            bcv[i][3] = v3;
        }
    };
    auto store_bc = [&](int buf) {
#pragma unroll
        for (int i = 0; i < G::kBcItems; ++i) {
            const int e = threadIdx.x + i * G::kThreads;
            if (e < kPairs * G::kTT) {
                const int p = e / G::kTT, tt = e % G::kTT;
                const int idx = p * G::kPairStride + (tt / T) * G::kSegStride + (tt % T);
                sB[buf][idx] = make_float2(bcv[i][0], bcv[i][1]);
                sC[buf][idx] = make_float2(bcv[i][2], bcv[i][3]);
            }
        }
    };

    if (ntiles > 0) {
        load_tokens(0);
        load_bc(0);
        store_bc(0);
    }
    __syncthreads();

    for (int64_t k = 0; k < ntiles; ++k) {
        const int64_t t0 = k * G::kTT;
        const int buf = (int)(k & 1);
        const Chunk<TIn, T> cu = nu, cd = nd, cz = nz;
        if (k + 1 < ntiles) {
            load_tokens(t0 + G::kTT);
            load_bc(t0 + G::kTT);
        }

        // Token prologue: step sizes, input term scale, D skip.
        const int64_t ts = t0 + seg * T;
        float dt[T], du[T];
        f2 y2[T];
        float dsum = 0.0f;
#pragma unroll
        for (int j = 0; j < T; ++j) {
            const float uj = cu.get(j);
            const float v = cd.get(j) + bias;
            const float step = sp ? softplus_f(v) : v;
            dt[j] = (ts + j < L) ? step : 0.0f;  // tokens past the end leave the state alone
            du[j] = dt[j] * uj;
            y2[j] = f2_make(Dd * uj, 0.0f);
            dsum += dt[j];
        }

        const float2 *bB = sB[buf] + seg * G::kSegStride;
        const float2 *bC = sC[buf] + seg * G::kSegStride;

#pragma unroll
        for (int p = 0; p < kPairs; ++p) {
            constexpr bool kDummy = false;
            (void)kDummy;
            const bool poly = p < NPOLY;
            const float4 *Bq = reinterpret_cast<const float4 *>(bB + p * G::kPairStride);
            const float4 *Cq = reinterpret_cast<const float4 *>(bC + p * G::kPairStride);
            if constexpr (SW == 1) {
                f2 h = carry[p];
#pragma unroll
                for (int j2 = 0; j2 < T / 2; ++j2) {
                    const float4 bq = Bq[j2];
                    const float4 cq = Cq[j2];
#pragma unroll
                    for (int s = 0; s < 2; ++s) {
                        const int j = 2 * j2 + s;
                        const f2 x2 = f2_mul(f2_splat(dt[j]), A2[p]);
                        const f2 a2 = poly ? exp2_pair<true>(x2) : exp2_pair<false>(x2);
                        const f2 Bp = s ? f2_make(bq.z, bq.w) : f2_make(bq.x, bq.y);
                        const f2 Cp = s ? f2_make(cq.z, cq.w) : f2_make(cq.x, cq.y);
                        h = f2_fma(a2, h, f2_mul(f2_splat(du[j]), Bp));
                        y2[j] = f2_fma(Cp, h, y2[j]);
                    }
                }
                carry[p] = h;
            } else {
                f2 av[T], wv[T];
                f2 H = f2_splat(0.0f);
#pragma unroll
                for (int j2 = 0; j2 < T / 2; ++j2) {
                    const float4 bq = Bq[j2];
#pragma unroll
                    for (int s = 0; s < 2; ++s) {
                        const int j = 2 * j2 + s;
                        const f2 x2 = f2_mul(f2_splat(dt[j]), A2[p]);
                        av[j] = poly ? exp2_pair<true>(x2) : exp2_pair<false>(x2);
                        const f2 Bp = s ? f2_make(bq.z, bq.w) : f2_make(bq.x, bq.y);
                        wv[j] = f2_mul(f2_splat(du[j]), Bp);
                        H = f2_fma(av[j], H, wv[j]);
                    }
                }
                const f2 xs = f2_mul(f2_splat(dsum), A2[p]);
                f2 P = poly ? exp2_pair<true>(xs) : exp2_pair<false>(xs);
#pragma unroll
                for (int off = 1; off < SW; off <<= 1) {
                    const f2 Pp = shfl_up_f2(P, off * G::kCW);
                    const f2 Hp = shfl_up_f2(H, off * G::kCW);
                    if (seg >= off) {
                        H = f2_fma(P, Hp, H);
                        P = f2_mul(P, Pp);
                    }
                }
                const f2 hout = f2_fma(P, carry[p], H);
                f2 h = shfl_up_f2(hout, G::kCW);
                if (seg == 0) h = carry[p];
                carry[p] = shfl_idx_f2(hout, (SW - 1) * G::kCW + cw);
#pragma unroll
                for (int j2 = 0; j2 < T / 2; ++j2) {
                    const float4 cq = Cq[j2];
#pragma unroll
                    for (int s = 0; s < 2; ++s) {
                        const int j = 2 * j2 + s;
                        const f2 Cp = s ? f2_make(cq.z, cq.w) : f2_make(cq.x, cq.y);
                        h = f2_fma(av[j], h, wv[j]);
                        y2[j] = f2_fma(Cp, h, y2[j]);
                    }
                }
            }
        }

        // Epilogue: readout halves, gate, store.
        float yo[T];
#pragma unroll
        for (int j = 0; j < T; ++j) {
            float lo, hi;
            f2_split(y2[j], lo, hi);
            float yv = lo + hi;
            if (has_z) yv *= silu_f(cz.get(j));
            yo[j] = yv;
        }
        if (active) store_y<TOut, T>(y_row, ts, L, vout, yo);

        if (k + 1 < ntiles) store_bc(buf ^ 1);
        __syncthreads();
    }

    if (active && seg == 0 && a.last != nullptr) {
        float *ls = a.last + (b * a.dim + d) * N;
#pragma unroll
        for (int p = 0; p < kPairs; ++p) {
            float h0, h1;
            f2_split(carry[p], h0, h1);
            if (2 * p < N) ls[2 * p] = h0;
            if (2 * p + 1 < N) ls[2 * p + 1] = h1;
        }
    }
}

template <typename TIn, typename TOut, int SW, int T, int NPOLY>
cudaError_t launch_one(const ScanArgs &a, cudaStream_t stream) {
    constexpr int NW = 4;
    using G = Geom<SW, T, NW>;
    const int64_t dblocks = (a.dim + G::kChannels - 1) / G::kChannels;
    const int64_t blocks = dblocks * a.batch;
    if (blocks <= 0) return cudaSuccess;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    scan_fwd_kernel<TIn, TOut, SW, T, NW, NPOLY><<<(unsigned)blocks, G::kThreads, 0, stream>>>(a);
    return cudaGetLastError();
}

template <typename TIn, typename TOut, int SW, int T>
cudaError_t launch_poly(const ScanArgs &a, int poly_pairs, cudaStream_t stream) {
    switch (poly_pairs) {
        case 0: return launch_one<TIn, TOut, SW, T, 0>(a, stream);
        case 2: return launch_one<TIn, TOut, SW, T, 2>(a, stream);
        case 4: return launch_one<TIn, TOut, SW, T, 4>(a, stream);
        default: return launch_one<TIn, TOut, SW, T, 8>(a, stream);
    }
}

template <typename TIn, typename TOut>
cudaError_t launch_types(const ScanArgs &a, const ScanPlan &pl, cudaStream_t stream) {
    switch (pl.seg_per_warp) {
        case 1: return launch_poly<TIn, TOut, 1, 16>(a, pl.poly_pairs, stream);
        case 2: return launch_poly<TIn, TOut, 2, 8>(a, pl.poly_pairs, stream);
        case 4: return launch_poly<TIn, TOut, 4, 8>(a, pl.poly_pairs, stream);
        default: return launch_poly<TIn, TOut, 8, 8>(a, pl.poly_pairs, stream);
    }
}

}  // namespace

cudaError_t launch_scan_fwd(const ScanArgs &a, const ScanPlan &plan, bool in_bf16, bool out_bf16,
                            cudaStream_t stream) {
    if (in_bf16) {
        return out_bf16 ? launch_types<__nv_bfloat16, __nv_bfloat16>(a, plan, stream)
                        : launch_types<__nv_bfloat16, float>(a, plan, stream);
    }
    return out_bf16 ? launch_types<float, __nv_bfloat16>(a, plan, stream)
                    : launch_types<float, float>(a, plan, stream);
}

ScanPlan plan_scan(const ScanArgs &a, bool in_bf16, int num_sms) {
    ScanPlan pl{};
    pl.warps_per_cta = 4;
    pl.tokens_per_seg = 8;
    // Enough warps to give every SM sub-partition at least two: split time
    // inside the warp until the channel count alone provides them.
    const int64_t channels = a.batch * a.dim;
    const int64_t want_warps = (int64_t)num_sms * 4 * 2;
    int sw = 1;
    while (sw < 8 && channels * sw / 32 < want_warps) sw *= 2;
    pl.seg_per_warp = sw;
    if (sw == 1) pl.tokens_per_seg = 16;
    // fp32 inputs: every exponential on the unbiased polynomial (slow-decay
    // accuracy); bf16 inputs: a share on the FMA pipe to balance the pipes.
    pl.poly_pairs = in_bf16 ? 2 : 8;
    return pl;
}

}  // namespace ms
