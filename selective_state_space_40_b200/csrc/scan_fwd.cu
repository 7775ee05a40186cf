// scan_fwd.cu -- selective scan forward on sm_100a.
//
// Per (batch b, channel d): Delta_t = softplus(delta_t + bias_d), A_bar =
// exp(Delta_t A[d,n]) ('Mamba (deep learning)' wiki page, state-space
// paragraph), h_t = A_bar h_{t-1} + Delta_t B_t u_t and y_t = C_t . h_t
// ('Mamba-1/2/3 Markdown図解' blog, section 1), plus D u_t inside the silu(z_t)
// gate (blog, section 2: the SSM output is gated by a second branch).
//
// Work decomposition. G consecutive lanes of a warp share one channel; lane g
// owns the 16/G states [16g/G, 16(g+1)/G) of that channel for the whole
// sequence, so the state never leaves registers (blog, section 2: the fused
// scan keeps the state on chip; only last_state is written). A warp holds
// 32/G channels of one batch row; a CTA of 4 warps shares the batch row's B
// and C. Tokens go in tiles of 8G; every tile runs three phases:
//   prologue  lane (c, g) takes the 8-token chunk g of its channel c: loads
//             u, delta, z (16-byte vectors), computes Delta (softplus),
//             Delta*u, D*u and silu(z) once per token; Delta and Delta*u go to
//             shared memory for the channel's G lanes, D*u and silu(z) stay in
//             registers for the epilogue. B and C of the tile are staged once
//             per CTA as fp32 rows [token][state].
//   states    lane (c, g) runs its states over the tile's tokens in order:
//             A_bar by exp2, h = A_bar h + (Delta u) B, readout C.h over its
//             states (packed f32x2 arithmetic). After every R tokens the G
//             partial readouts are summed by a reduce-scatter over the G lanes
//             (xor shuffles), so each lane ends up owning whole sums.
//   epilogue  lane (c, g) gathers the sums of its chunk, adds D*u, multiplies
//             by silu(z) and stores y with 16-byte stores.
// The next tile's global loads are issued before the current tile computes.
// exp(x) = 2^(x log2 e); a fixed, lane-uniform share (poly8 / 8) of the
// (state pair, token) slots uses the FMA-pipe polynomial, the rest the MUFU
// ex2, to balance the two pipes.
//
// Conv front-end (CONV): the block's input path (blog, section 2, block
// diagram) runs a short causal convolution per channel and silu before the
// SSM. With CONV the kernel reads that convolution's input x instead of u and
// forms u_t = silu(bias_d + sum_k w[d,k] x_{t-(W-1)+k}) in the prologue, so u
// never makes an HBM round trip. The 3 tokens before a lane's chunk come from
// the previous lane of the channel by shuffle (lane 0 takes the last lane's
// chunk of the previous tile, kept in registers; before token 0 the given
// history or zeros).

#include "ms_device.cuh"
#include "ms_internal.h"

namespace ms {

namespace {

// Tuning (measured on the 130M-class layer: 2 warps per CTA, the reduction
// pipelined against the next group and a register cap that keeps 6 CTAs per
// SM resident gave 221 us against 238 us for 4-warp CTAs without either;
// the packed Delta*A multiply took another 1 %).
#ifndef MS_SCAN_NW
#define MS_SCAN_NW 2              // warps per CTA
#endif
#ifndef MS_SCAN_MINB
#define MS_SCAN_MINB 6            // resident CTAs per SM the one-chunk kernels are capped for
#endif
#ifndef MS_SCAN_PIPE
#define MS_SCAN_PIPE 1            // 1: reduce a token group while the next group's states run
#endif
#ifndef MS_SCAN_PACKED_DA
#define MS_SCAN_PACKED_DA 1       // 1: Delta*A for a state pair as one packed multiply
#endif

constexpr int kNW = MS_SCAN_NW;
constexpr int kThreads = kNW * 32;
constexpr int kBCRow = 36;        // floats per staged token row: B[0..15], C[16..31], pad

template <int G, int CH>
struct Geom {
    static constexpr int kCW = 32 / G;          // channels per warp
    static constexpr int kTT = 8 * G * CH;      // tokens per tile: CH 8-token chunks per lane
    static constexpr int kStates = 16 / G;      // states per lane
    static constexpr int kPairs = kStates / 2;  // state pairs per lane
    static constexpr int kR = 8;                // tokens per reduction group
    static constexpr int kRow = kTT + 4;        // floats per per-channel smem row (padded)
    static constexpr int kChannels = kNW * kCW; // channels per CTA
    static constexpr int kSlots = kR * kPairs;  // (token, pair) slots per reduction group
};

template <int G, int CH>
struct SmemLayout {
    using Gm = Geom<G, CH>;
    static constexpr int kRows = G > 1 ? Gm::kCW : 1;  // per-channel rows (none needed when G == 1)
    static constexpr int kBCBytes = 2 * Gm::kTT * kBCRow * 4;
    static constexpr int kPairBytes = G > 1 ? kNW * kRows * Gm::kRow * 4 : 0;
    static constexpr int kYBytes = G > 1 ? kNW * kRows * Gm::kRow * 4 : 0;
    static constexpr int kOffDelta = kBCBytes;
    static constexpr int kOffDu = kOffDelta + kPairBytes;
    static constexpr int kOffY = kOffDu + kPairBytes;
    static constexpr int kTotal = kOffY + kYBytes;
};

// 8 consecutive elements of one row, kept in their storage format.
template <typename TIn>
struct Chunk8 {
    static constexpr int kWords = 8 * (int)sizeof(TIn) / 4;
    uint32_t w[kWords];

    __device__ __forceinline__ float get(int j) const {
        if constexpr (sizeof(TIn) == 4) return __uint_as_float(w[j]);
        else return (j & 1) ? bf16_hi(w[j >> 1]) : bf16_lo(w[j >> 1]);
    }
    __device__ __forceinline__ void clear() {
#pragma unroll
        for (int i = 0; i < kWords; ++i) w[i] = 0u;
    }
    // Tokens [t, t+8) of `row`; positions at or past L read as 0.
    __device__ __forceinline__ void load(const TIn *row, int64_t t, int64_t L, bool vec) {
        if (vec && t + 8 <= L) {
            const uint4 *p = reinterpret_cast<const uint4 *>(row + t);
#pragma unroll
            for (int i = 0; i < kWords / 4; ++i) {
                const uint4 v = __ldcs(p + i);
                w[4 * i + 0] = v.x;
                w[4 * i + 1] = v.y;
                w[4 * i + 2] = v.z;
                w[4 * i + 3] = v.w;
            }
        } else {
            clear();
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                if (t + j < L) {
                    if constexpr (sizeof(TIn) == 4) {
                        w[j] = __float_as_uint(__ldcs(reinterpret_cast<const float *>(row) + t + j));
                    } else {
                        const uint32_t bits = __ldcs(reinterpret_cast<const unsigned short *>(row) + t + j);
                        w[j >> 1] |= (j & 1) ? (bits << 16) : bits;
                    }
                }
            }
        }
    }
};

// One staged row of B (or C) for one token: 16 states, storage format.
template <typename TIn>
struct Row16 {
    static constexpr int kWords = 16 * (int)sizeof(TIn) / 4;
    uint32_t w[kWords];
    __device__ __forceinline__ float get(int n) const {
        if constexpr (sizeof(TIn) == 4) return __uint_as_float(w[n]);
        else return (n & 1) ? bf16_hi(w[n >> 1]) : bf16_lo(w[n >> 1]);
    }
    // Element n at base + n*stride (n < N, t < L), else 0.
    __device__ __forceinline__ void load(const TIn *base, int64_t stride, int N, bool ok) {
#pragma unroll
        for (int i = 0; i < kWords; ++i) w[i] = 0u;
        if (!ok) return;
#pragma unroll
        for (int n = 0; n < 16; ++n) {
            if (n < N) {
                if constexpr (sizeof(TIn) == 4) {
                    w[n] = __float_as_uint(__ldg(reinterpret_cast<const float *>(base) + n * stride));
                } else {
                    const uint32_t bits = __ldg(reinterpret_cast<const unsigned short *>(base) + n * stride);
                    w[n >> 1] |= (n & 1) ? (bits << 16) : bits;
                }
            }
        }
    }
};

template <typename TOut>
__device__ __forceinline__ void store8(TOut *row, int64_t t, int64_t L, bool vec, const float (&v)[8]) {
    if (vec && t + 8 <= L) {
        if constexpr (sizeof(TOut) == 4) {
            float4 *p = reinterpret_cast<float4 *>(row + t);
            __stcs(p, make_float4(v[0], v[1], v[2], v[3]));
            __stcs(p + 1, make_float4(v[4], v[5], v[6], v[7]));
        } else {
            uint32_t w[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                __nv_bfloat162 h2 = __floats2bfloat162_rn(v[2 * k], v[2 * k + 1]);
                w[k] = *reinterpret_cast<uint32_t *>(&h2);
            }
            __stcs(reinterpret_cast<uint4 *>(row + t), make_uint4(w[0], w[1], w[2], w[3]));
        }
    } else {
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if (t + j < L) Elem<TOut>::store(row + t + j, v[j]);
    }
}

// Reduce-scatter of v[0..G) over the G lanes of a group (lane bits below G):
// afterwards lane g holds the sum over the group of element g, in v[0].
template <int G>
__device__ __forceinline__ float reduce_scatter(float (&v)[G], int g) {
#pragma unroll
    for (int half = G / 2; half >= 1; half >>= 1) {
        const bool upper = (g & half) != 0;
#pragma unroll
        for (int i = 0; i < half; ++i) {
            const float send = upper ? v[i] : v[i + half];
            const float keep = upper ? v[i + half] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, half);
        }
    }
    return v[0];
}

// One token of the state phase for a lane owning P state pairs from n0:
// A_bar = 2^(Delta A log2e), h = A_bar h + (Delta u) B, returns C . h over
// the lane's states. `slot0` numbers the (token, pair) slots for the
// MUFU/polynomial split.
template <int P, int POLY8, int SLOTS>
__device__ __forceinline__ float state_token(const float *bcr, int n0, float dl, float du, const f2 (&A2)[P],
                                             f2 (&h)[P], int slot0) {
    f2 Bp[P], Cp[P];
    if constexpr (P >= 2) {
#pragma unroll
        for (int q = 0; q < P / 2; ++q) {
            lds_f2x2(bcr + n0 + 4 * q, Bp[2 * q], Bp[2 * q + 1]);
            lds_f2x2(bcr + 16 + n0 + 4 * q, Cp[2 * q], Cp[2 * q + 1]);
        }
    } else {
        Bp[0] = lds_f2(bcr + n0);
        Cp[0] = lds_f2(bcr + 16 + n0);
    }
    const f2 du2 = f2_splat(du);
#if MS_SCAN_PACKED_DA
    const f2 dl2 = f2_splat(dl);
#endif
    f2 acc = f2_splat(0.0f);
#pragma unroll
    for (int p = 0; p < P; ++p) {
        float xa, xb;
#if MS_SCAN_PACKED_DA
        f2_split(f2_mul(A2[p], dl2), xa, xb);
#else
        f2_split(A2[p], xa, xb);
        xa *= dl;
        xb *= dl;
#endif
        const bool poly = (slot0 + p) * 8 < POLY8 * SLOTS;
        const f2 ab = poly ? exp2_pair<true>(f2_make(xa, xb)) : f2_make(exp2_mufu(xa), exp2_mufu(xb));
        h[p] = f2_fma(ab, h[p], f2_mul(du2, Bp[p]));
        acc = (p == 0) ? f2_mul(Cp[p], h[p]) : f2_fma(Cp[p], h[p], acc);
    }
    float lo, hi;
    f2_split(acc, lo, hi);
    return lo + hi;
}

template <typename TIn, typename TOut, int G, int CH, int POLY8, bool CONV, bool CKPT>
__global__ void __launch_bounds__(kThreads, CH == 1 ? MS_SCAN_MINB : 1)
scan_fwd_kernel(const ScanArgs a) {
    static_assert(!CONV || CH == 1, "the conv front-end runs with one chunk per lane");
    static_assert(kCkptTokens % Geom<G, CH>::kTT == 0, "saved states fall on tile starts");
    using Gm = Geom<G, CH>;
    constexpr int TT = Gm::kTT;
    constexpr int S = Gm::kStates;
    constexpr int P = Gm::kPairs;
    constexpr int R = Gm::kR;
    using Sm = SmemLayout<G, CH>;
    constexpr int ROWS = Sm::kRows;

    // Dynamic shared memory: B/C tiles (double buffered, shared by the CTA),
    // then per warp: Delta, Delta*u and the reduced readout per token.
    extern __shared__ __align__(16) unsigned char smem_raw[];
    auto sBC = reinterpret_cast<float (*)[TT][kBCRow]>(smem_raw);
    auto sDelta = reinterpret_cast<float (*)[ROWS][Gm::kRow]>(smem_raw + Sm::kOffDelta);
    auto sDu = reinterpret_cast<float (*)[ROWS][Gm::kRow]>(smem_raw + Sm::kOffDu);
    auto sY = reinterpret_cast<float (*)[ROWS][Gm::kRow]>(smem_raw + Sm::kOffY);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int c = lane / G;   // channel within the warp
    const int g = lane % G;   // state group / prologue chunk group

    const int64_t dblocks = (a.dim + Gm::kChannels - 1) / Gm::kChannels;
    const int64_t b = blockIdx.x / dblocks;
    const int64_t d = (blockIdx.x % dblocks) * Gm::kChannels + warp * Gm::kCW + c;
    const bool active = d < a.dim;
    const int64_t dd = active ? d : 0;
    const int N = a.N;
    const int64_t L = a.L;
    const int n0 = g * S;  // first state of this lane

    // Per-lane state, transition scaled by log2 e.
    f2 A2[P], h[P];
#pragma unroll
    for (int p = 0; p < P; ++p) {
        const int na = n0 + 2 * p, nb = na + 1;
        const float aa = na < N ? __ldg(a.A + dd * N + na) * kLog2e : 0.0f;
        const float ab = nb < N ? __ldg(a.A + dd * N + nb) * kLog2e : 0.0f;
        A2[p] = f2_make(aa, ab);
        float ha = 0.0f, hb = 0.0f;
        if (a.h0 != nullptr && active) {
            const float *hs = a.h0 + (b * a.dim + d) * N;
            if (na < N) ha = __ldg(hs + na);
            if (nb < N) hb = __ldg(hs + nb);
        }
        h[p] = f2_make(ha, hb);
    }
    const float Dd = a.D ? __ldg(a.D + dd) : 0.0f;
    const float bias = a.bias ? __ldg(a.bias + dd) : 0.0f;
    const bool has_z = a.z != nullptr;
    const bool sp = a.softplus != 0;

    // Conv taps right-aligned in cw (cw[3] weights the current token) and the
    // 3 inputs before this lane's next chunk (only the channel's last lane's
    // copy is read: it feeds lane 0 of the next tile).
    float cw[4] = {0.0f, 0.0f, 0.0f, 0.0f}, cb = 0.0f;
    float keep[3] = {0.0f, 0.0f, 0.0f};
    if constexpr (CONV) {
        const int W = a.conv_width;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int src = k - (4 - W);
            if (src >= 0) cw[k] = __ldg(a.conv_w + dd * W + src);
        }
        cb = a.conv_b ? __ldg(a.conv_b + dd) : 0.0f;
        if (a.conv_x0 != nullptr && active) {
            const TIn *x0 = static_cast<const TIn *>(a.conv_x0) + (b * a.dim + d) * (W - 1);
#pragma unroll
            for (int j = 1; j <= 3; ++j)
                if (W - 1 - j >= 0) keep[3 - j] = Elem<TIn>::load(x0 + (W - 1 - j));
        }
    }

    const TIn *u_row = static_cast<const TIn *>(a.u) + b * a.u_sb + dd * a.u_sd;
    const TIn *d_row = static_cast<const TIn *>(a.delta) + b * a.dl_sb + dd * a.dl_sd;
    const TIn *z_row = has_z ? static_cast<const TIn *>(a.z) + b * a.z_sb + dd * a.z_sd : u_row;
    TOut *y_row = static_cast<TOut *>(a.y) + b * a.y_sb + dd * a.y_sd;
    TIn *uo_row = CONV && a.u_out ? static_cast<TIn *>(a.u_out) + b * a.uo_sb + dd * a.uo_sd : nullptr;
    const TIn *B_b = static_cast<const TIn *>(a.B) + b * a.B_sb;
    const TIn *C_b = static_cast<const TIn *>(a.C) + b * a.C_sb;
    const bool vin = a.vec_in != 0;
    const bool vout = a.vec_out != 0;

    // B/C staging: staged row r < TT is B of token r, TT <= r < 2TT is C of
    // token r - TT; thread i stages rows i, i + kThreads, ...
    constexpr int kBCPer = (2 * TT + kThreads - 1) / kThreads;

    const int64_t ntiles = (L + TT - 1) / TT;

    // Lane (c, g) owns the prologue/epilogue chunks g*CH .. g*CH+CH-1 of its
    // channel in every tile (8*CH consecutive tokens).
    Chunk8<TIn> nu[CH], nd[CH], nz[CH];
    Row16<TIn> nbc[kBCPer];
    auto prefetch = [&](int64_t t0) {
#pragma unroll
        for (int i = 0; i < CH; ++i) {
            const int64_t ts = t0 + 8 * (g * CH + i);
            if (active) {
                nu[i].load(u_row, ts, L, vin);
                nd[i].load(d_row, ts, L, vin);
                if (has_z) nz[i].load(z_row, ts, L, vin);
                else nz[i].clear();
            } else {
                nu[i].clear();
                nd[i].clear();
                nz[i].clear();
            }
        }
#pragma unroll
        for (int r = 0; r < kBCPer; ++r) {
            const int row = threadIdx.x + r * kThreads;
            const bool isC = row >= TT;
            const int64_t tb = t0 + (row % TT);
            nbc[r].load((isC ? C_b : B_b) + tb, isC ? a.C_sn : a.B_sn, N, row < 2 * TT && tb < L);
        }
    };

    if (ntiles > 0) prefetch(0);

    const int64_t nck = (L + kCkptTokens - 1) / kCkptTokens;
    float dsum_acc = 0.0f;  // this lane's tokens' Delta (saved-state kernels)
    for (int64_t k = 0; k < ntiles; ++k) {
        const int64_t t0 = k * TT;
        const int buf = (int)(k & 1);
        if (CKPT && a.ckpt != nullptr && active && t0 % kCkptTokens == 0) {
            // Training: the state before this block, for the backward's recompute.
            float *cs = a.ckpt + ((b * a.dim + d) * nck + t0 / kCkptTokens) * N;
#pragma unroll
            for (int p = 0; p < P; ++p) {
                float ha, hb;
                f2_split(h[p], ha, hb);
                const int na = n0 + 2 * p;
                if (na < N) cs[na] = ha;
                if (na + 1 < N) cs[na + 1] = hb;
            }
        }

        // ---- prologue: per-token quantities of this lane's chunks.
        float dl[CH][8], dlu[CH][8], dug[CH][8], gate[CH][8];
#pragma unroll
        for (int i = 0; i < CH; ++i) {
            const int64_t ts = t0 + 8 * (g * CH + i);
            float uv[8];
            if constexpr (CONV) {
                // Halo x_{ts-3..ts-1}: the previous lane's chunk tail, or for
                // lane 0 the last lane's tail from the previous tile.
                const float t5 = nu[i].get(5), t6 = nu[i].get(6), t7 = nu[i].get(7);
                const bool last_lane = g == G - 1;
                const int src = g == 0 ? lane + G - 1 : lane - 1;
                const float h0 = __shfl_sync(0xffffffffu, last_lane ? keep[0] : t5, src);
                const float h1 = __shfl_sync(0xffffffffu, last_lane ? keep[1] : t6, src);
                const float h2 = __shfl_sync(0xffffffffu, last_lane ? keep[2] : t7, src);
                keep[0] = t5;
                keep[1] = t6;
                keep[2] = t7;
                float xs[11];
                xs[0] = h0;
                xs[1] = h1;
                xs[2] = h2;
#pragma unroll
                for (int j = 0; j < 8; ++j) xs[3 + j] = nu[i].get(j);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    float v = fmaf(cw[0], xs[j], cb);
                    v = fmaf(cw[1], xs[j + 1], v);
                    v = fmaf(cw[2], xs[j + 2], v);
                    v = fmaf(cw[3], xs[j + 3], v);
                    uv[j] = a.conv_silu ? silu_f(v) : v;
                }
                if (uo_row != nullptr && active) store8<TIn>(uo_row, ts, L, a.vec_uout != 0, uv);
            } else {
#pragma unroll
                for (int j = 0; j < 8; ++j) uv[j] = nu[i].get(j);
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float uj = uv[j];
                const float v = nd[i].get(j) + bias;
                const float step = sp ? softplus_f(v) : v;
                dl[i][j] = (ts + j < L) ? step : 0.0f;  // past the end: the state is left alone
                if constexpr (CKPT) dsum_acc += dl[i][j];
                dlu[i][j] = dl[i][j] * uj;
                gate[i][j] = has_z ? silu_f(nz[i].get(j)) : 1.0f;
                dug[i][j] = Dd * uj * gate[i][j];
            }
            if constexpr (G > 1) {
                float4 *pd = reinterpret_cast<float4 *>(&sDelta[warp][c][8 * (g * CH + i)]);
                float4 *pu = reinterpret_cast<float4 *>(&sDu[warp][c][8 * (g * CH + i)]);
                pd[0] = make_float4(dl[i][0], dl[i][1], dl[i][2], dl[i][3]);
                pd[1] = make_float4(dl[i][4], dl[i][5], dl[i][6], dl[i][7]);
                pu[0] = make_float4(dlu[i][0], dlu[i][1], dlu[i][2], dlu[i][3]);
                pu[1] = make_float4(dlu[i][4], dlu[i][5], dlu[i][6], dlu[i][7]);
            }
        }
#pragma unroll
        for (int r = 0; r < kBCPer; ++r) {
            const int rr = threadIdx.x + r * kThreads;
            if (rr < 2 * TT && MS_CHECK(a.status, buf < 2 && rr % TT < TT)) {
                float4 *row = reinterpret_cast<float4 *>(&sBC[buf][rr % TT][rr >= TT ? 16 : 0]);
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    row[q] = make_float4(nbc[r].get(4 * q), nbc[r].get(4 * q + 1), nbc[r].get(4 * q + 2),
                                         nbc[r].get(4 * q + 3));
            }
        }
        // The next tile's loads stay in flight while this tile's states run.
        if (k + 1 < ntiles) prefetch(t0 + TT);
        __syncthreads();

        if constexpr (G == 1) {
            // ---- one lane per channel: states, readout and gate in registers.
#pragma unroll
            for (int i = 0; i < CH; ++i) {
                float yo[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float *bcr = sBC[buf][8 * i + j];
                    const float yv = state_token<P, POLY8, Gm::kSlots>(bcr, 0, dl[i][j], dlu[i][j], A2, h,
                                                                        j * P);
                    yo[j] = fmaf(yv, gate[i][j], dug[i][j]);
                }
                if (active && (!CKPT || a.y != nullptr)) store8<TOut>(y_row, t0 + 8 * i, L, vout, yo);
            }
        } else {
            __syncwarp();
            // ---- states: tokens of the tile in order.
            const float *dl_row = reinterpret_cast<const float *>(&sDelta[warp][c][0]);
            const float *du_row = reinterpret_cast<const float *>(&sDu[warp][c][0]);
            // G partial readouts per token -> whole sums owned by one lane each.
            auto reduce_group = [&](const float (&part)[R], int tr) {
#pragma unroll
                for (int blk = 0; blk < R / G; ++blk) {
                    float v[G];
#pragma unroll
                    for (int q = 0; q < G; ++q) v[q] = part[blk * G + q];
                    sY[warp][c][tr + blk * G + g] = reduce_scatter<G>(v, g);
                }
            };
            auto state_group = [&](float (&part)[R], int tr) {
                float dlv[R], duv[R];
#pragma unroll
                for (int q = 0; q < R / 4; ++q) {
                    const float4 x = *reinterpret_cast<const float4 *>(dl_row + tr + 4 * q);
                    const float4 y = *reinterpret_cast<const float4 *>(du_row + tr + 4 * q);
                    dlv[4 * q] = x.x; dlv[4 * q + 1] = x.y; dlv[4 * q + 2] = x.z; dlv[4 * q + 3] = x.w;
                    duv[4 * q] = y.x; duv[4 * q + 1] = y.y; duv[4 * q + 2] = y.z; duv[4 * q + 3] = y.w;
                }
#pragma unroll
                for (int j = 0; j < R; ++j)
                    part[j] = state_token<P, POLY8, Gm::kSlots>(sBC[buf][tr + j], n0, dlv[j], duv[j], A2, h,
                                                                 j * P);
            };
#if MS_SCAN_PIPE
            // The reduction of group k-1 sits in the same block as the state
            // work of group k, so its shuffles fill the state chain's stalls.
            float prev[R];
            state_group(prev, 0);
#pragma unroll
            for (int tr = R; tr < TT; tr += R) {
                float part[R];
                state_group(part, tr);
                reduce_group(prev, tr - R);
#pragma unroll
                for (int j = 0; j < R; ++j) prev[j] = part[j];
            }
            reduce_group(prev, TT - R);
#else
#pragma unroll 2
            for (int tr = 0; tr < TT; tr += R) {
                float part[R];
                state_group(part, tr);
                reduce_group(part, tr);
            }
#endif
            __syncwarp();

            // ---- epilogue: this lane's chunks.
#pragma unroll
            for (int i = 0; i < CH; ++i) {
                const int off = 8 * (g * CH + i);
                if (!MS_CHECK(a.status, off + 8 <= Gm::kRow && c < ROWS && warp < kNW)) continue;
                const float4 y0 = *reinterpret_cast<const float4 *>(&sY[warp][c][off]);
                const float4 y1 = *reinterpret_cast<const float4 *>(&sY[warp][c][off + 4]);
                const float ys[8] = {y0.x, y0.y, y0.z, y0.w, y1.x, y1.y, y1.z, y1.w};
                float yo[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) yo[j] = fmaf(ys[j], gate[i][j], dug[i][j]);
                if (active && (!CKPT || a.y != nullptr)) store8<TOut>(y_row, t0 + off, L, vout, yo);
            }
            __syncwarp();
        }
    }

    if constexpr (CKPT) {
        if (a.dsum != nullptr) {
            // the channel's G lanes hold disjoint token chunks: sum them
#pragma unroll
            for (int off = 1; off < G; off <<= 1) dsum_acc += __shfl_xor_sync(0xffffffffu, dsum_acc, off);
            if (active && g == 0) a.dsum[b * a.dim + d] = dsum_acc;
        }
    }
    if (active && a.last != nullptr) {
        float *ls = a.last + (b * a.dim + d) * N;
#pragma unroll
        for (int p = 0; p < P; ++p) {
            float ha, hb;
            f2_split(h[p], ha, hb);
            const int na = n0 + 2 * p;
            if (na < N) ls[na] = ha;
            if (na + 1 < N) ls[na + 1] = hb;
        }
    }
}

template <typename TIn, typename TOut, int G, int CH, int POLY8, bool CONV = false, bool CKPT = false>
cudaError_t launch_one(const ScanArgs &a, cudaStream_t stream) {
    using Gm = Geom<G, CH>;
    using Sm = SmemLayout<G, CH>;
    const int64_t dblocks = (a.dim + Gm::kChannels - 1) / Gm::kChannels;
    const int64_t blocks = dblocks * a.batch;
    if (blocks <= 0) return cudaSuccess;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    // Opt in to more than 48 KB of dynamic shared memory once per device and
    // instantiation (setting it twice from two host threads is harmless).
    static SmemOptIn opt_in;
    cudaError_t e = opt_in.ensure(reinterpret_cast<const void *>(scan_fwd_kernel<TIn, TOut, G, CH, POLY8, CONV, CKPT>), Sm::kTotal);
    if (e != cudaSuccess) return e;
    scan_fwd_kernel<TIn, TOut, G, CH, POLY8, CONV, CKPT><<<(unsigned)blocks, kThreads, Sm::kTotal, stream>>>(a);
    return cudaGetLastError();
}

template <typename TIn, typename TOut, int G, int CH>
cudaError_t launch_poly(const ScanArgs &a, int poly8, cudaStream_t stream) {
    switch (poly8) {
        case 0: return launch_one<TIn, TOut, G, CH, 0>(a, stream);
        case 2: return launch_one<TIn, TOut, G, CH, 2>(a, stream);
        case 4: return launch_one<TIn, TOut, G, CH, 4>(a, stream);
        default: return launch_one<TIn, TOut, G, CH, 8>(a, stream);
    }
}

template <typename TIn, typename TOut>
cudaError_t launch_types(const ScanArgs &a, const ScanPlan &pl, cudaStream_t stream) {
    const int ch = pl.chunks_per_lane;
    switch (pl.lanes_per_channel) {
        case 1: return ch == 1 ? launch_poly<TIn, TOut, 1, 1>(a, pl.poly8, stream)
                               : launch_poly<TIn, TOut, 1, 2>(a, pl.poly8, stream);
        case 2: return ch == 1 ? launch_poly<TIn, TOut, 2, 1>(a, pl.poly8, stream)
                               : launch_poly<TIn, TOut, 2, 2>(a, pl.poly8, stream);
        case 4: return ch == 1 ? launch_poly<TIn, TOut, 4, 1>(a, pl.poly8, stream)
                               : launch_poly<TIn, TOut, 4, 2>(a, pl.poly8, stream);
        default: return launch_poly<TIn, TOut, 8, 1>(a, pl.poly8, stream);
    }
}

// Conv front-end: one chunk per lane, exponentials all on MUFU or all on the
// polynomial.
template <typename TIn, typename TOut>
cudaError_t launch_types_conv(const ScanArgs &a, const ScanPlan &pl, cudaStream_t stream) {
    const bool poly = pl.poly8 != 0;
    switch (pl.lanes_per_channel) {
        case 1: return poly ? launch_one<TIn, TOut, 1, 1, 8, true>(a, stream)
                            : launch_one<TIn, TOut, 1, 1, 0, true>(a, stream);
        case 2: return poly ? launch_one<TIn, TOut, 2, 1, 8, true>(a, stream)
                            : launch_one<TIn, TOut, 2, 1, 0, true>(a, stream);
        case 4: return poly ? launch_one<TIn, TOut, 4, 1, 8, true>(a, stream)
                            : launch_one<TIn, TOut, 4, 1, 0, true>(a, stream);
        default: return poly ? launch_one<TIn, TOut, 8, 1, 8, true>(a, stream)
                             : launch_one<TIn, TOut, 8, 1, 0, true>(a, stream);
    }
}

// Training forward (saved states, y optional): one chunk per lane,
// exponentials all on MUFU or all on the polynomial (the automatic plans).
template <typename TIn, typename TOut>
cudaError_t launch_types_ckpt(const ScanArgs &a, const ScanPlan &pl, cudaStream_t stream) {
    const bool poly = pl.poly8 != 0;
    switch (pl.lanes_per_channel) {
        case 1: return poly ? launch_one<TIn, TOut, 1, 1, 8, false, true>(a, stream)
                            : launch_one<TIn, TOut, 1, 1, 0, false, true>(a, stream);
        case 2: return poly ? launch_one<TIn, TOut, 2, 1, 8, false, true>(a, stream)
                            : launch_one<TIn, TOut, 2, 1, 0, false, true>(a, stream);
        case 4: return poly ? launch_one<TIn, TOut, 4, 1, 8, false, true>(a, stream)
                            : launch_one<TIn, TOut, 4, 1, 0, false, true>(a, stream);
        default: return poly ? launch_one<TIn, TOut, 8, 1, 8, false, true>(a, stream)
                             : launch_one<TIn, TOut, 8, 1, 0, false, true>(a, stream);
    }
}

}  // namespace

cudaError_t launch_scan_fwd(const ScanArgs &a, const ScanPlan &plan, bool in_bf16, bool out_bf16,
                            cudaStream_t stream) {
    if (plan.engine == 1) {
        if (!scan_tmem_applies(a, in_bf16, out_bf16 ? 2 : 4)) return cudaErrorInvalidValue;
        int dev = 0, sms = 148;
        if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        return launch_scan_fwd_tmem(a, plan, in_bf16, out_bf16, sms > 0 ? sms : 148, stream);
    }
    if (a.ckpt != nullptr || a.dsum != nullptr) {
        if (plan.chunks_per_lane != 1 || (plan.poly8 != 0 && plan.poly8 != 8)) return cudaErrorInvalidValue;
        if (in_bf16) {
            return out_bf16 ? launch_types_ckpt<__nv_bfloat16, __nv_bfloat16>(a, plan, stream)
                            : launch_types_ckpt<__nv_bfloat16, float>(a, plan, stream);
        }
        return out_bf16 ? launch_types_ckpt<float, __nv_bfloat16>(a, plan, stream)
                        : launch_types_ckpt<float, float>(a, plan, stream);
    }
    if (a.conv_w != nullptr) {
        if (in_bf16) {
            return out_bf16 ? launch_types_conv<__nv_bfloat16, __nv_bfloat16>(a, plan, stream)
                            : launch_types_conv<__nv_bfloat16, float>(a, plan, stream);
        }
        return out_bf16 ? launch_types_conv<float, __nv_bfloat16>(a, plan, stream)
                        : launch_types_conv<float, float>(a, plan, stream);
    }
    if (in_bf16) {
        return out_bf16 ? launch_types<__nv_bfloat16, __nv_bfloat16>(a, plan, stream)
                        : launch_types<__nv_bfloat16, float>(a, plan, stream);
    }
    return out_bf16 ? launch_types<float, __nv_bfloat16>(a, plan, stream)
                    : launch_types<float, float>(a, plan, stream);
}

namespace {

__global__ void carry_combine_kernel(const float *E, const float *dsum, const float *A, const float *h0, float *Sin,
                                     int64_t dim, int N, int64_t S) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // (d, n)
    const int64_t cn = dim * N;
    if (i >= cn) return;
    const int64_t d = i / N;
    const float a = A[i];
    float st = h0 ? h0[i] : 0.0f;
    Sin[i] = st;
    for (int64_t k = 0; k + 1 < S; ++k) {
        st = fmaf(expf(a * dsum[k * dim + d]), st, E[k * cn + i]);
        Sin[(k + 1) * cn + i] = st;
    }
}

}  // namespace

cudaError_t launch_carry_combine(const float *E, const float *dsum, const float *A, const float *h0, float *Sin,
                                 int64_t dim, int N, int64_t S, cudaStream_t stream) {
    const int64_t cn = dim * N;
    if (cn <= 0) return cudaSuccess;
    const int64_t blocks = (cn + 255) / 256;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    carry_combine_kernel<<<(unsigned)blocks, 256, 0, stream>>>(E, dsum, A, h0, Sin, dim, N, S);
    return cudaGetLastError();
}

ScanPlan plan_scan(const ScanArgs &a, bool in_bf16, int num_sms) {
    ScanPlan pl{};
    const int64_t channels = a.batch * a.dim;
    const int64_t want_warps = (int64_t)num_sms * 4 * 2;
    pl.lanes_per_channel = (channels * 4 / 32 >= want_warps) ? 4 : 8;
    pl.chunks_per_lane = 1;
    pl.poly8 = in_bf16 ? 0 : 8;
    pl.engine = 0;
    return pl;
}

}  // namespace ms
