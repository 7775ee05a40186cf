// scan_bwd.cu -- gradients of the selective scan on sm_100a.
//
// Reverse mode of the forward recurrence ('Mamba (deep learning)' wiki page,
// state-space paragraph: A_bar = exp(Delta*A); 'Mamba-1/2/3 Markdown図解'
// blog, section 1: h_t = A_bar_t h_{t-1} + B_bar_t x_t, y_t = C_t h_t;
// section 2: the same model is trained through the scan). With q_t the
// pre-gate output and lam the adjoint of h_t, per channel from the last token
// back:
//   dq_t = dout_t silu(z_t), dz_t = dout_t q_t silu'(z_t)
//   lam = C_t dq_t + A_bar_{t+1} lam_{t+1}          (dL/dlast_state at the end)
//   dA += lam h_{t-1} A_bar_t Delta_t,  dDelta_t = sum_n lam (h_{t-1} A_bar_t A + u_t B_t)
//   du_t = D dq_t + sum_n lam Delta_t B_t,  dB_t += lam Delta_t u_t,  dC_t += dq_t h_t
//   ddelta_t = dDelta_t softplus'(delta_t + bias)
//
// The forward saved the state before every 64-token block. This kernel walks
// the blocks from the last: it recomputes the block forward from its saved
// state, keeping the state at every 8-token boundary in shared memory; then
// for each 8-token sub-chunk from the last it recomputes A_bar and h into
// registers and runs the adjoint back over those 8 tokens. Work split as in
// the forward: 4 lanes per channel, 4 states each; a CTA holds 32 channels of
// one batch row. B_t and C_t of the block are staged once per CTA as fp32
// token rows; u and dout of each sub-chunk reach shared memory by
// asynchronous copies issued one sub-chunk ahead. Sums over channels (dB, dC)
// are reduced within the warp by
// reduce-scatter shuffles, across the CTA's warps in shared memory, then
// added to global memory with fp32 atomics (run-to-run order of those adds
// varies, so dB/dC/dA/dD/dbias can differ in the last bits between runs).

#include "ms_device.cuh"
#include "ms_internal.h"

namespace ms {

namespace {

constexpr int kBNW = 4;                  // warps per CTA
constexpr int kBThreads = kBNW * 32;
constexpr int kG = 4;                    // lanes per channel
constexpr int kCW = 32 / kG;             // channels per warp
constexpr int kBCh = kBNW * kCW;         // channels per CTA
constexpr int kBlk = kCkptTokens;        // tokens per saved-state block
constexpr int kSub = 8;                  // tokens per sub-chunk
constexpr int kNSub = kBlk / kSub;
static_assert(kBlk % kSub == 0, "whole sub-chunks per block");
static_assert(2 * kBlk <= kBThreads, "one staging thread per B/C row");
static_assert(kBlk == 16 * kG, "each lane prepares 16 tokens of its channel's block");

struct BwdSmem {
    float bc[kBlk][36];                  // token rows: B[0..15], C[16..31], pad
    float sub[kBNW][kNSub][4][32];       // state at each sub-chunk start [warp][s][state][lane]
    float red[2][kBNW][kSub][32];        // warp sums of dB/dC per token, two sub-chunks in turn
    float tok[4][kBNW][kCW][kBlk + 4];   // per channel and token: Delta, softplus', gate, gate'
    // u and dout of one sub-chunk per channel in their storage format (up
    // to 8 fp32), two steps in turn: filled by asynchronous copies one step
    // ahead of their use
    alignas(16) unsigned char raw_u[2][kBNW][kCW][32];
    alignas(16) unsigned char raw_o[2][kBNW][kCW][32];
};
enum { kTokDelta = 0, kTokSig = 1, kTokGate = 2, kTokGateGrad = 3 };

template <typename T>
__device__ __forceinline__ float ld_elem(const T *p) {
    if constexpr (sizeof(T) == 4) return __ldg(reinterpret_cast<const float *>(p));
    else return bf16_bits_to_f32(__ldg(reinterpret_cast<const unsigned short *>(p)));
}

// 8 tokens [t, t+8) of a row as fp32 (0 past L): one or two 16-byte loads
// when the row allows, else element loads.
template <typename T>
__device__ __forceinline__ void load8(const T *row, int64_t t, int64_t L, bool vec, float (&v)[8]) {
    if (vec && t + 8 <= L) {
        if constexpr (sizeof(T) == 4) {
            const float4 a = __ldg(reinterpret_cast<const float4 *>(row + t));
            const float4 b = __ldg(reinterpret_cast<const float4 *>(row + t) + 1);
            v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
            v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
        } else {
            const uint4 w = __ldg(reinterpret_cast<const uint4 *>(row + t));
            v[0] = bf16_lo(w.x); v[1] = bf16_hi(w.x); v[2] = bf16_lo(w.y); v[3] = bf16_hi(w.y);
            v[4] = bf16_lo(w.z); v[5] = bf16_hi(w.z); v[6] = bf16_lo(w.w); v[7] = bf16_hi(w.w);
        }
    } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = (t + j < L) ? ld_elem(row + t + j) : 0.0f;
    }
}

// 16-byte asynchronous copy global -> shared (cached in L2 only).
__device__ __forceinline__ void cp_async16(void *sdst, const void *gsrc) {
    const unsigned d = static_cast<unsigned>(__cvta_generic_to_shared(sdst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

// Piece `piece` (16 bytes) of tokens [t, t+8) of `row` into dst, which holds
// the 8 elements in their storage format (zero past L): an asynchronous copy
// when the row allows 16-byte access, else element loads.
template <typename T>
__device__ __forceinline__ void stage8(unsigned char *dst, const T *row, int64_t t, int64_t L, bool vec, int piece) {
    constexpr int kPer = 16 / (int)sizeof(T);  // elements per piece
    if (vec && t + 8 <= L) {
        cp_async16(dst + 16 * piece, row + t + kPer * piece);
    } else {
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
            const int e = kPer * piece + j;
            const int64_t tt = t + e;
            if constexpr (sizeof(T) == 4) {
                reinterpret_cast<float *>(dst)[e] = tt < L ? __ldg(reinterpret_cast<const float *>(row) + tt) : 0.0f;
            } else {
                reinterpret_cast<unsigned short *>(dst)[e] =
                    tt < L ? __ldg(reinterpret_cast<const unsigned short *>(row) + tt) : (unsigned short)0;
            }
        }
    }
}
// The 8 staged elements as fp32.
template <typename T>
__device__ __forceinline__ void unstage8(const unsigned char *src, float (&v)[8]) {
    if constexpr (sizeof(T) == 4) {
        const float4 a = reinterpret_cast<const float4 *>(src)[0];
        const float4 b = reinterpret_cast<const float4 *>(src)[1];
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    } else {
        const uint4 w = *reinterpret_cast<const uint4 *>(src);
        v[0] = bf16_lo(w.x); v[1] = bf16_hi(w.x); v[2] = bf16_lo(w.y); v[3] = bf16_hi(w.y);
        v[4] = bf16_lo(w.z); v[5] = bf16_hi(w.z); v[6] = bf16_lo(w.w); v[7] = bf16_hi(w.w);
    }
}

// Reduce-scatter of v[0..8) over the 8 channel lanes of a warp (lane bits 2..4):
// afterwards lane (c, g) holds the sum over channels of v[c].
__device__ __forceinline__ float reduce_scatter_channels(float (&v)[8], int c) {
    const bool u2 = (c & 4) != 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float send = u2 ? v[i] : v[i + 4];
        const float keep = u2 ? v[i + 4] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
    const bool u1 = (c & 2) != 0;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const float send = u1 ? v[i] : v[i + 2];
        const float keep = u1 ? v[i + 2] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
    const bool u0 = (c & 1) != 0;
    const float send = u0 ? v[0] : v[1];
    const float keep = u0 ? v[1] : v[0];
    return keep + __shfl_xor_sync(0xffffffffu, send, 4);
}

// Reduce-scatter of v[0..8) over the 4 lanes of a channel (lane bits 0..1):
// afterwards lane g holds the sums of tokens 2g and 2g+1 in v[0], v[1].
__device__ __forceinline__ void reduce_scatter_lanes(float (&v)[8], int g) {
    const bool u1 = (g & 2) != 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float send = u1 ? v[i] : v[i + 4];
        const float keep = u1 ? v[i + 4] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
    }
    const bool u0 = (g & 1) != 0;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const float send = u0 ? v[i] : v[i + 2];
        const float keep = u0 ? v[i + 2] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 1);
    }
}

// softplus(v) and its derivative, the logistic function, from one e^{-|v|}
// (same series / logarithm split as the forward's softplus).
__device__ __forceinline__ void softplus_and_grad(float v, float &sp, float &sig) {
    const float e = exp2_mufu(-fabsf(v) * kLog2e);
    sp = softplus_e(v, e);
#if MS_FMA_NONLIN
    const float r = rcp_1to2(1.0f + e);
#else
    const float r = rcp_mufu(1.0f + e);
#endif
    sig = v >= 0.0f ? r : e * r;
}
// the logistic function sigma(z)
__device__ __forceinline__ float logistic_f(float z) {
#if MS_FMA_NONLIN
    const float e = exp2_mufu(-fabsf(z) * kLog2e);
    const float r = rcp_1to2(1.0f + e);
    return z >= 0.0f ? r : e * r;
#else
    return rcp_mufu(1.0f + exp2_mufu(-z * kLog2e));
#endif
}

struct F4 { float v[4]; };
__device__ __forceinline__ F4 lds4(const float *p) {
    const float4 x = *reinterpret_cast<const float4 *>(p);
    return F4{{x.x, x.y, x.z, x.w}};
}

template <typename TIn, typename TOut>
__global__ void __launch_bounds__(kBThreads, 3) scan_bwd_kernel(const BwdArgs a) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    BwdSmem &sm = *reinterpret_cast<BwdSmem *>(smem_raw);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = lane / kG, g = lane % kG;
    const int64_t dblocks = (a.dim + kBCh - 1) / kBCh;
    const int64_t b = blockIdx.x / dblocks;
    const int64_t d = (blockIdx.x % dblocks) * kBCh + warp * kCW + c;
    const bool active = d < a.dim;
    const int64_t dd = active ? d : 0;
    const int N = a.N;
    const int64_t L = a.L;
    // debug build: the grid covers exactly batch x ceil(dim / channels per CTA)
    if (!MS_CHECK(a.status, b < a.batch && N <= 16)) return;
    [[maybe_unused]] const int64_t grad_elems = a.batch * a.dim * L;  // each dense gradient [batch, dim, L]
    const int n0 = g * 4;

    // the lane's 4 states as 2 packed pairs (states n0+2p, n0+2p+1)
    f2 A2[2], An[2], carry[2], dAacc[2];
#pragma unroll
    for (int p = 0; p < 2; ++p) {
        float an[2], cr[2];
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const int n = n0 + 2 * p + k;
            an[k] = n < N ? __ldg(a.A + dd * N + n) : 0.0f;
            cr[k] = (a.dlast != nullptr && active && n < N) ? __ldg(a.dlast + (b * a.dim + d) * N + n) : 0.0f;
        }
        An[p] = f2_make(an[0], an[1]);
        A2[p] = f2_make(an[0] * kLog2e, an[1] * kLog2e);
        carry[p] = f2_make(cr[0], cr[1]);
        dAacc[p] = f2_splat(0.0f);
    }
    const float Dd = a.D ? __ldg(a.D + dd) : 0.0f;
    const float bias = a.bias ? __ldg(a.bias + dd) : 0.0f;
    const bool has_z = a.z != nullptr;
    const bool sp = a.softplus != 0;
    const bool vin = a.vec_in != 0, vout = a.vec_out != 0;
    float dDacc = 0.0f, dbacc = 0.0f;

    const TIn *u_row = static_cast<const TIn *>(a.u) + b * a.u_sb + dd * a.u_sd;
    const TIn *d_row = static_cast<const TIn *>(a.delta) + b * a.dl_sb + dd * a.dl_sd;
    const TIn *z_row = has_z ? static_cast<const TIn *>(a.z) + b * a.z_sb + dd * a.z_sd : nullptr;
    const TOut *o_row = static_cast<const TOut *>(a.dout) + b * a.y_sb + dd * a.y_sd;
    const TIn *B_b = static_cast<const TIn *>(a.B) + b * a.B_sb;
    const TIn *C_b = static_cast<const TIn *>(a.C) + b * a.C_sb;
    const int64_t grow = (b * a.dim + dd) * L;  // dense gradient row
    const float *tk_dl = sm.tok[kTokDelta][warp][c];
    const float *tk_sig = sm.tok[kTokSig][warp][c];
    const float *tk_gate = sm.tok[kTokGate][warp][c];
    const float *tk_gp = sm.tok[kTokGateGrad][warp][c];

    // u and dout arrive one step ahead. The steps of block kb are numbered
    // li = 0..15: pass A's sub-chunks 0..7 (u), then pass B's sub-chunks
    // 7..0 (u and dout); step li uses buffer li & 1. The u piece(s) are
    // copied by lanes g < kUPieces, the dout piece(s) by lanes 2, 3.
    constexpr int kUPieces = 8 * (int)sizeof(TIn) / 16;
    constexpr int kOPieces = 8 * (int)sizeof(TOut) / 16;
    auto issue_step = [&](int64_t kb2, int li2) {
        if (kb2 >= 0) {
            const int s2 = li2 < kNSub ? li2 : 2 * kNSub - 1 - li2;
            const int64_t t = kb2 * kBlk + s2 * kSub;
            const int bf = li2 & 1;
            if (g < kUPieces) stage8<TIn>(sm.raw_u[bf][warp][c], u_row, t, L, vin, g);
            if (li2 >= kNSub && g >= 2 && g < 2 + kOPieces) stage8<TOut>(sm.raw_o[bf][warp][c], o_row, t, L, vout, g - 2);
        }
        cp_async_commit();  // one group per step, empty past the last
    };
    // start of step li of block kb: issue the next step's copies, wait for this one's
    auto begin_step = [&](int64_t kb2, int li2) {
        __syncwarp();  // every lane is done with the buffers the next copies fill
        const bool wrap = li2 == 2 * kNSub - 1;
        issue_step(wrap ? kb2 - 1 : kb2, wrap ? 0 : li2 + 1);
        cp_async_wait1();
        __syncwarp();
    };

    const int64_t nblk = (L + kBlk - 1) / kBlk;
    if (nblk > 0) issue_step(nblk - 1, 0);
    for (int64_t kb = nblk - 1; kb >= 0; --kb) {
        const int64_t tb = kb * kBlk;
        __syncthreads();  // the previous block is done with bc and tok

        // ---- B and C of the block as fp32 token rows
        if (threadIdx.x < 2 * kBlk) {
            const int r = threadIdx.x;
            const bool isC = r >= kBlk;
            const int64_t t = tb + (r % kBlk);
            const TIn *base = (isC ? C_b : B_b) + t;
            const int64_t sn = isC ? a.C_sn : a.B_sn;
            float *row = &sm.bc[r % kBlk][isC ? 16 : 0];
#pragma unroll
            for (int n = 0; n < 16; ++n) row[n] = (n < N && t < L) ? ld_elem(base + n * sn) : 0.0f;
        }
        // ---- per-token quantities of the channel, once: lane g takes 16 tokens
#pragma unroll
        for (int h8 = 0; h8 < 2; ++h8) {
            const int off = 16 * g + 8 * h8;
            const int64_t ts = tb + off;
            float dv[8], zv[8];
            load8(d_row, ts, L, vin, dv);
            if (has_z) load8(z_row, ts, L, vin, zv);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float v = dv[j] + bias;
                float spv = v, sgv = 1.0f;
                if (sp) softplus_and_grad(v, spv, sgv);
                float gt = 1.0f, gp = 0.0f;
                if (has_z) {
                    const float zz = zv[j];
                    const float sz = logistic_f(zz);
                    gt = zz * sz;
                    gp = sz * (1.0f + zz * (1.0f - sz));
                }
                sm.tok[kTokDelta][warp][c][off + j] = (ts + j < L) ? spv : 0.0f;
                sm.tok[kTokSig][warp][c][off + j] = sgv;
                sm.tok[kTokGate][warp][c][off + j] = gt;
                sm.tok[kTokGateGrad][warp][c][off + j] = gp;
            }
        }
        __syncthreads();

        // ---- pass A: the block forward from its saved state; keep the state
        // at every sub-chunk start.
        f2 h[2];
        {
            float hv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                hv[i] = (active && n0 + i < N && MS_CHECK(a.status, kb >= 0 && kb < nblk))
                            ? __ldg(a.ckpt + ((b * a.dim + d) * nblk + kb) * N + n0 + i)
                            : 0.0f;
            h[0] = f2_make(hv[0], hv[1]);
            h[1] = f2_make(hv[2], hv[3]);
        }
        for (int s = 0; s < kNSub; ++s) {
#pragma unroll
            for (int p = 0; p < 2; ++p) {
                float lo, hi;
                f2_split(h[p], lo, hi);
                sm.sub[warp][s][2 * p][lane] = lo;
                sm.sub[warp][s][2 * p + 1][lane] = hi;
            }
            begin_step(kb, s);
            float uv[8];
            unstage8<TIn>(sm.raw_u[s & 1][warp][c], uv);
            const F4 dl0 = lds4(tk_dl + s * kSub), dl1 = lds4(tk_dl + s * kSub + 4);
#pragma unroll
            for (int j = 0; j < kSub; ++j) {
                const float dl = j < 4 ? dl0.v[j & 3] : dl1.v[j & 3];
                const f2 dl2 = f2_splat(dl), du2 = f2_splat(dl * uv[j]);
                f2 Bp[2];
                lds_f2x2(sm.bc[s * kSub + j] + n0, Bp[0], Bp[1]);
#pragma unroll
                for (int p = 0; p < 2; ++p) h[p] = f2_fma(exp2_mufu2(f2_mul(dl2, A2[p])), h[p], f2_mul(du2, Bp[p]));
            }
        }

        // ---- sub-chunks from the last: recompute, then the adjoint
        for (int s = kNSub - 1; s >= 0; --s) {
            const int64_t ts = tb + s * kSub;
            const int rb = s & 1;
            const int li = 2 * kNSub - 1 - s;
            begin_step(kb, li);
            float uv[8], ov[8];
            unstage8<TIn>(sm.raw_u[li & 1][warp][c], uv);
            // an idle lane (channel past dim) gets dout = 0: with its zero
            // starting adjoint every contribution to the channel sums is 0
            unstage8<TOut>(sm.raw_o[li & 1][warp][c], ov);
#pragma unroll
            for (int j = 0; j < kSub; ++j) ov[j] = active ? ov[j] : 0.0f;
            float dl[8], gate[8];
            {
                const F4 a0 = lds4(tk_dl + s * kSub), a1 = lds4(tk_dl + s * kSub + 4);
                const F4 g0 = lds4(tk_gate + s * kSub), g1 = lds4(tk_gate + s * kSub + 4);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    dl[j] = a0.v[j]; dl[4 + j] = a1.v[j];
                    gate[j] = g0.v[j]; gate[4 + j] = g1.v[j];
                }
            }
            // recompute A_bar and h of the sub-chunk, and the pre-gate output q
            f2 hs[2], ab[kSub][2], hh[kSub][2];
            float dq[kSub], qp[kSub];  // qp: the lane's share of the readout C . h
            hs[0] = f2_make(sm.sub[warp][s][0][lane], sm.sub[warp][s][1][lane]);
            hs[1] = f2_make(sm.sub[warp][s][2][lane], sm.sub[warp][s][3][lane]);
#pragma unroll
            for (int j = 0; j < kSub; ++j) {
                const f2 dl2 = f2_splat(dl[j]), du2 = f2_splat(dl[j] * uv[j]);
                f2 Bp[2], Cp[2];
                lds_f2x2(sm.bc[s * kSub + j] + n0, Bp[0], Bp[1]);
                lds_f2x2(sm.bc[s * kSub + j] + 16 + n0, Cp[0], Cp[1]);
                f2 acc = f2_splat(0.0f);
#pragma unroll
                for (int p = 0; p < 2; ++p) {
                    ab[j][p] = exp2_mufu2(f2_mul(dl2, A2[p]));
                    const f2 hp = j == 0 ? hs[p] : hh[j - 1][p];
                    hh[j][p] = f2_fma(ab[j][p], hp, f2_mul(du2, Bp[p]));
                    acc = f2_fma(Cp[p], hh[j][p], acc);
                }
                float plo, phi;
                f2_split(acc, plo, phi);
                qp[j] = plo + phi;
                dq[j] = ov[j] * gate[j];
            }
            // adjoint over the sub-chunk, last token first
            float ddt[kSub], dus[kSub];
#pragma unroll
            for (int j = kSub - 1; j >= 0; --j) {
                const f2 dq2 = f2_splat(dq[j]), dl2 = f2_splat(dl[j]), u2 = f2_splat(uv[j]);
                const f2 du2 = f2_splat(dl[j] * uv[j]);
                f2 Bp[2], Cp[2];
                lds_f2x2(sm.bc[s * kSub + j] + n0, Bp[0], Bp[1]);
                lds_f2x2(sm.bc[s * kSub + j] + 16 + n0, Cp[0], Cp[1]);
                f2 pdt = f2_splat(0.0f), pdu = f2_splat(0.0f), vB[2], vC[2];
#pragma unroll
                for (int p = 0; p < 2; ++p) {
                    const f2 lam = f2_fma(Cp[p], dq2, carry[p]);
                    const f2 hp = j == 0 ? hs[p] : hh[j - 1][p];
                    const f2 dab = f2_mul(lam, f2_mul(hp, ab[j][p]));
                    dAacc[p] = f2_fma(dab, dl2, dAacc[p]);
                    pdt = f2_fma(dab, An[p], pdt);
                    const f2 lb = f2_mul(lam, Bp[p]);
                    pdt = f2_fma(lb, u2, pdt);
                    pdu = f2_fma(lb, dl2, pdu);
                    vB[p] = f2_mul(lam, du2);        // dB
                    vC[p] = f2_mul(dq2, hh[j][p]);   // dC
                    carry[p] = f2_mul(ab[j][p], lam);
                }
                float x0, x1;
                f2_split(pdt, x0, x1);
                ddt[j] = x0 + x1;
                f2_split(pdu, x0, x1);
                dus[j] = x0 + x1;
                float v8[8];
                f2_split(vB[0], v8[0], v8[1]);
                f2_split(vB[1], v8[2], v8[3]);
                f2_split(vC[0], v8[4], v8[5]);
                f2_split(vC[1], v8[6], v8[7]);
                sm.red[rb][warp][j][lane] = reduce_scatter_channels(v8, c);
            }
            // per-token sums over the channel's 4 lanes; lane g owns tokens 2g, 2g+1
            // and writes both with one 8-byte store per gradient (full sectors
            // across the warp's 8 channels)
            reduce_scatter_lanes(ddt, g);
            reduce_scatter_lanes(dus, g);
            reduce_scatter_lanes(qp, g);  // the readout of tokens 2g, 2g+1 (only dz needs it)
            {
                // v[2g + k] from compile-time indices
                auto pick = [&](const float (&v)[kSub], int k) {
                    const float a0 = v[k], a1 = v[2 + k], a2 = v[4 + k], a3 = v[6 + k];
                    return g == 0 ? a0 : (g == 1 ? a1 : (g == 2 ? a2 : a3));
                };
                const int j0 = s * kSub + 2 * g;
                const int64_t t = ts + 2 * g;
                float ddv[2], duv[2], dzv[2];
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const float dqk = pick(dq, k);
                    ddv[k] = ddt[k] * tk_sig[j0 + k];
                    duv[k] = fmaf(Dd, dqk, dus[k]);
                    dzv[k] = pick(ov, k) * fmaf(Dd, pick(uv, k), qp[k]) * tk_gp[j0 + k];
                    if (active && t + k < L) {
                        dDacc = fmaf(dqk, pick(uv, k), dDacc);
                        dbacc += ddv[k];
                    }
                }
                const bool want_dz = has_z && a.dz != nullptr;
                if (active && t + 1 < L && MS_CHECK(a.status, t >= 0 && grow + t + 1 < grad_elems) &&
                    ((reinterpret_cast<uintptr_t>(a.ddelta + grow + t) | reinterpret_cast<uintptr_t>(a.du + grow + t) |
                      (want_dz ? reinterpret_cast<uintptr_t>(a.dz + grow + t) : 0)) & 7u) == 0) {
                    *reinterpret_cast<float2 *>(a.ddelta + grow + t) = make_float2(ddv[0], ddv[1]);
                    *reinterpret_cast<float2 *>(a.du + grow + t) = make_float2(duv[0], duv[1]);
                    if (want_dz) *reinterpret_cast<float2 *>(a.dz + grow + t) = make_float2(dzv[0], dzv[1]);
                } else if (active) {
#pragma unroll
                    for (int k = 0; k < 2; ++k) {
                        if (t + k < L && MS_CHECK(a.status, t + k >= 0 && grow + t + k < grad_elems)) {
                            a.ddelta[grow + t + k] = ddv[k];
                            a.du[grow + t + k] = duv[k];
                            if (want_dz) a.dz[grow + t + k] = dzv[k];
                        }
                    }
                }
            }
            // dB / dC: sum the warps' partial sums (this sub-chunk's buffer;
            // the other buffer is being filled by the next sub-chunk), then
            // one 4-token atomic per output row segment
            __syncthreads();
            if (threadIdx.x < 64) {
                const int col = threadIdx.x & 31;        // value column: lane that held it
                const int qd = threadIdx.x >> 5;         // token quad
                const int cg = col / kG, gg = col % kG;  // channel slot -> value, lane group -> states
                const bool isC = cg >= 4;
                const int n = gg * 4 + (cg & 3);
                float sum[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int j = 4 * qd + k;
                    sum[k] = 0.0f;
#pragma unroll
                    for (int w = 0; w < kBNW; ++w) sum[k] += sm.red[rb][w][j][col];
                }
                const int64_t t = ts + 4 * qd;
                if (n < N && MS_CHECK(a.status, t >= 0 && b < a.batch)) {
                    float *dst = (isC ? a.dC : a.dB) + (b * N + n) * L + t;
                    if (a.vec_bc && t + 4 <= L) {
                        atomicAdd(reinterpret_cast<float4 *>(dst), make_float4(sum[0], sum[1], sum[2], sum[3]));
                    } else {
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            if (t + k < L) atomicAdd(dst + k, sum[k]);
                    }
                }
            }
        }
    }

    // ---- per-channel results
    if (active) {
        float cv[4], av[4];
        f2_split(carry[0], cv[0], cv[1]);
        f2_split(carry[1], cv[2], cv[3]);
        f2_split(dAacc[0], av[0], av[1]);
        f2_split(dAacc[1], av[2], av[3]);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int n = n0 + i;
            if (n < N) {
                if (a.dh0 != nullptr) a.dh0[(b * a.dim + d) * N + n] = cv[i];
                atomicAdd(a.dA + d * N + n, av[i]);
            }
        }
    }
    dDacc += __shfl_xor_sync(0xffffffffu, dDacc, 1);
    dDacc += __shfl_xor_sync(0xffffffffu, dDacc, 2);
    dbacc += __shfl_xor_sync(0xffffffffu, dbacc, 1);
    dbacc += __shfl_xor_sync(0xffffffffu, dbacc, 2);
    if (active && g == 0) {
        if (a.dD != nullptr) atomicAdd(a.dD + d, dDacc);
        if (a.dbias != nullptr) atomicAdd(a.dbias + d, dbacc);
    }
}

template <typename TIn, typename TOut>
cudaError_t launch_bwd(const BwdArgs &a, unsigned grid, cudaStream_t stream) {
    // more than 48 KB of shared memory: opt in once per device
    static SmemOptIn opt_in;
    cudaError_t e = opt_in.ensure(reinterpret_cast<const void *>(scan_bwd_kernel<TIn, TOut>), (int)sizeof(BwdSmem));
    if (e != cudaSuccess) return e;
    scan_bwd_kernel<TIn, TOut><<<grid, kBThreads, sizeof(BwdSmem), stream>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_scan_bwd(const BwdArgs &a, bool in_bf16, bool out_bf16, cudaStream_t stream) {
    const int64_t dblocks = (a.dim + kBCh - 1) / kBCh;
    const int64_t blocks = dblocks * a.batch;
    if (blocks <= 0) return cudaSuccess;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    const unsigned grid = (unsigned)blocks;
    if (in_bf16) {
        return out_bf16 ? launch_bwd<__nv_bfloat16, __nv_bfloat16>(a, grid, stream)
                        : launch_bwd<__nv_bfloat16, float>(a, grid, stream);
    }
    return out_bf16 ? launch_bwd<float, __nv_bfloat16>(a, grid, stream) : launch_bwd<float, float>(a, grid, stream);
}

}  // namespace ms
