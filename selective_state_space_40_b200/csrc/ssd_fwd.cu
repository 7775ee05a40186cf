// ssd_fwd.cu -- Mamba-2 state space duality layer (forward) on sm_100a.
//
// 'Mamba-1/2/3 Markdown図解' blog, section 3: the SSD model has a recurrent
// view (one state update per token, for decoding) and a matrix view computed
// chunk by chunk for training and prefill: inside a chunk the work is matrix
// products, between chunks the state is passed on; the transition is a
// scalar times the identity within a head. Per batch row b and head h (state
// S [P x N], group g of B and C):
//   S_t = exp(Delta_t A_h) S_{t-1} + Delta_t x_t B_t^T,   y_t = S_t C_t + D_h x_t
// With cs_t = A_h sum_{r<=t} Delta_r inside a chunk of Q tokens and S_in the
// state entering it:
//   y_t   = exp(cs_t) C_t . S_in + sum_{s<=t} (C_t . B_s) exp(cs_t - cs_s) Delta_s x_s + D x_t
//   S_out = exp(cs_Q) S_in + sum_s exp(cs_Q - cs_s) Delta_s x_s B_s^T
// i.e. four products per chunk: Y = C S_in (scaled by row), G = C B^T (masked
// and scaled), Y += G' X, S_out = exp(cs_Q) S_in + B'^T X.
//
// One CTA of 4 warps walks the chunks of one (b, h) in order; the state lives
// in the warps' tensor-core accumulators (fp32) for the whole sequence. The
// products run on the tensor cores as bf16 x bf16 -> fp32 (mma.sync
// m16n8k16). Operands that are not bf16 inputs (the scaled G', B' and the
// state) are split into a high and a low bf16 part, v = hi + lo, and both
// parts are multiplied, which keeps about 16 significant bits.

#include <cstdint>

#include "ms_device.cuh"
#include "ms_internal.h"

namespace ms {

namespace {

constexpr int kQ = 32;            // tokens per chunk
constexpr int kP = 64;            // head dim
constexpr int kN = 128;           // state size
constexpr int kSW = 4;            // warps
constexpr int kST = kSW * 32;     // threads
// Shared row strides in bf16 elements: K/2 + 4 words, so that 8 rows x 4
// words of one fragment load fall in 32 distinct banks.
constexpr int kLdN = kN + 8;      // rows of K = N
constexpr int kLdQ = kQ + 8;      // rows of K = Q

struct SsdSmem {
    __nv_bfloat16 C[kQ][kLdN];        // C_t [t][n]
    __nv_bfloat16 B[kQ][kLdN];        // B_s [s][n]
    __nv_bfloat16 Xt[kP][kLdQ];       // x^T [p][s]
    __nv_bfloat16 G[2][kQ][kLdQ];     // G' hi / lo [t][s]
    __nv_bfloat16 Bt[2][kN][kLdQ];    // B'^T hi / lo [n][s]
    __nv_bfloat16 S[2][kP][kLdN];     // state^T hi / lo [p][n]
    float dl[kQ];                     // Delta_t
    float cs[kQ];                     // A sum_{r<=t} Delta_r
};

__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t ld32(const __nv_bfloat16 *p) { return *reinterpret_cast<const uint32_t *>(p); }

// acc[16 x 8 tile] += A[m0.., k0..k0+16) * B[k0.., n0..n0+8), with A stored
// [m][k] (row stride lda) and B stored [n][k] (row stride ldb), bf16.
__device__ __forceinline__ void mma_tile(float (&acc)[4], const __nv_bfloat16 *A, int lda, int m0,
                                         const __nv_bfloat16 *Bm, int ldb, int n0, int k0, int gid, int tig) {
    const __nv_bfloat16 *ar = A + (m0 + gid) * lda + k0 + 2 * tig;
    const __nv_bfloat16 *br = Bm + (n0 + gid) * ldb + k0 + 2 * tig;
    mma_bf16(acc, ld32(ar), ld32(ar + 8 * lda), ld32(ar + 8), ld32(ar + 8 * lda + 8), ld32(br), ld32(br + 8));
}

__device__ __forceinline__ void split_bf16(float v, __nv_bfloat16 &hi, __nv_bfloat16 &lo) {
    hi = __float2bfloat16_rn(v);
    lo = __float2bfloat16_rn(v - __bfloat162float(hi));
}

template <typename TIn>
__device__ __forceinline__ float ld1(const TIn *p) {
    if constexpr (sizeof(TIn) == 4) return __ldg(reinterpret_cast<const float *>(p));
    else return bf16_bits_to_f32(__ldg(reinterpret_cast<const unsigned short *>(p)));
}

template <typename TOut>
__global__ void __launch_bounds__(kST, 2) ssd_fwd_kernel(const SsdArgs a) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    SsdSmem &sm = *reinterpret_cast<SsdSmem *>(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int gid = lane >> 2, tig = lane & 3;
    const int64_t b = blockIdx.x / a.H, h = blockIdx.x % a.H;
    const int64_t g = h / (a.H / a.G);
    const int64_t L = a.L;
    const float Ah = __ldg(a.A + h);
    const float Dh = a.D ? __ldg(a.D + h) : 0.0f;
    const float bias = a.dt_bias ? __ldg(a.dt_bias + h) : 0.0f;
    const bool sp = a.softplus != 0;

    const __nv_bfloat16 *xb = static_cast<const __nv_bfloat16 *>(a.x) + b * a.x_sb + h * a.x_sh;
    const __nv_bfloat16 *dtb = static_cast<const __nv_bfloat16 *>(a.dt) + b * a.dt_sb + h;
    const __nv_bfloat16 *Bb = static_cast<const __nv_bfloat16 *>(a.B) + b * a.B_sb + g * a.B_sg;
    const __nv_bfloat16 *Cb = static_cast<const __nv_bfloat16 *>(a.C) + b * a.C_sb + g * a.C_sg;
    TOut *yb = static_cast<TOut *>(a.y) + b * a.y_sb + h * a.y_sh;

    // State accumulators: warp w holds rows n in [32w, 32w+32) (two m-tiles)
    // and all 64 columns p (eight n-tiles): element (n, p) of S^T... i.e.
    // S[p][n] sits at n = 32w + 16mt + gid (+8), p = 8nt + 2tig (+1).
    float sacc[2][8][4];
    const float *s0 = a.s0 ? a.s0 + (b * a.H + h) * kP * kN : nullptr;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int n = 32 * warp + 16 * mt + gid + (e >= 2 ? 8 : 0);
                const int p = 8 * nt + 2 * tig + (e & 1);
                sacc[mt][nt][e] = s0 ? __ldg(s0 + p * kN + n) : 0.0f;
            }
    // state^T into shared memory as hi/lo bf16 [p][n]
    auto store_state = [&]() {
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int n = 32 * warp + 16 * mt + gid + (e >= 2 ? 8 : 0);
                    const int p = 8 * nt + 2 * tig + (e & 1);
                    split_bf16(sacc[mt][nt][e], sm.S[0][p][n], sm.S[1][p][n]);
                }
    };
    store_state();

    const int64_t nch = (L + kQ - 1) / kQ;
    for (int64_t ck = 0; ck < nch; ++ck) {
        const int64_t t0 = ck * kQ;
        __syncthreads();  // everyone is done with the previous chunk's tiles
        // ---- load the chunk: C, B rows (16-byte pieces), x transposed, Delta
        for (int i = tid; i < kQ * (kN / 8); i += kST) {
            const int t = i / (kN / 8), q = i % (kN / 8);
            uint4 vc = make_uint4(0u, 0u, 0u, 0u), vb = vc;
            if (t0 + t < L) {
                vc = __ldg(reinterpret_cast<const uint4 *>(Cb + (t0 + t) * a.C_sl) + q);
                vb = __ldg(reinterpret_cast<const uint4 *>(Bb + (t0 + t) * a.B_sl) + q);
            }
            *reinterpret_cast<uint4 *>(&sm.C[t][8 * q]) = vc;
            *reinterpret_cast<uint4 *>(&sm.B[t][8 * q]) = vb;
        }
        for (int i = tid; i < kQ * (kP / 8); i += kST) {
            const int t = i / (kP / 8), q = i % (kP / 8);
            uint4 vx = make_uint4(0u, 0u, 0u, 0u);
            if (t0 + t < L) vx = __ldg(reinterpret_cast<const uint4 *>(xb + (t0 + t) * a.x_sl) + q);
            const __nv_bfloat16 *e = reinterpret_cast<const __nv_bfloat16 *>(&vx);
#pragma unroll
            for (int k = 0; k < 8; ++k) sm.Xt[8 * q + k][t] = e[k];
        }
        if (tid < kQ) {
            const int64_t t = t0 + tid;
            float d = 0.0f;
            if (t < L) {
                const float v = ld1(dtb + t * a.dt_sl) + bias;
                d = sp ? softplus_f(v) : v;
            }
            sm.dl[tid] = d;
        }
        __syncthreads();
        if (tid == 0) {
            float c = 0.0f;
            for (int t = 0; t < kQ; ++t) {
                c = fmaf(Ah, sm.dl[t], c);
                sm.cs[t] = c;
            }
        }
        __syncthreads();
        const float cs_end = sm.cs[kQ - 1];

        // ---- Y = exp(cs_t) C_t . S_in  (warp: rows 16(w%2).., cols 32(w/2)..)
        const int ym = 16 * (warp & 1), yn = 32 * (warp >> 1);
        float yacc[4][4];
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) yacc[nt][e] = 0.0f;
#pragma unroll
        for (int k0 = 0; k0 < kN; k0 += 16)
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int part = 0; part < 2; ++part)
                    mma_tile(yacc[nt], &sm.C[0][0], kLdN, ym, &sm.S[part][0][0], kLdN, yn + 8 * nt, k0, gid, tig);
        {
            const float e0 = __expf(sm.cs[ym + gid]), e1 = __expf(sm.cs[ym + gid + 8]);
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                yacc[nt][0] *= e0; yacc[nt][1] *= e0;
                yacc[nt][2] *= e1; yacc[nt][3] *= e1;
            }
        }

        // ---- G = C B^T, masked and scaled: G'_ts = G exp(cs_t - cs_s) Delta_s, s <= t
        {
            const int gm = 16 * (warp & 1), gn = 16 * (warp >> 1);
            if (gn <= gm + 15) {
                float gacc[2][4];
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) gacc[nt][e] = 0.0f;
#pragma unroll
                for (int k0 = 0; k0 < kN; k0 += 16)
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt)
                        mma_tile(gacc[nt], &sm.C[0][0], kLdN, gm, &sm.B[0][0], kLdN, gn + 8 * nt, k0, gid, tig);
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int t = gm + gid + (e >= 2 ? 8 : 0);
                        const int s = gn + 8 * nt + 2 * tig + (e & 1);
                        const float v = s <= t ? gacc[nt][e] * __expf(sm.cs[t] - sm.cs[s]) * sm.dl[s] : 0.0f;
                        split_bf16(v, sm.G[0][t][s], sm.G[1][t][s]);
                    }
            } else {
                // strictly above the diagonal: zeros
                for (int i = lane; i < 16 * 16; i += 32) {
                    const int t = gm + i / 16, s = gn + i % 16;
                    sm.G[0][t][s] = __float2bfloat16_rn(0.0f);
                    sm.G[1][t][s] = __float2bfloat16_rn(0.0f);
                }
            }
        }
        __syncthreads();

        // ---- Y += G' X over the causal part, then y = Y + D x
#pragma unroll
        for (int k0 = 0; k0 < kQ; k0 += 16) {
            if (k0 > ym + 15) continue;
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int part = 0; part < 2; ++part)
                    mma_tile(yacc[nt], &sm.G[part][0][0], kLdQ, ym, &sm.Xt[0][0], kLdQ, yn + 8 * nt, k0, gid, tig);
        }
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int t = ym + gid + 8 * r;
                const int p = yn + 8 * nt + 2 * tig;
                if (t0 + t < L) {
                    const float v0 = yacc[nt][2 * r] + Dh * __bfloat162float(sm.Xt[p][t]);
                    const float v1 = yacc[nt][2 * r + 1] + Dh * __bfloat162float(sm.Xt[p + 1][t]);
                    TOut *dst = yb + (t0 + t) * a.y_sl + p;
                    if constexpr (sizeof(TOut) == 4) {
                        *reinterpret_cast<float2 *>(dst) = make_float2(v0, v1);
                    } else {
                        *reinterpret_cast<__nv_bfloat162 *>(dst) = __floats2bfloat162_rn(v0, v1);
                    }
                }
            }

        // ---- B'^T [n][s] = exp(cs_Q - cs_s) Delta_s B_s[n], hi / lo
        for (int i = tid; i < kN * kQ; i += kST) {
            const int n = i / kQ, s = i % kQ;
            const float v = __bfloat162float(sm.B[s][n]) * __expf(cs_end - sm.cs[s]) * sm.dl[s];
            split_bf16(v, sm.Bt[0][n][s], sm.Bt[1][n][s]);
        }
        __syncthreads();

        // ---- S_out = exp(cs_Q) S_in + B'^T X  (rows n, columns p)
        const float decay = __expf(cs_end);
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) sacc[mt][nt][e] *= decay;
#pragma unroll
        for (int k0 = 0; k0 < kQ; k0 += 16)
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                    for (int part = 0; part < 2; ++part)
                        mma_tile(sacc[mt][nt], &sm.Bt[part][0][0], kLdQ, 32 * warp + 16 * mt, &sm.Xt[0][0], kLdQ,
                                 8 * nt, k0, gid, tig);
        __syncthreads();  // the state's old copy is no longer read (Y above)
        store_state();
    }

    if (a.s_last != nullptr) {
        float *sl = a.s_last + (b * a.H + h) * kP * kN;
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int n = 32 * warp + 16 * mt + gid + (e >= 2 ? 8 : 0);
                    const int p = 8 * nt + 2 * tig + (e & 1);
                    sl[p * kN + n] = sacc[mt][nt][e];
                }
    }
}

template <typename TOut>
cudaError_t launch_ssd_t(const SsdArgs &a, cudaStream_t stream) {
    static bool opted[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 64 || !opted[dev]) {
        e = cudaFuncSetAttribute(ssd_fwd_kernel<TOut>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)sizeof(SsdSmem));
        if (e != cudaSuccess) return e;
        if (dev < 64) opted[dev] = true;
    }
    const int64_t blocks = a.batch * a.H;
    if (blocks <= 0) return cudaSuccess;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    ssd_fwd_kernel<TOut><<<(unsigned)blocks, kST, sizeof(SsdSmem), stream>>>(a);
    return cudaGetLastError();
}

}  // namespace

bool ssd_shape_supported(int64_t headdim, int64_t dstate) { return headdim == kP && dstate == kN; }

cudaError_t launch_ssd_fwd(const SsdArgs &a, bool out_bf16, cudaStream_t stream) {
    return out_bf16 ? launch_ssd_t<__nv_bfloat16>(a, stream) : launch_ssd_t<float>(a, stream);
}

}  // namespace ms
