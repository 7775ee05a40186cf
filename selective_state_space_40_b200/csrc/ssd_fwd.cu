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
// One CTA of 4 warps walks the chunks of one (b, h) in order. Everything is
// computed transposed, S^T [P x N] and Y^T [P x Q]: warp w owns rows
// p in [16w, 16w+16) of both, so the state stays in its tensor-core
// accumulators (fp32) for the whole sequence and feeds the next chunk's
// S^T C^T product directly as register operands (an m16n8 accumulator pair
// has the layout of an m16n8k16 A operand). The products run on the tensor
// cores as bf16 x bf16 -> fp32 (mma.sync m16n8k16). Operands that are not
// bf16 inputs (the scaled G', B' and the state) are split into a high and a
// low bf16 part, v = hi + lo, and both parts are multiplied, which keeps
// about 16 significant bits. The next chunk's inputs are copied in
// asynchronously while the current one computes. A chunk has two phases
// between barriers: (1) the readout of the entering state, the masked C B^T
// and the weighted, split x^T; (2) the intra-chunk product, the output and
// the state update.

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
constexpr int kLdP = kP + 8;      // x rows (p contiguous): 8 rows of a transposing fragment load hit distinct banks
static_assert(kQ == 32, "one warp handles one token of the chunk per lane");
// the warp that prepares the chunk parameters (its tile of C B^T lies above
// the diagonal, so its share of that product is a zero fill)
constexpr int kParamWarp = 2;

struct SsdSmem {
    __nv_bfloat16 C[2][kQ][kLdN];     // C_t [t][n], this chunk and the next (copies in flight)
    __nv_bfloat16 B[2][kQ][kLdN];     // B_s [s][n]
    __nv_bfloat16 X[2][kQ][kLdP];     // x [s][p] as loaded
    __nv_bfloat16 G[2][kQ][kLdQ];     // G' hi / lo [t][s]
    __nv_bfloat16 Xw[2][kP][kLdQ];    // (x_s w_s)^T hi / lo [p][s], w_s = exp(cs_Q - cs_s) Delta_s
    // per-token chunk parameters, for this chunk and the next
    float dl[2][kQ];                  // Delta_t
    float cs[2][kQ];                  // A sum_{r<=t} Delta_r
    float wq[2][kQ];                  // exp(cs_Q - cs_s) Delta_s
    float ecs[2][kQ];                 // exp(cs_t)
};

// A operand fragment of the 16 x 16 tile at (m0, k0) of a row-major [m][k]
// bf16 array, in one ldmatrix (lane l addresses row m0 + l%8 + 8((l/8)%2),
// column k0 + 8(l/16)).
__device__ __forceinline__ void ldsm_a(const __nv_bfloat16 *base, int ld, int m0, int k0, int lane, uint32_t (&a)[4]) {
    const __nv_bfloat16 *p = base + (m0 + (lane & 7) + 8 * ((lane >> 3) & 1)) * ld + k0 + 8 * (lane >> 4);
    const unsigned ad = static_cast<unsigned>(__cvta_generic_to_shared(p));
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
                 : "r"(ad));
}
// B operand fragments (b0, b1) of the two 8-wide n-tiles at n0 and n0 + 8,
// k-step k0, from a [n][k] bf16 array (k contiguous), in one ldmatrix.
__device__ __forceinline__ void ldsm_b2(const __nv_bfloat16 *base, int ld, int n0, int k0, int lane, uint32_t (&b)[4]) {
    const __nv_bfloat16 *p = base + (n0 + (lane & 7) + 8 * (lane >> 4)) * ld + k0 + 8 * ((lane >> 3) & 1);
    const unsigned ad = static_cast<unsigned>(__cvta_generic_to_shared(p));
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(b[0]), "=r"(b[1]), "=r"(b[2]), "=r"(b[3])
                 : "r"(ad));
}

// B operand fragments of two adjacent 8-column tiles from a row-major [k][n]
// bf16 tile (k rows 16 bytes apart per 8 columns): ldmatrix with transpose
// hands each thread the (k = 2tig, 2tig+1) pairs of its column.
__device__ __forceinline__ void ldsm_x4_trans(const __nv_bfloat16 *row_addr, uint32_t &r0, uint32_t &r1,
                                              uint32_t &r2, uint32_t &r3) {
    const unsigned a = static_cast<unsigned>(__cvta_generic_to_shared(row_addr));
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(a));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo_elem, float hi_elem) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo_elem, hi_elem);
    return *reinterpret_cast<uint32_t *>(&v);
}
// hi and lo bf16 pairs of (x, y): x ~ hi.x + lo.x
__device__ __forceinline__ void split_pair(float x, float y, uint32_t &hi, uint32_t &lo) {
    __nv_bfloat162 h = __floats2bfloat162_rn(x, y);
    hi = *reinterpret_cast<uint32_t *>(&h);
    lo = pack_bf16(x - __low2float(h), y - __high2float(h));
}

__device__ __forceinline__ void cp_async16(void *sdst, const void *gsrc, int src_bytes) {
    const unsigned d = static_cast<unsigned>(__cvta_generic_to_shared(sdst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(gsrc), "r"(src_bytes) : "memory");
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
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
__global__ void __launch_bounds__(kST, 3) ssd_fwd_kernel(const SsdArgs a) {
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

    // S^T accumulators: warp w holds rows p in [16w, 16w+16) and all 128
    // columns n (16 n-tiles): sacc[j][e] is S[p][n] with p = 16w + gid (+8
    // for e >= 2), n = 8j + 2tig (+1 for odd e).
    const int pw = 16 * warp;
    float sacc[16][4];
    const float *s0 = a.s0 ? a.s0 + (b * a.H + h) * kP * kN : nullptr;
#pragma unroll
    for (int j = 0; j < 16; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int p = pw + gid + (e >= 2 ? 8 : 0);
            const int n = 8 * j + 2 * tig + (e & 1);
            sacc[j][e] = s0 ? __ldg(s0 + p * kN + n) : 0.0f;
        }

    const int64_t nch = (L + kQ - 1) / kQ;
    // Chunk inputs arrive by asynchronous copies one chunk ahead (rows past L
    // are zero-filled); dt goes through a register, one token per thread of
    // the parameter warp.
    auto issue_chunk = [&](int64_t ck, int buf) {
        const int64_t t0 = ck * kQ;
        for (int i = tid; i < kQ * (kN / 8); i += kST) {
            const int t = i / (kN / 8), q = i % (kN / 8);
            const bool in = t0 + t < L;
            const int64_t tt = in ? t0 + t : 0;
            cp_async16(&sm.C[buf][t][8 * q], Cb + tt * a.C_sl + 8 * q, in ? 16 : 0);
            cp_async16(&sm.B[buf][t][8 * q], Bb + tt * a.B_sl + 8 * q, in ? 16 : 0);
        }
        for (int i = tid; i < kQ * (kP / 8); i += kST) {
            const int t = i / (kP / 8), q = i % (kP / 8);
            const bool in = t0 + t < L;
            const int64_t tt = in ? t0 + t : 0;
            cp_async16(&sm.X[buf][t][8 * q], xb + tt * a.x_sl + 8 * q, in ? 16 : 0);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    float dt_next = 0.0f;
    auto load_dt = [&](int64_t ck) {
        const int64_t t = ck * kQ + lane;
        dt_next = (warp == kParamWarp && t < L) ? ld1(dtb + t * a.dt_sl) : 0.0f;
    };
    // parameter warp: Delta, the decay prefix and the per-token weights of chunk ck
    // (its dt already in dt_next) into parameter buffer pb
    auto chunk_params = [&](int64_t ck, int pb) {
        if (warp != kParamWarp) return;
        float d = 0.0f;
        if (ck * kQ + lane < L) {
            const float v = dt_next + bias;
            d = sp ? softplus_f(v) : v;
        }
        float c = Ah * d;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float o = __shfl_up_sync(0xffffffffu, c, off);
            if (lane >= off) c += o;
        }
        const float cend = __shfl_sync(0xffffffffu, c, kQ - 1);
        sm.dl[pb][lane] = d;
        sm.cs[pb][lane] = c;
        sm.wq[pb][lane] = __expf(cend - c) * d;
        sm.ecs[pb][lane] = __expf(c);
    };
    if (nch > 0) {
        issue_chunk(0, 0);
        load_dt(0);
        chunk_params(0, 0);
    }
    for (int64_t ck = 0; ck < nch; ++ck) {
        const int64_t t0 = ck * kQ;
        const int buf = (int)(ck & 1);
        asm volatile("cp.async.wait_group 0;" ::: "memory");
        __syncthreads();  // chunk ck in buf for everyone; chunk ck-1 is done with every tile
        // next chunk's copies (into the buffers chunk ck-1 used) run under this chunk's products
        if (ck + 1 < nch) {
            issue_chunk(ck + 1, buf ^ 1);
            load_dt(ck + 1);
        }
        const float *pcs = sm.cs[buf], *pdl = sm.dl[buf], *pwq = sm.wq[buf], *pecs = sm.ecs[buf];
        const float cs_end = pcs[kQ - 1];
        // ---- (x w)^T, hi / lo: warp task = 8 rows p x 8 tokens s; lane
        // (r, k) = (lane / 4, lane % 4) converts tokens 2k, 2k+1 of row r
        // (one bf16 pair per part: 32 distinct banks per store)
        for (int task = warp; task < (kP / 8) * (kQ / 8); task += kSW) {
            const int p = 8 * (task % (kP / 8)) + (lane >> 2);
            const int s = 8 * (task / (kP / 8)) + 2 * (lane & 3);
            const float x0 = __bfloat162float(sm.X[buf][s][p]) * pwq[s];
            const float x1 = __bfloat162float(sm.X[buf][s + 1][p]) * pwq[s + 1];
            uint32_t hi, lo;
            split_pair(x0, x1, hi, lo);
            *reinterpret_cast<uint32_t *>(&sm.Xw[0][p][s]) = hi;
            *reinterpret_cast<uint32_t *>(&sm.Xw[1][p][s]) = lo;
        }

        // ---- Y^T = S_in^T C^T, columns scaled by exp(cs_t): the state
        // accumulators are the A operand (hi and lo parts), C rows the B operand
        float yacc[4][4];
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) yacc[nt][e] = 0.0f;
#pragma unroll
        for (int kk = 0; kk < kN / 16; ++kk) {
            uint32_t ah[4], al[4];
            split_pair(sacc[2 * kk][0], sacc[2 * kk][1], ah[0], al[0]);
            split_pair(sacc[2 * kk][2], sacc[2 * kk][3], ah[1], al[1]);
            split_pair(sacc[2 * kk + 1][0], sacc[2 * kk + 1][1], ah[2], al[2]);
            split_pair(sacc[2 * kk + 1][2], sacc[2 * kk + 1][3], ah[3], al[3]);
#pragma unroll
            for (int np = 0; np < 2; ++np) {
                uint32_t bb[4];
                ldsm_b2(&sm.C[buf][0][0], kLdN, 16 * np, 16 * kk, lane, bb);
                mma_bf16(yacc[2 * np], ah[0], ah[1], ah[2], ah[3], bb[0], bb[1]);
                mma_bf16(yacc[2 * np + 1], ah[0], ah[1], ah[2], ah[3], bb[2], bb[3]);
                mma_bf16(yacc[2 * np], al[0], al[1], al[2], al[3], bb[0], bb[1]);
                mma_bf16(yacc[2 * np + 1], al[0], al[1], al[2], al[3], bb[2], bb[3]);
            }
        }
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
            const float e0 = pecs[8 * nt + 2 * tig], e1 = pecs[8 * nt + 2 * tig + 1];
            yacc[nt][0] *= e0; yacc[nt][1] *= e1;
            yacc[nt][2] *= e0; yacc[nt][3] *= e1;
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
                for (int k0 = 0; k0 < kN; k0 += 16) {
                    uint32_t af[4], bb[4];
                    ldsm_a(&sm.C[buf][0][0], kLdN, gm, k0, lane, af);
                    ldsm_b2(&sm.B[buf][0][0], kLdN, gn, k0, lane, bb);
                    mma_bf16(gacc[0], af[0], af[1], af[2], af[3], bb[0], bb[1]);
                    mma_bf16(gacc[1], af[0], af[1], af[2], af[3], bb[2], bb[3]);
                }
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int r = 0; r < 2; ++r) {
                        // elements (t, s) and (t, s + 1): one bf16 pair per part
                        const int t = gm + gid + 8 * r;
                        const int s = gn + 8 * nt + 2 * tig;
                        const float v0 = s <= t ? gacc[nt][2 * r] * __expf(pcs[t] - pcs[s]) * pdl[s] : 0.0f;
                        const float v1 =
                            s + 1 <= t ? gacc[nt][2 * r + 1] * __expf(pcs[t] - pcs[s + 1]) * pdl[s + 1] : 0.0f;
                        uint32_t hi, lo;
                        split_pair(v0, v1, hi, lo);
                        *reinterpret_cast<uint32_t *>(&sm.G[0][t][s]) = hi;
                        *reinterpret_cast<uint32_t *>(&sm.G[1][t][s]) = lo;
                    }
            } else {
                // strictly above the diagonal: zeros
                for (int i = lane; i < 16 * 8; i += 32) {
                    const int t = gm + i / 8, s = gn + 2 * (i % 8);
                    *reinterpret_cast<uint32_t *>(&sm.G[0][t][s]) = 0u;
                    *reinterpret_cast<uint32_t *>(&sm.G[1][t][s]) = 0u;
                }
            }
        }
        // the next chunk's parameters (its dt has arrived during this phase);
        // this chunk's were read above, the next chunk reads them after a barrier
        if (ck + 1 < nch) chunk_params(ck + 1, buf ^ 1);
        __syncthreads();

        // ---- Y^T += X^T G'^T over the causal part, then y = Y + D x
#pragma unroll
        for (int k0 = 0; k0 < kQ; k0 += 16) {
            // A = x^T rows p, columns s: transposing loads of the x tile
            // (matrix i = lane / 8: rows p + 8 (i & 1), tokens k0 + 8 (i / 2))
            uint32_t af[4];
            ldsm_x4_trans(&sm.X[buf][k0 + 8 * (lane >> 4) + (lane & 7)][pw + 8 * ((lane >> 3) & 1)], af[0], af[1],
                          af[2], af[3]);
#pragma unroll
            for (int part = 0; part < 2; ++part)
#pragma unroll
                for (int np = 0; np < 2; ++np) {
                    if (k0 > 16 * np + 15) continue;  // s > t for both tiles
                    uint32_t bb[4];
                    ldsm_b2(&sm.G[part][0][0], kLdQ, 16 * np, k0, lane, bb);
                    mma_bf16(yacc[2 * np], af[0], af[1], af[2], af[3], bb[0], bb[1]);
                    mma_bf16(yacc[2 * np + 1], af[0], af[1], af[2], af[3], bb[2], bb[3]);
                }
        }
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int p = pw + gid + (e >= 2 ? 8 : 0);
                const int t = 8 * nt + 2 * tig + (e & 1);
                if (t0 + t < L) {
                    const float v = yacc[nt][e] + Dh * __bfloat162float(sm.X[buf][t][p]);
                    TOut *dst = yb + (t0 + t) * a.y_sl + p;
                    if constexpr (sizeof(TOut) == 4) *dst = v;
                    else *dst = __float2bfloat16_rn(v);
                }
            }

        // ---- S_out^T = exp(cs_Q) S_in^T + (x w)^T B  (rows p, columns n): A
        // from the weighted x (hi / lo), B straight from the chunk's B rows
        const float decay = __expf(cs_end);
#pragma unroll
        for (int j = 0; j < 16; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) sacc[j][e] *= decay;
#pragma unroll
        for (int k0 = 0; k0 < kQ; k0 += 16) {
            uint32_t ah[4], al[4];
            ldsm_a(&sm.Xw[0][0][0], kLdQ, pw, k0, lane, ah);
            ldsm_a(&sm.Xw[1][0][0], kLdQ, pw, k0, lane, al);
#pragma unroll
            for (int j = 0; j < 16; j += 2) {
                // lanes 0-15: rows k0..k0+15 of columns 8j..; lanes 16-31: columns 8(j+1)..
                const __nv_bfloat16 *rowp = &sm.B[buf][k0 + (lane & 15)][8 * j + 8 * (lane >> 4)];
                uint32_t b0, b1, b2, b3;
                ldsm_x4_trans(rowp, b0, b1, b2, b3);
                mma_bf16(sacc[j], ah[0], ah[1], ah[2], ah[3], b0, b1);
                mma_bf16(sacc[j + 1], ah[0], ah[1], ah[2], ah[3], b2, b3);
                mma_bf16(sacc[j], al[0], al[1], al[2], al[3], b0, b1);
                mma_bf16(sacc[j + 1], al[0], al[1], al[2], al[3], b2, b3);
            }
        }
    }

    if (a.s_last != nullptr) {
        float *sl = a.s_last + (b * a.H + h) * kP * kN;
#pragma unroll
        for (int j = 0; j < 16; ++j)
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int p = pw + gid + 8 * r;
                const int n = 8 * j + 2 * tig;
                *reinterpret_cast<float2 *>(sl + p * kN + n) = make_float2(sacc[j][2 * r], sacc[j][2 * r + 1]);
            }
    }
}

template <typename TOut>
cudaError_t launch_ssd_t(const SsdArgs &a, cudaStream_t stream) {
    static SmemOptIn opt_in;
    cudaError_t e = opt_in.ensure(reinterpret_cast<const void *>(ssd_fwd_kernel<TOut>), (int)sizeof(SsdSmem));
    if (e != cudaSuccess) return e;
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
