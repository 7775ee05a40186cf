// ssd_chunk_cb.cu -- the intra-chunk product C B^T of the Mamba-2 SSD layer
// on the sm_100a tensor cores (tcgen05, accumulator in tensor memory).
//
// 'Mamba-1/2/3 Markdown図解' blog, section 3: in the matrix view of the SSD
// model the output of a chunk is built from the products C_t . B_s of the
// chunk's own tokens (the attention-like part), masked causally and weighted
// by the decay between s and t. The products C_t . B_s depend only on the
// batch row, the group of B/C and the chunk, not on the head, so they are
// formed once here for every head of the group:
//     cb[b][g][k][i][j] = sum_n C[b, 32k+i, g, n] B[b, 32k+j, g, n]
// for chunks of 32 tokens (i, j < 32; tokens past the sequence count as 0).
//
// One CTA (4 warps) per (batch row, group, tile of 128 tokens). The C and B
// rows of the tile (128 x 128 bf16 each) are copied to shared memory in the
// canonical K-major layout without swizzle: 8-row x 16-byte core matrices,
// the 16 core matrices of a row group adjacent along K (128 bytes apart), row
// groups 2048 bytes apart. One thread issues eight tcgen05.mma (M = N = 128,
// K = 16 each, bf16 x bf16 -> fp32) into a 128-column tensor-memory
// accumulator and commits them to an mbarrier; each warp then reads its 32
// accumulator lanes (tokens 32w..32w+31 of the tile) and stores the 32 x 32
// diagonal block of chunk w (columns 32w..32w+31). The off-diagonal blocks
// (pairs of tokens in different chunks) are computed and discarded.

#include <cstdint>

#include "mambascan.h"
#include "ms_device.cuh"
#include "ms_internal.h"

namespace ms {

namespace {

constexpr int kTileTok = 128;        // tokens per tile (the MMA's M and N)
constexpr int kChunkTok = 32;        // tokens per SSD chunk
constexpr int kK = 128;              // state size (the MMA's K)
constexpr int kCbThreads = 128;      // 4 warps: one per 32 accumulator lanes
constexpr uint32_t kTmemCols = 128;  // fp32 accumulator columns
constexpr uint32_t kWaitLimit = 1u << 20;

struct CbSmem {
    unsigned char a[kTileTok * kK * 2];  // C tile, canonical K-major (core matrices of 128 B)
    unsigned char b[kTileTok * kK * 2];  // B tile, same layout
    uint64_t bar;                        // MMA completion
    uint32_t tmem_base;                  // written by tcgen05.alloc
};

// Byte offset of the 16-byte piece (row r, K elements 8kc..8kc+7) in a tile:
// core matrix (r / 8, kc) at ((r / 8) * 16 + kc) * 128, row r % 8 inside it.
__device__ __forceinline__ uint32_t tile_off(int r, int kc) {
    return (uint32_t)((((r >> 3) * (kK / 8) + kc) * 8 + (r & 7)) * 16);
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Shared-memory matrix descriptor (tcgen05): start address, leading byte
// offset (between the two K core matrices of one K = 16 step), stride byte
// offset (between 8-row groups), all in 16-byte units; version 1; no swizzle.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}

// Instruction descriptor, kind::f16: fp32 accumulator (bits 4-5 = 1), A and B
// bf16 (bits 7-9 = 1, 10-12 = 1), both K-major (bits 15, 16 = 0), N >> 3 at
// bit 17, M >> 4 at bit 24.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kTileTok >> 3) << 17) |
                            ((uint32_t)(kTileTok >> 4) << 24);

__device__ __forceinline__ void cp_async16_zfill(uint32_t sdst, const void *gsrc, int src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(sdst), "l"(gsrc), "r"(src_bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity) {
    for (uint32_t i = 0; i < kWaitLimit; ++i) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(bar), "r"(parity)
            : "memory");
        if (done) return true;
    }
    return false;
}

__global__ void __launch_bounds__(kCbThreads) ssd_chunk_cb_kernel(const SsdCbArgs a) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    CbSmem &sm = *reinterpret_cast<CbSmem *>(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t tiles = (a.L + kTileTok - 1) / kTileTok;
    const int64_t tile = blockIdx.x % tiles;
    const int64_t bg = blockIdx.x / tiles;
    const int64_t b = bg / a.G, g = bg % a.G;
    const int64_t t0 = tile * kTileTok;
    const __nv_bfloat16 *Cg = static_cast<const __nv_bfloat16 *>(a.C) + b * a.C_sb + g * a.C_sg;
    const __nv_bfloat16 *Bg = static_cast<const __nv_bfloat16 *>(a.B) + b * a.B_sb + g * a.B_sg;

    // tile rows -> shared memory (16-byte pieces; rows past the sequence zero-filled)
    const uint32_t sa = smem_u32(sm.a), sb = smem_u32(sm.b);
    for (int i = tid; i < kTileTok * (kK / 8); i += kCbThreads) {
        const int r = i / (kK / 8), kc = i % (kK / 8);
        const bool in = t0 + r < a.L;
        const int64_t t = in ? t0 + r : 0;
        cp_async16_zfill(sa + tile_off(r, kc), Cg + t * a.C_sl + 8 * kc, in ? 16 : 0);
        cp_async16_zfill(sb + tile_off(r, kc), Bg + t * a.B_sl + 8 * kc, in ? 16 : 0);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");

    const uint32_t bar = smem_u32(&sm.bar);
    if (warp == 0) {
        // tensor memory for the accumulator (one warp allocates, frees at the end)
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&sm.tmem_base)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar) : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    // the copies (async proxy writes) and the thread writes -> visible to the tensor cores
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = sm.tmem_base;

    if (tid == 0) {
#pragma unroll
        for (int s = 0; s < kK / 16; ++s) {
            // K step s: core matrices 2s and 2s + 1 of every row group
            const uint64_t da = smem_desc(sa + 256u * s, 128u, 2048u);
            const uint64_t db = smem_desc(sb + 256u * s, 128u, 2048u);
            const uint32_t acc = s > 0 ? 1u : 0u;
            asm volatile(
                "{\n\t.reg .pred p;\n\t"
                "setp.ne.b32 p, %4, 0;\n\t"
                "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}"
                :
                : "r"(tmem), "l"(da), "l"(db), "r"(kIdesc), "r"(acc), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
                : "memory");
        }
        asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                     : "memory");
    }
    // one decision per warp: the tensor-memory load below is warp-collective
    const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(bar, 0));
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (!ok) {
        if (lane == 0 && a.status) atomicOr(a.status, MS_ERR_TIMEOUT);
    } else {
        // warp w: accumulator lanes 32w.. (tokens of chunk w), columns 32w.. (the same chunk)
        uint32_t v[32];
        const uint32_t taddr = tmem + ((uint32_t)(32 * warp) << 16) + (uint32_t)(32 * warp);
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
            "%13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, "
            "[%32];"
            : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
              "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]),
              "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]),
              "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]),
              "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
            : "r"(taddr)
            : "memory");
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
        const int64_t nch = (a.L + kChunkTok - 1) / kChunkTok;
        const int64_t ck = tile * (kTileTok / kChunkTok) + warp;
        if (ck < nch) {
            float4 *dst = reinterpret_cast<float4 *>(a.cb + (((bg * nch + ck) * kChunkTok) + lane) * kChunkTok);
#pragma unroll
            for (int q = 0; q < 8; ++q)
                dst[q] = make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                                     __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == 0) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                     : "memory");
    }
}

}  // namespace

bool ssd_cb_shape_supported(int64_t dstate) { return dstate == kK; }

cudaError_t launch_ssd_chunk_cb(const SsdCbArgs &a, cudaStream_t stream) {
    static SmemOptIn opt_in;
    cudaError_t e = opt_in.ensure(reinterpret_cast<const void *>(ssd_chunk_cb_kernel), (int)sizeof(CbSmem));
    if (e != cudaSuccess) return e;
    const int64_t tiles = (a.L + kTileTok - 1) / kTileTok;
    const int64_t blocks = a.batch * a.G * tiles;
    if (blocks <= 0) return cudaSuccess;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    ssd_chunk_cb_kernel<<<(unsigned)blocks, kCbThreads, sizeof(CbSmem), stream>>>(a);
    return cudaGetLastError();
}

}  // namespace ms
