// ssd_fwd_tc.cu -- Mamba-2 state space duality (SSD) layer, forward, chunk-
// parallel on the sm_100a tensor cores (tcgen05, accumulators in tensor
// memory).
//
// 'Mamba-1/2/3 Markdown図解' blog, section 3: the SSD model has a recurrent
// view and a matrix view computed chunk by chunk -- matrix products inside a
// chunk, the state handed from one chunk to the next; the transition is a
// scalar times the identity within a head. Per batch row b and head h (state
// S [N x P] here, group g of B and C):
//   S_t = exp(Delta_t A_h) S_{t-1} + B_t (Delta_t x_t)^T,   y_t = S_t^T C_t + D_h x_t
// With cs_t = A_h sum_{r<=t} Delta_r inside a chunk of Q tokens (t = 0..Q-1)
// and S_in the state entering it:
//   y_t   = exp(cs_t) sum_n C_t[n] S_in[n][.] + sum_{s<=t} (C_t . B_s) exp(cs_t - cs_s) Delta_s x_s + D x_t
//   S_out = exp(cs_{Q-1}) S_in + sum_s B_s (w_s x_s)^T,   w_s = exp(cs_{Q-1} - cs_s) Delta_s
// Four products per chunk and head, each M = 128 on the tensor cores
// (bf16 x bf16 -> fp32; CB is formed again for every head, in the tensor
// memory G' then takes):
//   CB    [Q x Q] = C B^T
//   S_c   [N x P] = B^T X'        X'[s] = w_s x_s
//   Y_i   [Q x P] = G' X          G'[t][s] = CB[t][s] exp(cs_t - cs_s) Delta_s (s <= t)
//   Y_s   [Q x P] = C S_in
// and y_t = exp(cs_t) Y_s[t] + Y_i[t] + D x_t, S_out = exp(cs_{Q-1}) S_in + S_c.
// Operands that are not bf16 inputs (X', G', S_in) are split into a high and
// a low bf16 part, v = hi + lo, and both are multiplied (about 16 significant
// bits).
//
// Work item = (chunk k, batch row b, block of up to 8 heads of one group).
// Items are claimed in ticket order from a global counter, chunk-major, so the
// item holding chunk k - 1 of the same heads was claimed before this one. The
// kernel is persistent (one CTA per SM): a CTA holds at most the item it
// computes and the one its producer warp prepares, and the smallest unfinished
// ticket is always one that some CTA computes, so every wait ends. Only
// Y_s and S_out depend on the entering state: each head computes CB, S_c and
// Y_i first, then waits for chunk k - 1's item to publish S_in (a per-(b, h)
// counter in global memory), writes S_out over it and publishes it for chunk
// k + 1. The running state lives in the workspace and crosses chunks through
// L2, so HBM sees each input once.
//
// CTA: two groups of 4 compute warps, one MMA warp (lane 0 issues every
// tcgen05.mma and commit) and one producer warp, which claims the next item,
// forms its per-head Delta, cumulative decay and w_s into the other of two
// parameter buffers while the current item computes, and loads the item's C
// tile into the other of two C buffers and its B tile once every S_c of the
// previous item has completed (tensor copies). The MMA warp runs each slot's
// heads as its own sequence, so a group enters the next item while the other
// finishes this one; each thread of a group copies its x row of the group's
// next head as soon as it has read the current one. The groups take alternate
// heads of the item, each
// with its own half of tensor memory (a slot: CB, overwritten in place by G'
// as packed bf16 hi / lo, the A operand of Y_i; S_c, later Y_s; Y_i) and its
// own x and X' (later S_in) buffers, so one group's products run while the
// other group computes. In a group, thread t of warp w owns accumulator lane
// 32 (w % 4) + lane: a token row (CB, G', Y) or a state row (S_c). The MMA
// warp serves whichever slot is ready. Shared-memory operands use the
// canonical layouts without swizzle (8-row x 16-byte core matrices): K-major
// for C (and B in C B^T), MN-major for B (in B^T X'), x, X' and S_in -- the
// same bytes of the B tile serve both of its roles. Every wait is bounded: on a
// timeout the CTA records MS_ERR_TIMEOUT, stops, waits (bounded) for its
// issued products and frees its tensor memory.

#include <cuda.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "mambascan.h"
#include "ms_device.cuh"
#include "ms_internal.h"

// MN-major no-swizzle descriptor fields: 1 = leading byte offset along K,
// stride byte offset along M/N (the K-major assignment); 0 = the reverse.
#ifndef MS_SSD_MN_LBO_K
#define MS_SSD_MN_LBO_K 1
#endif
// Back-off (ns) of the MMA warp's polling rounds that find no event: the warp
// shares its scheduler with compute warps.
#ifndef MS_SSD_POLL_NS
#define MS_SSD_POLL_NS 20
#endif

namespace ms {

namespace {

constexpr int kQ = 128;        // tokens per chunk
constexpr int kP = 64;         // head dim
constexpr int kN = 128;        // state size
constexpr int kHB = 4;         // most heads per work item
constexpr int kGroupWarps = 4;                       // one warp per 32 accumulator lanes
constexpr int kGroupThreads = 32 * kGroupWarps;
constexpr int kComputeWarps = 2 * kGroupWarps;
constexpr int kMmaWarp = kComputeWarps;              // issues every product
constexpr int kProdWarp = kComputeWarps + 1;         // claims items, forms their parameters, loads C and B
constexpr int kThreads = 32 * (kComputeWarps + 2);
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSlotCols = 256;
// columns inside a slot: CB (fp32, 128), then G' in place -- the 32 tokens s of
// CB block c (columns 32c..32c+31) become 16 columns of packed hi pairs and 16
// of lo pairs in the same columns; S_c, then Y_s (64); Y_i (64)
constexpr uint32_t kColCB = 0, kColSC = 128, kColYI = 192;
// G' of K-step ks (tokens 16ks..16ks+15), part 0 = hi / 1 = lo
__host__ __device__ constexpr uint32_t g_col(int ks, int part) {
    return (uint32_t)(32 * (ks >> 1) + 16 * part + 8 * (ks & 1));
}
constexpr uint32_t kSpinTries = 1u << 20;       // mbarrier try_wait rounds
constexpr uint32_t kFlagTries = 1u << 22;       // polls of a predecessor's counter (with a short sleep)
constexpr uint32_t kIdleTries = 1u << 24;       // MMA warp polls without an event

// shared-memory map (bytes)
constexpr int kTileHalf = kQ * kP * 2;            // 16 KB: one [128 x 64] bf16 operand
constexpr int kTileCB = kQ * kN * 2;              // one C or B tile, 32 KB
constexpr int kOffC = 0;                          // two C tiles (items alternate)
constexpr int kOffB = kOffC + 2 * kTileCB;        // the B tile
constexpr int kOffSlot = kOffB + kTileCB;         // per slot: X' / S_in hi, lo 32 KB; x [s][p] MN-major 16 KB
constexpr int kSlotBytes = 3 * kTileHalf;
constexpr int kParBytes = 4 * kHB * kQ * 4;          // dl, cs2, w, fd: [kHB][kQ] floats each
constexpr int kOffPar = kOffSlot + 2 * kSlotBytes;  // two parameter buffers (items alternate)
constexpr int kOffBar = kOffPar + 2 * kParBytes;
enum { kBarXP = 0, kBarCB, kBarSC, kBarG, kBarYI, kBarS, kBarYS, kBarsPerSlot };
constexpr int kBarParFull = 2 * kBarsPerSlot;  // [2] an item's descriptor and parameters are in buffer i
constexpr int kBarParFree = kBarParFull + 2;   // [2] every consumer is done with buffer i
constexpr int kBarCFull = kBarParFree + 2;     // [2] item i's C tile is in buffer i % 2
constexpr int kBarCFree = kBarCFull + 2;       // [2] the products of the item in C buffer i are done
constexpr int kBarBFull = kBarCFree + 2;       // the B tile of the next item to read it is in
constexpr int kBarBFree = kBarBFull + 1;       // every product reading an item's B tile is done
constexpr int kBarEnd = kBarBFree + 1, kNumBars = kBarEnd + 1;

// A work item as the producer warp hands it to the others (valid = 0: no more)
struct ItemDesc {
    long long k, b, g, h0;
    int nh, valid;
};
constexpr int kOffDesc = kOffBar + 8 * kNumBars;                // ItemDesc per parameter buffer
constexpr int kOffMisc = kOffDesc + 2 * (int)sizeof(ItemDesc);  // tensor-memory base, -, abort
constexpr int kSmemBytes = kOffMisc + 16;

// C / B tile [128 tokens x 128 states] bf16 as [n / 8][t][n % 8] (the order a
// tensor copy writes its box {8 states, 128 tokens, 16 state chunks}): core
// matrix (t / 8, n / 8) -- 8 token rows of 16 bytes -- at (n / 8) * 2048 + (t / 8)
// * 128. Read K-major (K = n: C, and B in C B^T) the K-direction core stride is
// 2048 and the token-direction one 128; read M(n)-major (B in B^T X') the
// K(t)-direction stride is 128 and the n-direction one 2048.
__device__ __forceinline__ uint32_t cb_off(int t, int kc) { return (uint32_t)(kc * 2048 + t * 16); }
// MN-major no-swizzle [k rows x 64] bf16 operand (k = token or state, 64
// columns p): core matrix (k / 8, p / 8) at (k / 8) * 1024 + (p / 8) * 128,
// k % 8 at 16-byte steps inside it.
__device__ __forceinline__ uint32_t mn64_off(int k, int pc) {
    return (uint32_t)((k >> 3) * 1024 + pc * 128 + (k & 7) * 16);
}

__device__ __forceinline__ uint32_t saddr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}
// K-major: leading offset between the two core matrices along K, stride
// between 8-row groups.
__device__ __forceinline__ uint64_t desc_k(uint32_t addr, uint32_t k_stride, uint32_t mn_stride) {
    return sdesc(addr, k_stride, mn_stride);
}
__device__ __forceinline__ uint64_t desc_mn(uint32_t addr, uint32_t k_stride, uint32_t mn_stride) {
#if MS_SSD_MN_LBO_K
    return sdesc(addr, k_stride, mn_stride);
#else
    return sdesc(addr, mn_stride, k_stride);
#endif
}
// Instruction descriptor, kind::f16: fp32 D (bits 4-5), bf16 A and B (bits
// 7-9, 10-12), A / B major-ness (bit 15 / 16: 1 = M/N-major), N >> 3 at bit
// 17, M >> 4 at bit 24.
constexpr uint32_t idesc(int n, bool a_mn, bool b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
           ((uint32_t)(n >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

__device__ __forceinline__ void mma(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t id, bool acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        :
        : "r"(tmem_d), "l"(da), "l"(db), "r"(id), "r"(acc ? 1u : 0u)
        : "memory");
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}
__device__ __forceinline__ void bar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void bar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool bar_wait(uint32_t bar, uint32_t parity) {
    for (uint32_t i = 0; i < kSpinTries; ++i) {
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
// Named barrier `id` over `n` threads, and-reducing a predicate: the compute
// warps (id 1) or one group (id 2 + group).
template <int kThreadsIn>
__device__ __forceinline__ bool sync_and(int id, bool ok) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "barrier.cta.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(ok ? 1u : 0u), "r"(id), "n"(kThreadsIn)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ bool bar_test(uint32_t bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    return done != 0;
}
// D (tensor memory) [+]= A (tensor memory) x B (shared memory)
__device__ __forceinline__ void mma_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t db, uint32_t id, bool acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
        :
        : "r"(tmem_d), "r"(tmem_a), "l"(db), "r"(id), "r"(acc ? 1u : 0u)
        : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16};"
        :
        : "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
          "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
// Tensor store (no multicast) of a 4-D box from shared memory, and its groups
__device__ __forceinline__ void tma_store4(const CUtensorMap *map, uint32_t src, int c0, int c1, int c2, int c3) {
    asm volatile("cp.async.bulk.tensor.4d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(map),
                 "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
                 : "memory");
}
// Tensor copy (no multicast) of a 5-D box into shared memory, completing on an mbarrier
__device__ __forceinline__ void tma_load5(const CUtensorMap *map, uint32_t dst, uint32_t bar, int c0, int c1, int c2,
                                          int c3, int c4) {
    asm volatile(
        "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6, "
        "%7}], [%2];" ::"r"(dst),
        "l"(map), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4)
        : "memory");
}
__device__ __forceinline__ void bar_arrive_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void cp_async16(uint32_t sdst, const void *gsrc, int src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(sdst), "l"(gsrc), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_wait0() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void tc_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 columns of this warp's 32 tensor-memory lanes, waited for in the same statement
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ uint32_t pack2(float lo_elem, float hi_elem) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo_elem, hi_elem);
    return *reinterpret_cast<uint32_t *>(&v);
}
// 8 floats -> one 16-byte piece of high parts and one of low parts
__device__ __forceinline__ void split8(const float *v, uint4 &hi, uint4 &lo) {
    uint32_t h[4], l[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 hh = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
        h[i] = *reinterpret_cast<const uint32_t *>(&hh);
        l[i] = pack2(v[2 * i] - __low2float(hh), v[2 * i + 1] - __high2float(hh));
    }
    hi = make_uint4(h[0], h[1], h[2], h[3]);
    lo = make_uint4(l[0], l[1], l[2], l[3]);
}
__device__ __forceinline__ void unpack8(const uint4 &q, float *v) {
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

__device__ __forceinline__ int ld_acquire(const int *p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release(int *p, int v) {
    asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

template <typename TOut>
__global__ void __launch_bounds__(kThreads, 1) ssd_fwd_tc_kernel(const SsdArgs a, const SsdTcArgs w,
                                                                  const __grid_constant__ CUtensorMap ymap,
                                                                  const __grid_constant__ CUtensorMap cmap,
                                                                  const __grid_constant__ CUtensorMap bmap) {
    extern __shared__ __align__(1024) unsigned char smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t sbase = saddr(smem);
    auto bar = [&](int i) { return sbase + (uint32_t)(kOffBar + 8 * i); };
    auto sbar = [&](int slot, int e) { return bar(slot * kBarsPerSlot + e); };
    uint32_t *misc = reinterpret_cast<uint32_t *>(smem + kOffMisc);  // [0] tmem base, [2] abort
    volatile uint32_t *abort_flag = misc + 2;
    ItemDesc *desc = reinterpret_cast<ItemDesc *>(smem + kOffDesc);

    if (tid == 0) {
        misc[2] = 0u;
        for (int sl = 0; sl < 2; ++sl) {
            bar_init(sbar(sl, kBarXP), kGroupWarps);
            bar_init(sbar(sl, kBarCB), 1);
            bar_init(sbar(sl, kBarSC), 1);
            bar_init(sbar(sl, kBarG), kGroupWarps);
            bar_init(sbar(sl, kBarYI), 1);
            bar_init(sbar(sl, kBarS), kGroupWarps);
            bar_init(sbar(sl, kBarYS), 1);
        }
        for (int pb = 0; pb < 2; ++pb) {
            bar_init(bar(kBarParFull + pb), 1);
            bar_init(bar(kBarParFree + pb), kComputeWarps + 1);
        }
        for (int cb = 0; cb < 2; ++cb) {
            bar_init(bar(kBarCFull + cb), 1);
            bar_init(bar(kBarCFree + cb), 1);
        }
        bar_init(bar(kBarBFull), 1);
        bar_init(bar(kBarBFree), 1);
        bar_init(bar(kBarEnd), 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(sbase + kOffMisc),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_before();
    __syncthreads();
    tc_after();
    const uint32_t tmem = misc[0];

    const int64_t hpg = a.H / a.G;                       // heads per group
    const int64_t nhb = (hpg + w.hb - 1) / w.hb;         // head blocks per group
    const int64_t per_chunk = a.batch * a.G * nhb;
    const int64_t L = a.L;
    auto params = [&](int pb) { return reinterpret_cast<float *>(smem + kOffPar + pb * kParBytes); };

    if (warp == kProdWarp) {
        // ============================== producer warp ==============================
        // Claims items in ticket order (one ahead of the item it prepares), writes
        // each item's descriptor and per-head parameters into the free buffer, and
        // loads the item's C and B tiles once the previous item's products are done
        // with them. The next item is thus ready while the current one computes.
        bool ok = true;
        int tma_last = -1;  // the last item whose tiles came by tensor copies
        long long T = 0;
        // one C or B tile [128 tokens x 128 states] (rows past L zero-filled): a tensor copy
        // whose bytes the barrier counts, else 16-byte copies by the warp; the barrier is
        // arrived on either way (also when the CTA is stopping)
        auto load_tile = [&](bool go, const CUtensorMap *map, const __nv_bfloat16 *src, int64_t sl, uint32_t dst,
                             uint32_t br, int64_t t0, int64_t g, int64_t b) {
            if (go && w.cb_tma) {
                if (lane == 0) {
                    bar_arrive_tx(br, (uint32_t)kTileCB);
                    tma_load5(map, dst, br, 0, (int)t0, 0, (int)g, (int)b);
                }
                return;
            }
            if (go) {
                for (int i = lane; i < kQ * (kN / 8); i += 32) {
                    const int t = i >> 4, kc = i & 15;
                    const bool in = t0 + t < L;
                    cp_async16(dst + cb_off(t, kc), src + (in ? t0 + t : 0) * sl + 8 * kc, in ? 16 : 0);
                }
                cp_commit();
                cp_wait0();          // this lane's copies are in
                fence_async_smem();  // ... and visible to the tensor cores
            }
            __syncwarp();
            if (lane == 0) bar_arrive(br);
        };
        if (lane == 0) T = (long long)(unsigned)atomicAdd(w.counter, 1);
        T = __shfl_sync(0xffffffffu, T, 0);
        for (int it = 0;; ++it) {
            const int pb = it & 1;
            if (it >= 2) ok = bar_wait(bar(kBarParFree + pb), (uint32_t)(((it - 2) >> 1) & 1));
            ok = __all_sync(0xffffffffu, ok && *abort_flag == 0u);
            const int64_t k = T / per_chunk, r0 = T % per_chunk;
            const int64_t b = r0 / (a.G * nhb), g = (r0 / nhb) % a.G, hbk = r0 % nhb;
            const int64_t h0 = g * hpg + hbk * w.hb;
            // debug build: a ticket below the item count names a chunk of the sequence,
            // a batch row and a block of its group's heads (an item that fails is dropped)
            const bool valid = ok && T < w.items &&
                               MS_CHECK(a.status, k * kQ < L && b < a.batch && g < a.G && hbk * w.hb < hpg);
            const int64_t left = hpg - hbk * w.hb;
            const int nh = valid ? (int)(left < (int64_t)w.hb ? left : (int64_t)w.hb) : 0;
            const int64_t t0 = k * kQ;
            long long Tn = 0;
            if (valid && lane == 0) Tn = (long long)(unsigned)atomicAdd(w.counter, 1);
            if (valid) {
                // per head: Delta, cs log2(e) and w_s of the chunk's tokens, 4 tokens a lane
                float *dlp = params(pb), *cs2p = dlp + kHB * kQ, *wp = cs2p + kHB * kQ, *fdp = wp + kHB * kQ;
                const unsigned short *dtp = static_cast<const unsigned short *>(a.dt) + b * a.dt_sb + h0;
                unsigned short raw[kHB][4];
#pragma unroll
                for (int jj = 0; jj < kHB; ++jj)
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int64_t t = t0 + 4 * lane + i;
                        raw[jj][i] = (jj < nh && t < L) ? __ldg(dtp + t * a.dt_sl + jj) : (unsigned short)0;
                    }
#pragma unroll
                for (int jj = 0; jj < kHB; ++jj) {
                    if (jj < nh) {
                        const int64_t h = h0 + jj;
                        const float A2 = __ldg(a.A + h) * kLog2e;
                        const float bias = a.dt_bias ? __ldg(a.dt_bias + h) : 0.0f;
                        float dl[4], c = 0.0f;
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            float d = 0.0f;
                            if (t0 + 4 * lane + i < L) {
                                const float v = bf16_bits_to_f32(raw[jj][i]) + bias;
                                d = a.softplus ? softplus_f(v) : v;
                            }
                            dl[i] = d;
                            c += d;
                        }
                        // inclusive prefix of the lanes' sums
                        float incl = c;
#pragma unroll
                        for (int off = 1; off < 32; off <<= 1) {
                            const float o = __shfl_up_sync(0xffffffffu, incl, off);
                            if (lane >= off) incl += o;
                        }
                        float run = incl - c;  // sum before this lane's tokens
                        const float total = __shfl_sync(0xffffffffu, incl, 31);
                        const float cend = A2 * total;  // cs_{Q-1} log2(e): padded tokens add nothing
                        float c2[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            run += dl[i];
                            c2[i] = A2 * run;
                        }
                        // cs of the last token of this lane's 32-token block (lanes 8c..8c+7)
                        const float cblk = __shfl_sync(0xffffffffu, c2[3], lane | 7);
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int t = 4 * lane + i;
                            dlp[jj * kQ + t] = dl[i];
                            cs2p[jj * kQ + t] = c2[i];
                            wp[jj * kQ + t] = exp2_mufu(cend - c2[i]) * dl[i];
                            fdp[jj * kQ + t] = exp2_mufu(cblk - c2[i]) * dl[i];
                        }
                    }
                }
            }
            if (lane == 0) {
                ItemDesc d;
                d.k = k;
                d.b = b;
                d.g = g;
                d.h0 = h0;
                d.nh = nh;
                d.valid = valid ? 1 : 0;
                desc[pb] = d;
            }
            __syncwarp();
            if (lane == 0) bar_arrive(bar(kBarParFull + pb));
            if (!valid) break;
            // C into buffer it % 2 once item it - 2's products are done with it; B once
            // every product of item it - 1 that reads B has completed
            if (it >= 2) ok = bar_wait(bar(kBarCFree + pb), (uint32_t)(((it - 2) >> 1) & 1));
            ok = __all_sync(0xffffffffu, ok && *abort_flag == 0u);
            load_tile(ok, &cmap, static_cast<const __nv_bfloat16 *>(a.C) + b * a.C_sb + g * a.C_sg, a.C_sl,
                      sbase + (uint32_t)(kOffC + pb * kTileCB), bar(kBarCFull + pb), t0, g, b);
            if (ok && it >= 1) ok = bar_wait(bar(kBarBFree), (uint32_t)((it - 1) & 1));
            ok = __all_sync(0xffffffffu, ok && *abort_flag == 0u);
            load_tile(ok, &bmap, static_cast<const __nv_bfloat16 *>(a.B) + b * a.B_sb + g * a.B_sg, a.B_sl,
                      sbase + (uint32_t)kOffB, bar(kBarBFull), t0, g, b);
            if (ok && w.cb_tma) tma_last = it;
            if (!ok) break;
            T = __shfl_sync(0xffffffffu, Tn, 0);
        }
        if (!ok && lane == 0) {
            *abort_flag = 1u;
            if (a.status) atomicOr(a.status, MS_ERR_TIMEOUT);
        }
        // the last tensor copies have landed before the CTA can exit (bounded; at once
        // when the MMA warp has consumed them)
        if (tma_last >= 0 && lane == 0) {
            (void)bar_wait(bar(kBarBFull), (uint32_t)(tma_last & 1));
            for (int i = tma_last > 0 ? tma_last - 1 : 0; i <= tma_last; ++i)
                (void)bar_wait(bar(kBarCFull + (i & 1)), (uint32_t)((i >> 1) & 1));
        }
    } else if (warp == kMmaWarp) {
        // ================================ MMA warp ================================
        if (lane == 0) {
            const uint32_t sB = sbase + kOffB;
            auto sC = [&](int cb) { return sbase + (uint32_t)(kOffC + cb * kTileCB); };
            bool ok = true;
            // Each slot runs its own sequence of heads (s, s + 2, ... of every item) and
            // may enter the next item while the other finishes this one. Per slot: item,
            // head, step (-1: item's descriptor; 0: C B^T once the item's tiles are in;
            // 1: X' ready -> S_c; 2: G' ready -> Y_i; 3: S_in ready -> Y_s).
            int s_it[2] = {0, 0}, s_j[2] = {0, 1}, s_step[2] = {-1, -1};
            bool s_done[2] = {false, false};
            uint32_t used[2] = {0u, 0u};  // heads each slot has taken (barrier parities)
            // per item parity: the item read, its heads and validity, and the slots still to
            // issue their last S_c (the item's last B readers) and their last Y_s (C readers)
            int known[2] = {-1, -1}, inh[2] = {0, 0}, ivalid[2] = {0, 0}, sc_left[2] = {0, 0}, ys_left[2] = {0, 0};
            uint32_t idle = 0;
            // CB = C B^T (both K-major) into a slot's first 128 columns: issued behind the
            // slot's previous head's last product (products run in issue order, so that
            // head's G' has been read), so the group finds it ready
            auto issue_cb = [&](int sl, int cb) {
                const uint32_t tb = tmem + (uint32_t)sl * kSlotCols;
#pragma unroll 1
                for (int ks = 0; ks < kN / 16; ++ks)
                    mma(tb + kColCB, desc_k(sC(cb) + 4096u * ks, 2048u, 128u), desc_k(sB + 4096u * ks, 2048u, 128u),
                        idesc(kQ, false, false), ks > 0);
                mma_commit(sbar(sl, kBarCB));
            };
            while (ok && !(s_done[0] && s_done[1])) {
                bool progressed = false;
#pragma unroll
                for (int sl = 0; sl < 2; ++sl) {
                    if (s_done[sl]) continue;
                    const int it = s_it[sl], pb = it & 1;
                    if (s_step[sl] < 0) {
                        if (known[pb] != it) {
                            if (!bar_test(bar(kBarParFull + pb), (uint32_t)((it >> 1) & 1))) continue;
                            inh[pb] = desc[pb].nh;
                            ivalid[pb] = desc[pb].valid;
                            known[pb] = it;
                            sc_left[pb] = ys_left[pb] = inh[pb] < 2 ? inh[pb] : 2;
                            bar_arrive(bar(kBarParFree + pb));  // the descriptor is all this warp reads
                        }
                        if (!ivalid[pb]) {
                            s_done[sl] = true;
                        } else if (s_j[sl] >= inh[pb]) {
                            s_it[sl] = it + 1;  // no head of this item for the slot
                            s_j[sl] = sl;
                        } else {
                            s_step[sl] = 0;
                        }
                        progressed = true;
                        continue;
                    }
                    const int j = s_j[sl];
                    const uint32_t ph = used[sl] & 1u;
                    const uint32_t tb = tmem + (uint32_t)sl * kSlotCols;
                    const uint32_t sXP = sbase + (uint32_t)(kOffSlot + sl * kSlotBytes);
                    const uint32_t sX = sXP + (uint32_t)(2 * kTileHalf);
                    const bool last = j + 2 >= inh[pb];
                    if (s_step[sl] == 0) {
                        if (!bar_test(bar(kBarCFull + pb), (uint32_t)((it >> 1) & 1)) ||
                            !bar_test(bar(kBarBFull), (uint32_t)(it & 1)))
                            continue;
                        tc_after();
                        issue_cb(sl, pb);
                        s_step[sl] = 1;
                        progressed = true;
                        continue;
                    }
                    const int ev = s_step[sl] == 1 ? kBarXP : (s_step[sl] == 2 ? kBarG : kBarS);
                    if (!bar_test(sbar(sl, ev), ph)) continue;
                    tc_after();
                    if (s_step[sl] == 1) {
                        // S_c [n x p] = B^T X': A = the B tile read M(n)-major, B = X' (hi, lo)
#pragma unroll 1
                        for (int ks = 0; ks < kQ / 16; ++ks)
#pragma unroll
                            for (int part = 0; part < 2; ++part)
                                mma(tb + kColSC, desc_mn(sB + 256u * ks, 128u, 2048u),
                                    desc_mn(sXP + (uint32_t)(part * kTileHalf) + 2048u * ks, 1024u, 128u),
                                    idesc(kP, true, true), ks > 0 || part > 0);
                        mma_commit(sbar(sl, kBarSC));
                        // B is free once the item's last S_c of both slots has completed (each
                        // slot's C B^T products were issued before its S_c)
                        if (last && --sc_left[pb] == 0) mma_commit(bar(kBarBFree));
                        s_step[sl] = 2;
                    } else if (s_step[sl] == 2) {
                        // Y_i [t x p] = G' X: A = G' (hi, lo) packed in tensor memory, B = x
#pragma unroll 1
                        for (int ks = 0; ks < kQ / 16; ++ks)
#pragma unroll
                            for (int part = 0; part < 2; ++part)
                                mma_ts(tb + kColYI, tb + g_col(ks, part), desc_mn(sX + 2048u * ks, 1024u, 128u),
                                       idesc(kP, false, true), ks > 0 || part > 0);
                        mma_commit(sbar(sl, kBarYI));
                        s_step[sl] = 3;
                    } else {
                        // Y_s [t x p] = C S_in (hi, lo), into S_c's columns
#pragma unroll 1
                        for (int ks = 0; ks < kN / 16; ++ks)
#pragma unroll
                            for (int part = 0; part < 2; ++part)
                                mma(tb + kColSC, desc_k(sC(pb) + 4096u * ks, 2048u, 128u),
                                    desc_mn(sXP + (uint32_t)(part * kTileHalf) + 2048u * ks, 1024u, 128u),
                                    idesc(kP, false, true), ks > 0 || part > 0);
                        mma_commit(sbar(sl, kBarYS));
                        ++used[sl];
                        if (last) {
                            // C buffer pb is free once the item's last Y_s of both slots has completed
                            if (--ys_left[pb] == 0) mma_commit(bar(kBarCFree + pb));
                            s_it[sl] = it + 1;
                            s_j[sl] = sl;
                            s_step[sl] = -1;
                        } else {
                            s_j[sl] = j + 2;
                            s_step[sl] = 0;
                        }
                    }
                    progressed = true;
                }
                if (progressed) {
                    idle = 0;
                } else {
                    if (++idle > kIdleTries || *abort_flag != 0u) ok = false;
                    __nanosleep(MS_SSD_POLL_NS);  // leave the issue slots to the compute warps
                }
            }
            if (!ok) {
                *abort_flag = 1u;
                if (a.status) atomicOr(a.status, MS_ERR_TIMEOUT);
            }
            // every product issued above has completed before the tensor memory is freed
            mma_commit(bar(kBarEnd));
            (void)bar_wait(bar(kBarEnd), 0u);
        }
        __syncwarp();
    } else {
        // ============================== compute groups ==============================
        const int gi = warp / kGroupWarps, qd = warp % kGroupWarps;
        const int gtid = tid % kGroupThreads;
        const int gbar = 2 + gi;                                     // the group's named barrier
        const int row = 32 * qd + lane;                              // accumulator lane: token t or state n
        const uint32_t tb = tmem + (uint32_t)gi * kSlotCols + ((uint32_t)(32 * qd) << 16);
        unsigned char *XP = smem + kOffSlot + gi * kSlotBytes;       // X' hi / lo, later S_in hi / lo
        const unsigned char *X = XP + 2 * kTileHalf;                 // x of the group's current head
        bool ok = true, fin = false;
        bool x_ahead = false;  // x of the group's first head of the next item is requested
        uint32_t used = 0;     // heads this group has taken (barrier parities of its slot)

        // x of head j of item d: each thread copies its own token row, the only row
        // it reads (X' and D x); rows past L are zero-filled
        auto load_x = [&](const ItemDesc &d, int j) {
            const int64_t ts = d.k * kQ + row;
            const bool in = ts < L && MS_CHECK(a.status, ts >= 0 && d.b < a.batch && d.h0 + j < a.H);
            const __nv_bfloat16 *src =
                static_cast<const __nv_bfloat16 *>(a.x) + d.b * a.x_sb + (d.h0 + j) * a.x_sh + (in ? ts : 0) * a.x_sl;
            const uint32_t dst = saddr(X);
#pragma unroll
            for (int pc = 0; pc < 8; ++pc) cp_async16(dst + mn64_off(row, pc), src + 8 * pc, in ? 16 : 0);
            cp_commit();
        };

        for (int it = 0;; ++it) {
            const int pb = it & 1;
            const bool got = ok && bar_wait(bar(kBarParFull + pb), (uint32_t)((it >> 1) & 1));
            // the group agrees before anything it does together
            ok = sync_and<kGroupThreads>(gbar, ok && got && *abort_flag == 0u);
            if (!ok) break;
            const ItemDesc &d = desc[pb];
            if (!d.valid) {
                fin = true;
                break;
            }
            const int nh = d.nh;
            const int64_t k = d.k, b = d.b, t0 = k * kQ;
            const float *dlp = params(pb), *cs2p = dlp + kHB * kQ, *wp = cs2p + kHB * kQ, *fdp = wp + kHB * kQ;
            if (gi < nh && !x_ahead) load_x(d, gi);
            x_ahead = false;

            for (int j = gi; j < nh; j += 2, ++used) {
                const uint32_t ph = used & 1u;
                const int64_t h = d.h0 + j;
                const float *cs2 = cs2p + j * kQ;
                cp_wait0();  // x of head j is in
                fence_async_smem();
                if (gtid == 0 && w.y_tma) bulk_wait_read0();  // the previous head's y has left the staging buffer
                ok = sync_and<kGroupThreads>(gbar, ok && *abort_flag == 0u);
                if (!ok) break;
                // ---- X' = w_s x_s (row s, all 64 columns p), hi / lo
                {
                    const int s = row;
                    const float ws = wp[j * kQ + s];
#pragma unroll
                    for (int pc = 0; pc < 8; ++pc) {
                        float v[8];
                        unpack8(*reinterpret_cast<const uint4 *>(X + mn64_off(s, pc)), v);
#pragma unroll
                        for (int e = 0; e < 8; ++e) v[e] *= ws;
                        uint4 hi, lo;
                        split8(v, hi, lo);
                        *reinterpret_cast<uint4 *>(XP + mn64_off(s, pc)) = hi;
                        *reinterpret_cast<uint4 *>(XP + kTileHalf + mn64_off(s, pc)) = lo;
                    }
                }
                fence_async_smem();
                __syncwarp();
                if (lane == 0) bar_arrive(sbar(gi, kBarXP));
                // ---- G'[t][s] = CB[t][s] exp(cs_t - cs_s) Delta_s for s <= t, hi / lo packed
                // in place of CB, one 32-column block at a time; blocks entirely above
                // the diagonal are zeros
                ok = __all_sync(0xffffffffu, ok && bar_wait(sbar(gi, kBarCB), ph));
                tc_after();
                {
                    const int t = row;
                    const float ct = cs2[t];
                    const float *dls = dlp + j * kQ;
                    const float *fds = fdp + j * kQ;
#pragma unroll 1
                    for (int c = 0; c < 4; ++c) {
                        uint32_t hi[16], lo[16];
                        if (c <= qd && ok) {
                            float v[32];
                            tmem_ld32(tb + kColCB + (uint32_t)(32 * c), v);
                            if (c < qd) {
                                // block below the diagonal: exp(cs_t - cs_s) = exp(cs_t - m) exp(m - cs_s),
                                // m = cs of the block's last token, both factors <= 1
                                const float et = exp2_mufu(ct - cs2[32 * c + 31]);
#pragma unroll
                                for (int e = 0; e < 32; ++e) v[e] = (v[e] * et) * fds[32 * c + e];
                            } else {
#pragma unroll
                                for (int e = 0; e < 32; ++e) {
                                    const int s = 32 * c + e;
                                    v[e] = s <= t ? v[e] * exp2_mufu(ct - cs2[s]) * dls[s] : 0.0f;
                                }
                            }
#pragma unroll
                            for (int e = 0; e < 16; ++e) {
                                const __nv_bfloat162 hh = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
                                hi[e] = *reinterpret_cast<const uint32_t *>(&hh);
                                lo[e] = pack2(v[2 * e] - __low2float(hh), v[2 * e + 1] - __high2float(hh));
                            }
                        } else {
#pragma unroll
                            for (int e = 0; e < 16; ++e) hi[e] = lo[e] = 0u;
                        }
                        tmem_st16(tb + kColCB + (uint32_t)(32 * c), hi);
                        tmem_st16(tb + kColCB + (uint32_t)(32 * c + 16), lo);
                    }
                }
                tmem_st_wait();
                tc_before();
                __syncwarp();
                if (lane == 0) bar_arrive(sbar(gi, kBarG));

                // ---- S_out = decay S_in + S_c; S_in (hi, lo) for Y_s; publish S_out. The
                // running state is [p / 4][n][4] per head in the workspace (a warp's 16-byte
                // loads of one p-quad are contiguous); the first chunk reads
                // initial_state [p][n], the last one also writes final_state [p][n]. S_in
                // (once chunk k - 1 has published it) is loaded before the wait for S_c,
                // so its trip through L2 overlaps the product.
                {
                    int *flag = w.flags + (b * a.H + h);
                    if (k > 0 && ok) {
                        uint32_t i = 0;
                        while (ld_acquire(flag) < (int)k && i < kFlagTries) {
                            __nanosleep(32);
                            ++i;
                        }
                        ok = i < kFlagTries;
                    }
                    ok = __all_sync(0xffffffffu, ok);
                    const int n = row;
                    const size_t blk = (size_t)(b * a.H + h) * kP * kN;
                    float4 *run4 = reinterpret_cast<float4 *>(w.state + blk) + n;  // quad q at run4[q * kN]
                    // every S_in load of the row issued before any S_out store
                    float sv[64];
                    if (ok && k > 0) {
#pragma unroll
                        for (int q = 0; q < 16; ++q) {
                            const float4 v4 = run4[q * kN];
                            sv[4 * q] = v4.x; sv[4 * q + 1] = v4.y; sv[4 * q + 2] = v4.z; sv[4 * q + 3] = v4.w;
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 64; ++e) sv[e] = (ok && a.s0) ? a.s0[blk + (size_t)e * kN + n] : 0.0f;
                    }
                    ok = __all_sync(0xffffffffu, ok && bar_wait(sbar(gi, kBarSC), ph));
                    tc_after();
                    const float decay = exp2_mufu(cs2[kQ - 1]);
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        if (ok) {
                            float sc[32];
                            tmem_ld32(tb + kColSC + (uint32_t)(32 * half), sc);
                            float so[32];
#pragma unroll
                            for (int e = 0; e < 32; ++e) so[e] = fmaf(decay, sv[32 * half + e], sc[e]);
#pragma unroll
                            for (int q = 0; q < 8; ++q)
                                run4[(8 * half + q) * kN] = make_float4(so[4 * q], so[4 * q + 1], so[4 * q + 2], so[4 * q + 3]);
                            if (w.last_chunk == k && a.s_last != nullptr) {
#pragma unroll
                                for (int e = 0; e < 32; ++e) a.s_last[blk + (size_t)(32 * half + e) * kN + n] = so[e];
                            }
                        }
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            uint4 hi, lo;
                            split8(sv + 32 * half + 8 * q, hi, lo);
                            const int pc = 4 * half + q;
                            *reinterpret_cast<uint4 *>(XP + mn64_off(n, pc)) = hi;
                            *reinterpret_cast<uint4 *>(XP + kTileHalf + mn64_off(n, pc)) = lo;
                        }
                    }
                    fence_async_smem();
                    tc_before();
                    // this warp has read its S_c rows and written its S_in rows: Y_s may
                    // overwrite the one and read the other once every warp is here
                    __syncwarp();
                    if (lane == 0) bar_arrive(sbar(gi, kBarS));
                    // the group's S_out is stored: publish it for chunk k + 1 (the release
                    // orders the group's stores, which the barrier put before it)
                    ok = sync_and<kGroupThreads>(gbar, ok);
                    if (gtid == 0 && ok) st_release(flag, (int)k + 1);
                }
                if (!ok) break;

                // ---- y_t = exp(cs_t) Y_s[t] + Y_i[t] + D x_t (row t, all 64 columns p): Y_i and
                // D x first, while Y_s is still being formed
                ok = __all_sync(0xffffffffu, ok && bar_wait(sbar(gi, kBarYI), ph));
                tc_after();
                if (ok) {
                    const int t = row;
                    const float et = exp2_mufu(cs2[t]);
                    const float Dh = a.D ? __ldg(a.D + h) : 0.0f;
                    TOut *yp = static_cast<TOut *>(a.y) + b * a.y_sb + (t0 + t) * a.y_sl + h * a.y_sh;
                    float yi[64];
                    tmem_ld32(tb + kColYI, *reinterpret_cast<float(*)[32]>(yi));
                    tmem_ld32(tb + kColYI + 32u, *reinterpret_cast<float(*)[32]>(yi + 32));
#pragma unroll
                    for (int pc = 0; pc < 8; ++pc) {
                        float xv[8];
                        unpack8(*reinterpret_cast<const uint4 *>(X + mn64_off(t, pc)), xv);
#pragma unroll
                        for (int e = 0; e < 8; ++e) yi[8 * pc + e] = fmaf(Dh, xv[e], yi[8 * pc + e]);
                    }
                    // this thread is done with its x row and Y_i has read the tile: the row
                    // takes the group's next head, in this item or (once its descriptor is
                    // in) the next item's first, while Y_s completes
                    if (j + 2 < nh) {
                        load_x(d, j + 2);
                    } else {
                        const bool gn = bar_wait(bar(kBarParFull + (pb ^ 1)), (uint32_t)(((it + 1) >> 1) & 1));
                        ok = ok && gn;
                        if (gn) {
                            const ItemDesc &dn = desc[pb ^ 1];
                            if (dn.valid && gi < dn.nh) {
                                load_x(dn, gi);
                                x_ahead = true;
                            }
                        }
                    }
                    ok = __all_sync(0xffffffffu, ok && bar_wait(sbar(gi, kBarYS), ph));
                    tc_after();
                    if (w.y_tma) {
                        // y row t into the staging buffer (S_in has been consumed by Y_s) in the
                        // tensor map's box layout: rows of 128 bytes, 16-byte chunk i of row t
                        // at chunk i ^ (t % 8) (128-byte swizzle); fp32: two boxes of 32
                        // columns, bf16: one box of 64
#pragma unroll
                        for (int half = 0; half < 2 && ok; ++half) {
                            float ys[32];
                            tmem_ld32(tb + kColSC + (uint32_t)(32 * half), ys);
#pragma unroll
                            for (int e = 0; e < 32; ++e) yi[32 * half + e] = fmaf(et, ys[e], yi[32 * half + e]);
                        }
                        if constexpr (sizeof(TOut) == 4) {
#pragma unroll
                            for (int c = 0; c < 2; ++c)
#pragma unroll
                                for (int i = 0; i < 8; ++i)
                                    *reinterpret_cast<float4 *>(XP + c * kTileHalf + t * 128 + ((i ^ (t & 7)) << 4)) =
                                        make_float4(yi[32 * c + 4 * i], yi[32 * c + 4 * i + 1], yi[32 * c + 4 * i + 2],
                                                    yi[32 * c + 4 * i + 3]);
                        } else {
#pragma unroll
                            for (int i = 0; i < 8; ++i)
                                *reinterpret_cast<uint4 *>(XP + t * 128 + ((i ^ (t & 7)) << 4)) =
                                    make_uint4(pack2(yi[8 * i], yi[8 * i + 1]), pack2(yi[8 * i + 2], yi[8 * i + 3]),
                                               pack2(yi[8 * i + 4], yi[8 * i + 5]), pack2(yi[8 * i + 6], yi[8 * i + 7]));
                        }
                        fence_async_smem();
                    } else {
#pragma unroll
                        for (int half = 0; half < 2 && ok; ++half) {
                            float ys[32];
                            tmem_ld32(tb + kColSC + (uint32_t)(32 * half), ys);
                            if (t0 + t < L && MS_CHECK(a.status, b < a.batch && h < a.H)) {
#pragma unroll
                                for (int q = 0; q < 4; ++q) {
                                    float yo[8];
#pragma unroll
                                    for (int e = 0; e < 8; ++e) yo[e] = fmaf(et, ys[8 * q + e], yi[32 * half + 8 * q + e]);
                                    TOut *yq = yp + 32 * half + 8 * q;
                                    if constexpr (sizeof(TOut) == 4) {
                                        if (w.y_vec16) {
                                            float4 *p4 = reinterpret_cast<float4 *>(yq);
                                            p4[0] = make_float4(yo[0], yo[1], yo[2], yo[3]);
                                            p4[1] = make_float4(yo[4], yo[5], yo[6], yo[7]);
                                        } else {
                                            float2 *p2 = reinterpret_cast<float2 *>(yq);
#pragma unroll
                                            for (int e = 0; e < 4; ++e) p2[e] = make_float2(yo[2 * e], yo[2 * e + 1]);
                                        }
                                    } else {
                                        if (w.y_vec16) {
                                            *reinterpret_cast<uint4 *>(yq) = make_uint4(pack2(yo[0], yo[1]), pack2(yo[2], yo[3]),
                                                                                        pack2(yo[4], yo[5]), pack2(yo[6], yo[7]));
                                        } else {
                                            uint32_t *p1 = reinterpret_cast<uint32_t *>(yq);
#pragma unroll
                                            for (int e = 0; e < 4; ++e) p1[e] = pack2(yo[2 * e], yo[2 * e + 1]);
                                        }
                                    }
                                }
                            }
                        }
                    }
                    }
                if (w.y_tma) {
                    // every thread of the group has staged its row (or given up): one thread
                    // stores the tile (rows past the sequence are outside the map, not written)
                    ok = sync_and<kGroupThreads>(gbar, ok);
                    if (gtid == 0 && ok) {
                        if constexpr (sizeof(TOut) == 4) {
                            tma_store4(&ymap, saddr(XP), 0, (int)h, (int)t0, (int)b);
                            tma_store4(&ymap, saddr(XP) + kTileHalf, 32, (int)h, (int)t0, (int)b);
                        } else {
                            tma_store4(&ymap, saddr(XP), 0, (int)h, (int)t0, (int)b);
                        }
                        bulk_commit();
                    }
                }
                tc_before();
                ok = sync_and<kGroupThreads>(gbar, ok && *abort_flag == 0u);
                if (!ok) break;
            }
            // every warp of the group is done with this item's parameters and descriptor
            __syncwarp();
            if (lane == 0) bar_arrive(bar(kBarParFree + pb));
        }
        if (!fin && gtid == 0) {
            *abort_flag = 1u;
            if (a.status) atomicOr(a.status, MS_ERR_TIMEOUT);
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
        if (gtid == 0 && w.y_tma) bulk_wait0();
    }

    // ---- tear-down: the MMA warp has drained its products; free the tensor memory
    tc_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                     : "memory");
    }
}

template <typename TOut>
cudaError_t launch_t(const SsdArgs &a, const SsdTcArgs &w, const CUtensorMap &ymap, const CUtensorMap &cmap,
                     const CUtensorMap &bmap, int64_t items, int num_sms, cudaStream_t stream) {
    static SmemOptIn opt_in;
    cudaError_t e = opt_in.ensure(reinterpret_cast<const void *>(ssd_fwd_tc_kernel<TOut>), kSmemBytes);
    if (e != cudaSuccess) return e;
    // persistent: one CTA per SM (the shared memory allows no second), items claimed in ticket order
    const int64_t grid = (num_sms > 0 && items > (int64_t)num_sms) ? (int64_t)num_sms : items;
    ssd_fwd_tc_kernel<TOut><<<(unsigned)grid, kThreads, kSmemBytes, stream>>>(a, w, ymap, cmap, bmap);
    return cudaGetLastError();
}

using PfnEncodeTiled = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                    const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                    CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
PfnEncodeTiled encode_fn() {
    static std::once_flag once;
    static PfnEncodeTiled fn = nullptr;
    std::call_once(once, [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PfnEncodeTiled>(f);
        cudaGetLastError();
    });
    return fn;
}

// y [batch][L][H][64] as a 4-D map {p, h, t, b}: box {128 bytes of p, 1 head,
// 128 tokens, 1 row}, 128-byte swizzle; rows t >= L lie outside the map.
bool encode_y(CUtensorMap *m, const SsdArgs &a, bool bf16) {
    PfnEncodeTiled fn = encode_fn();
    if (!fn) return false;
    const uint64_t es = bf16 ? 2 : 4;
    const uint64_t sh = (uint64_t)a.y_sh * es, sl = (uint64_t)a.y_sl * es;
    const uint64_t sb = a.batch > 1 ? (uint64_t)a.y_sb * es : sl * (uint64_t)a.L;
    if (sh == 0 || sl == 0 || sb == 0) return false;
    const cuuint64_t dims[4] = {(cuuint64_t)kP, (cuuint64_t)a.H, (cuuint64_t)a.L, (cuuint64_t)a.batch};
    const cuuint64_t strides[3] = {(cuuint64_t)sh, (cuuint64_t)sl, (cuuint64_t)sb};
    const cuuint32_t box[4] = {(cuuint32_t)(128 / es), 1u, (cuuint32_t)kQ, 1u};
    const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
    return fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, a.y, dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// B or C [batch][L][G][128] bf16 as a 5-D map {8 states, t, 16 state chunks, g, b}
// (the row's 128 states split into chunk and element, chunk outside t): the box
// {8, 128, 16, 1, 1} lands as [n / 8][t][n % 8]; rows t >= L lie outside the map
// and read as zeros.
bool encode_cb(CUtensorMap *m, const void *base, int64_t sb, int64_t sl, int64_t sg, const SsdArgs &a) {
    PfnEncodeTiled fn = encode_fn();
    if (!fn || reinterpret_cast<uintptr_t>(base) % 16 != 0) return false;
    const uint64_t bsl = (uint64_t)sl * 2;
    const uint64_t bsg = a.G > 1 ? (uint64_t)sg * 2 : 16;
    const uint64_t bsb = a.batch > 1 ? (uint64_t)sb * 2 : 16;
    if (bsl == 0 || bsl % 16 != 0 || bsg == 0 || bsg % 16 != 0 || bsb == 0 || bsb % 16 != 0) return false;
    const cuuint64_t dims[5] = {8u, (cuuint64_t)a.L, (cuuint64_t)(kN / 8), (cuuint64_t)a.G, (cuuint64_t)a.batch};
    const cuuint64_t strides[4] = {(cuuint64_t)bsl, 16u, (cuuint64_t)bsg, (cuuint64_t)bsb};
    const cuuint32_t box[5] = {8u, (cuuint32_t)kQ, (cuuint32_t)(kN / 8), 1u, 1u};
    const cuuint32_t estr[5] = {1u, 1u, 1u, 1u, 1u};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool ssd_shape_supported(int64_t headdim, int64_t dstate) { return headdim == kP && dstate == kN; }

int ssd_tc_head_block(int64_t batch, int64_t seqlen, int64_t nheads, int64_t ngroups, int num_sms) {
    // time ~ waves x (item start + head steps of the busier group), a head step
    // costing about 2.3 item starts (measured on the 2.7B-class layer)
    const int64_t hpg = nheads / ngroups, nch = (seqlen + kQ - 1) / kQ;
    int best = 1;
    double best_cost = 1e300;
    for (int hb = kHB; hb >= 1; --hb) {
        const int64_t items = nch * batch * ngroups * ((hpg + hb - 1) / hb);
        const int64_t waves = (items + num_sms - 1) / num_sms;
        const int steps = (int)((std::min<int64_t>(hb, hpg) + 1) / 2);
        const double cost = (double)waves * (1.0 + 2.3 * steps);
        if (cost < best_cost - 1e-9) {
            best_cost = cost;
            best = hb;
        }
    }
    return best;
}

size_t ssd_tc_workspace_size(int64_t batch, int64_t nheads) {
    const size_t flags = ((size_t)batch * (size_t)nheads + 1) * sizeof(int);
    const size_t flags_al = (flags + 255) / 256 * 256;
    return flags_al + (size_t)batch * nheads * kP * kN * sizeof(float);
}

cudaError_t launch_ssd_fwd_tc(const SsdArgs &a, bool out_bf16, void *workspace, int num_sms, cudaStream_t stream) {
    const int64_t nch = (a.L + kQ - 1) / kQ;
    if (a.batch <= 0 || nch <= 0) return cudaSuccess;
    SsdTcArgs w{};
    w.hb = ssd_tc_head_block(a.batch, a.L, a.H, a.G, num_sms);
    const int64_t hpg = a.H / a.G;
    const int64_t items = nch * a.batch * a.G * ((hpg + w.hb - 1) / w.hb);
    if (items > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    const size_t flags = ((size_t)a.batch * (size_t)a.H + 1) * sizeof(int);
    const size_t flags_al = (flags + 255) / 256 * 256;
    w.flags = static_cast<int *>(workspace);
    w.counter = w.flags + a.batch * a.H;
    w.state = reinterpret_cast<float *>(static_cast<unsigned char *>(workspace) + flags_al);
    w.last_chunk = nch - 1;
    w.items = items;
    const size_t ysz = out_bf16 ? 2 : 4;
    w.y_vec16 = ((reinterpret_cast<uintptr_t>(a.y) % 16) == 0 && (a.y_sb * ysz) % 16 == 0 && (a.y_sl * ysz) % 16 == 0 &&
                 (a.y_sh * ysz) % 16 == 0)
                    ? 1
                    : 0;
    CUtensorMap ymap;
    memset(&ymap, 0, sizeof(ymap));
    w.y_tma = (w.y_vec16 && a.H <= 0x7fffffff && a.L <= 0x7fffffff && a.batch <= 0x7fffffff &&
               encode_y(&ymap, a, out_bf16))
                  ? 1
                  : 0;
    CUtensorMap cmap, bmap;
    memset(&cmap, 0, sizeof(cmap));
    memset(&bmap, 0, sizeof(bmap));
    w.cb_tma = (a.L <= 0x7fffffff && a.batch <= 0x7fffffff && a.G <= 0x7fffffff &&
                encode_cb(&cmap, a.C, a.C_sb, a.C_sl, a.C_sg, a) && encode_cb(&bmap, a.B, a.B_sb, a.B_sl, a.B_sg, a))
                   ? 1
                   : 0;
    cudaError_t e = cudaMemsetAsync(workspace, 0, flags, stream);
    if (e != cudaSuccess) return e;
    return out_bf16 ? launch_t<__nv_bfloat16>(a, w, ymap, cmap, bmap, items, num_sms, stream)
                    : launch_t<float>(a, w, ymap, cmap, bmap, items, num_sms, stream);
}

}  // namespace ms
