// scan_fwd_tmem.cu -- selective scan forward on sm_100a with the token tiles
// streamed by the TMA engine and B/C broadcast through tensor memory.
//
// Same operation as scan_fwd.cu: per (batch b, channel d), Delta_t =
// softplus(delta_t + bias_d), A_bar = exp(Delta_t A[d,n]) ('Mamba (deep
// learning)' wiki page, state-space paragraph), h_t = A_bar h_{t-1} + Delta_t
// B_t u_t, y_t = C_t . h_t ('Mamba-1/2/3 Markdown図解' blog, section 1), plus
// D u_t inside the silu(z_t) gate (blog, section 2). The state stays in
// registers for the whole sequence (blog, section 2: the fused scan keeps the
// expanded state on chip).
//
// Why this variant. Per channel-token the recurrence needs the 16 B and 16 C
// values of the token in the lanes that own the states. Read from shared
// memory that is 32 words per channel-token, and shared memory delivers 32
// words per clock per SM: as costly as the 16 exponentials on the MUFU pipe.
// Tensor memory reads (tcgen05.ld) deliver about three times as many words
// per clock. The tensor cores put the values there: one tcgen05.mma per tile
// multiplies a fixed 0/1 selection matrix S [128 x 16] by the tile's B/C
// values, so that accumulator lane m holds the B/C values of state group
// m % 4 for every token (the tensor cores do the 32-fold replication).
//
// Work split (G = 4 lanes per channel): lane (c, g) of a warp owns states
// 4g..4g+3 of channel c (8 channels per warp). A CTA is one batch row and
// 8W consecutive channels: W compute warps plus one producer warp. Tokens go
// in tiles of 32:
//   producer  lane 0 issues the tile's TMA loads (u, delta, z boxes of
//             [8W channels x 32 tokens], B and C boxes of [16 x 32]) into a
//             ring of stages (mbarrier per stage, several tiles ahead). The
//             warp then rearranges the tile's B/C into the MMA operand V
//             [256 x 16] (row 8t + v, column k = group: v < 4 -> B[4k+v][t],
//             else C[4k+v-4][t]; for fp32 inputs the value is split into three
//             bf16 parts in columns k, 4 + k, 8 + k), and lane 0 issues
//             D[128 x 256] = S x V^T into one of two tensor-memory buffers,
//             committed to an mbarrier.
//   compute   lane (c, g) takes the 8-token chunk g of its channel from the
//             stage (u, delta, z), computes Delta, Delta*u, silu(z), D*u*silu(z)
//             once per token and passes Delta and Delta*u to the channel's 4
//             lanes through shared memory. Per 4 tokens one tcgen05.ld
//             (32x32b.x32) gives the lane its 4 B and 4 C values of 4 tokens;
//             A_bar by exp2 (MUFU, or a fixed share on the FMA-pipe
//             polynomial), h = A_bar h + (Delta u) B and the partial readout
//             C . h run on packed f32x2 pairs. The 4 partial readouts of a
//             token are summed through shared memory; lane (c, g) adds D u,
//             multiplies by silu(z) and stores its 8 tokens of y.
// Every mbarrier wait is bounded: on a timeout the CTA records MS_ERR_TIMEOUT
// in the caller's status word, stops issuing work, drains what it has in
// flight (bounded) and frees its tensor memory.

#include <cuda.h>

#include <cstdint>
#include <mutex>

#include "mambascan.h"
#include "ms_device.cuh"
#include "ms_internal.h"

namespace ms {

namespace {

constexpr int kT = 32;                 // tokens per tile
// Instantiations by compute warps per CTA: the block's warps spread over the
// SM's four schedulers, each with a quarter of the register file, so 12
// warps leave 168 registers a thread, 16 warps 128 and 19 warps 96.
constexpr int kMaxWSmall = 11;
constexpr int kMaxWMid = 15;
constexpr int kMaxWLarge = 18;
constexpr int kCW = 8;                 // channels per compute warp (4 lanes each)
constexpr int kRow = 36;               // floats per padded exchange row (bank spread)
constexpr int kRowS = 4 * 32 + 4;      // floats per padded row of splatted pairs
constexpr int kTmemCols = 512;         // two buffers of 256 columns
constexpr int kBufCols = 256;          // 32 tokens x 8 values
// Compile-time variants (measured; the defaults are the faster ones):
//   MS_TMEM_SPLAT    1: Delta / Delta*u stored as splatted pairs (one 16-byte
//                    load per token gives both f32x2 operands) in the 12-warp
//                    variant; 0: plain rows, pairs formed in registers.
//   MS_TMEM_SUSPEND  1: bounded waits pass a suspend-time hint to try_wait.
//   MS_TMEM_MMA_FIRST 1: the producer issues a tile's product before the next
//                    tile's loads; 0: loads first.
#ifndef MS_TMEM_SPLAT
#define MS_TMEM_SPLAT 0
#endif
#ifndef MS_TMEM_SUSPEND
#define MS_TMEM_SUSPEND 0
#endif
#ifndef MS_TMEM_MMA_FIRST
#define MS_TMEM_MMA_FIRST 0
#endif
//   MS_TMEM_SCALAR   1: the state loop in scalar fp32 (no register pairs to
//                    form from the tensor-memory loads, no Delta splats);
//                    0: packed f32x2 pairs.
#ifndef MS_TMEM_SCALAR
#define MS_TMEM_SCALAR 0
#endif
//   MS_TMEM_DB       1: the next group's tensor-memory load in flight while a
//                    group computes (4-token loads in the 12-warp variant,
//                    2-token loads in the larger ones); 0: one 4-token load
//                    per group, waited for at once.
#ifndef MS_TMEM_DB
#define MS_TMEM_DB 0
#endif
//   MS_TMEM_FUSED    1: in the 12-warp variant, the next tile's per-token
//                    quantities (Delta, Delta*u, silu(z), D*u*silu(z)) are
//                    computed inside the current tile's state loop, one
//                    token of the lane's chunk per group of 4 tokens, so
//                    their chains interleave with the recurrence and the
//                    MUFU work is spread over the tile; 0: a separate
//                    prologue per tile.
#ifndef MS_TMEM_FUSED
#define MS_TMEM_FUSED 0
#endif
//   MS_TMEM_UNROLL   groups of 4 tokens unrolled together in the state loop
//                    of the kernels that write y (8 = the whole tile in one
//                    basic block); the y-less pass keeps the loop rolled.
#ifndef MS_TMEM_UNROLL
#define MS_TMEM_UNROLL 8
#endif
//   MS_TMEM_LD64     1: in the 12-warp variant that writes y, one 64-column
//                    load (two groups of 4 tokens) per wait; 0: one 32-column
//                    load per group.
#ifndef MS_TMEM_LD64
#define MS_TMEM_LD64 1
#endif
//   MS_TMEM_LDCLOB   1: the combined load-and-wait is a compiler memory
//                    barrier; 0: it only defines its registers (shared
//                    loads of later groups may move above it).
//   MS_TMEM_SERIES   1: with every exponential on the FMA pipe (poly8 = 8),
//                    a token (or a whole tile) whose exponents |Delta A| are
//                    all <= 1/2 on every lane of the warp takes its decays
//                    from the expm1 series; 0: the polynomial throughout. On
//                    the long-context layer few tiles qualify and the
//                    per-token vote costs more than the series saves.
#ifndef MS_TMEM_SERIES
#define MS_TMEM_SERIES 0
#endif
#ifndef MS_TMEM_LDCLOB
#define MS_TMEM_LDCLOB 1
#endif
#if MS_TMEM_LDCLOB
#define MS_TMEM_LD_CLOBBER : "memory"
#else
#define MS_TMEM_LD_CLOBBER
#endif
constexpr int kUnrollGroups = MS_TMEM_UNROLL;

// Bounded waits: kSpin tries of mbarrier.try_wait (each may suspend the
// thread for a system-dependent time, or up to kSuspendNs with the hint).
constexpr uint32_t kSuspendNs = 20000;
constexpr uint32_t kSpin = MS_TMEM_SUSPEND ? (1u << 15) : (1u << 20);

// Shared memory layout for W compute warps and S stages (host and device).
struct TmLayout {
    int W, S, in_bytes;
    __host__ __device__ int cwc() const { return kCW * W; }
    // offset 0: mbarriers full[S], empty[S], mma[2], tfree[2], then two words
    __host__ __device__ int tmem_slot() const { return 8 * (2 * S + 4); }
    __host__ __device__ int abort_slot() const { return tmem_slot() + 4; }
    __host__ __device__ int asel() const { return 1024; }              // S: 128 rows x 32 bytes
    __host__ __device__ int op(int b) const { return 1024 + 4096 + b * 8192; }  // V: 256 rows x 32 bytes
    __host__ __device__ int chan_tile() const { return cwc() * kT * in_bytes; }
    __host__ __device__ int bc_tile() const { return 16 * kT * in_bytes; }
    __host__ __device__ int stage_bytes() const { return 3 * chan_tile() + 2 * bc_tile(); }
    __host__ __device__ int stage(int s) const { return 1024 + 4096 + 2 * 8192 + s * stage_bytes(); }
    // per-warp exchange: Delta and Delta*u (as splatted pairs (Delta, Delta,
    // Delta*u, Delta*u) per token in the 12-warp instantiation, else two
    // plain rows), then the partial readouts [8 channels x 4 lanes][kRow]
    __host__ __device__ bool splat() const { return MS_TMEM_SPLAT && !MS_TMEM_SCALAR && W <= 11; }
    __host__ __device__ int xch_bytes() const {
        return ((splat() ? kCW * kRowS : 2 * kCW * kRow) + kCW * 4 * kRow) * 4;
    }
    __host__ __device__ int xch(int w) const { return stage(S) + w * xch_bytes(); }
    __host__ __device__ int total() const { return xch(W); }
};

struct TmMaps {
    CUtensorMap u, dl, z, B, C;
};

__device__ __forceinline__ uint32_t sa(const void *p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }

__device__ __forceinline__ void bar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void bar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void bar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool bar_wait(uint32_t bar, uint32_t parity) {
    for (uint32_t i = 0; i < kSpin; ++i) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
#if MS_TMEM_SUSPEND
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
#else
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
#endif
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(bar), "r"(parity), "r"(kSuspendNs)
            : "memory");
        if (done) return true;
    }
    return false;
}

// 3-D tiled TMA load (no multicast) of box {x, y, 1} at coordinates (x, y, z).
__device__ __forceinline__ void tma_load3(uint32_t dst, const CUtensorMap *map, int x, int y, int z, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
        "[%5];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
        : "memory");
}

// Shared-memory matrix descriptor (K-major, no swizzle): start address,
// leading byte offset (the two 8-element K core matrices), stride byte offset
// (8-row groups), in 16-byte units; descriptor version 1.
__device__ __forceinline__ uint64_t mat_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}

// kind::f16 instruction descriptor: fp32 accumulator, bf16 A and B, both
// K-major, N = 256 (N >> 3 at bit 17), M = 128 (M >> 4 at bit 24).
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(256 >> 3) << 17) |
                            ((uint32_t)(128 >> 4) << 24);

// Byte offset of row r (16-byte piece kc of K) in a K-major no-swizzle tile
// with 16 K elements: core matrix (r / 8, kc) at ((r / 8) * 2 + kc) * 128.
__device__ __forceinline__ int op_off(int r, int kc) { return (((r >> 3) * 2 + kc) * 8 + (r & 7)) * 16; }

// 32 consecutive tensor-memory columns, loaded and waited for in one asm
// statement: where registers are short (the larger instantiations spill a
// few values) nothing can be spilled while the load is still in flight.
__device__ __forceinline__ void tmem_ld32_sync(uint32_t taddr, uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
          "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
          "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr) MS_TMEM_LD_CLOBBER);
}

// 64 consecutive tensor-memory columns of this warp's 32 lanes, waited for in
// the same statement.
__device__ __forceinline__ void tmem_ld64_sync(uint32_t taddr, uint32_t (&v)[64]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%64];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31]), "=r"(v[32]), "=r"(v[33]), "=r"(v[34]), "=r"(v[35]), "=r"(v[36]), "=r"(v[37]), "=r"(v[38]), "=r"(v[39]), "=r"(v[40]), "=r"(v[41]), "=r"(v[42]), "=r"(v[43]), "=r"(v[44]), "=r"(v[45]), "=r"(v[46]), "=r"(v[47]), "=r"(v[48]), "=r"(v[49]), "=r"(v[50]), "=r"(v[51]), "=r"(v[52]), "=r"(v[53]), "=r"(v[54]), "=r"(v[55]), "=r"(v[56]), "=r"(v[57]), "=r"(v[58]), "=r"(v[59]), "=r"(v[60]), "=r"(v[61]), "=r"(v[62]), "=r"(v[63])
        : "r"(taddr) MS_TMEM_LD_CLOBBER);
}

// 16 consecutive tensor-memory columns of this warp's 32 lanes.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr)
        : "memory");
}
__device__ __forceinline__ void tmem_wait16(uint32_t (&v)[16]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]), "+r"(v[6]), "+r"(v[7]),
                   "+r"(v[8]), "+r"(v[9]), "+r"(v[10]), "+r"(v[11]), "+r"(v[12]), "+r"(v[13]), "+r"(v[14]),
                   "+r"(v[15])
                 :
                 : "memory");
}

// 32 consecutive tensor-memory columns of this warp's 32 lanes.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
          "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
          "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr)
        : "memory");
}
// Waits for this thread's tensor-memory loads; the registers are in-out
// operands so that no use of them moves above the wait.
__device__ __forceinline__ void tmem_wait(uint32_t (&v)[32]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]), "+r"(v[6]), "+r"(v[7]),
                   "+r"(v[8]), "+r"(v[9]), "+r"(v[10]), "+r"(v[11]), "+r"(v[12]), "+r"(v[13]), "+r"(v[14]),
                   "+r"(v[15]), "+r"(v[16]), "+r"(v[17]), "+r"(v[18]), "+r"(v[19]), "+r"(v[20]), "+r"(v[21]),
                   "+r"(v[22]), "+r"(v[23]), "+r"(v[24]), "+r"(v[25]), "+r"(v[26]), "+r"(v[27]), "+r"(v[28]),
                   "+r"(v[29]), "+r"(v[30]), "+r"(v[31])
                 :
                 : "memory");
}

template <int NCOL>
__device__ __forceinline__ void tmem_ld(uint32_t taddr, uint32_t (&v)[NCOL]) {
    if constexpr (NCOL == 32) tmem_ld32(taddr, v);
    else tmem_ld16(taddr, v);
}
template <int NCOL>
__device__ __forceinline__ void tmem_wait(uint32_t (&v)[NCOL]) {
    if constexpr (NCOL == 32) tmem_wait(v);
    else tmem_wait16(v);
}

// N (2 or 4) consecutive floats of shared memory (8- or 16-byte aligned).
template <int N>
__device__ __forceinline__ void lds_vec(const float *p, float (&v)[N]) {
    if constexpr (N == 4) {
        const float4 q = *reinterpret_cast<const float4 *>(p);
        v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
    } else {
        const float2 q = *reinterpret_cast<const float2 *>(p);
        v[0] = q.x; v[1] = q.y;
    }
}
template <int N>
__device__ __forceinline__ void sts_vec(float *p, const float (&v)[N]) {
    if constexpr (N == 4) *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
    else *reinterpret_cast<float2 *>(p) = make_float2(v[0], v[1]);
}

__device__ __forceinline__ void report_abort(const ScanArgs &a, volatile int *abort_flag) {
    *abort_flag = 1;
    if (a.status) atomicOr(a.status, MS_ERR_TIMEOUT);
}

// One value of B (v < 4) or C (v >= 4) for state group k and token t from
// the staged [16][32] tiles, as fp32.
template <typename TIn>
__device__ __forceinline__ float bc_value(const unsigned char *Bs, const unsigned char *Cs, int t, int k, int v) {
    const unsigned char *src = v < 4 ? Bs : Cs;
    const int n = 4 * k + (v & 3);
    const TIn *p = reinterpret_cast<const TIn *>(src) + n * kT + t;
    return to_f32(*p);
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 h2 = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h2);
}

// One input element as fp32.
template <typename T>
__device__ __forceinline__ float ld_in(const T *p) {
    if constexpr (sizeof(T) == 4) return __ldg(reinterpret_cast<const float *>(p));
    else return bf16_bits_to_f32(__ldg(reinterpret_cast<const unsigned short *>(p)));
}
// 8 fp32 values stored as 8 consecutive input-dtype elements (one or two
// 16-byte stores when the row allows, else element stores).
template <typename T>
__device__ __forceinline__ void store8_in(T *p, bool vec, const float (&v)[8]) {
    if constexpr (sizeof(T) == 4) {
        if (vec) {
            reinterpret_cast<float4 *>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
            reinterpret_cast<float4 *>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
        } else {
#pragma unroll
            for (int j = 0; j < 8; ++j) reinterpret_cast<float *>(p)[j] = v[j];
        }
    } else {
        if (vec) {
            *reinterpret_cast<uint4 *>(p) =
                make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]), pack_bf16(v[4], v[5]), pack_bf16(v[6], v[7]));
        } else {
#pragma unroll
            for (int j = 0; j < 8; ++j) p[j] = __float2bfloat16_rn(v[j]);
        }
    }
}


// YOUT false: the first pass of a sequence split (no y; the end state and
// the sum of Delta over the tokens per channel instead). CKPT: the training
// forward of a layer wider than the 12-warp instantiation covers (that one
// saves states whenever it is given a buffer; in the wider ones the store
// costs the plain forward's state loop spills, so they have their own).
template <typename TIn, typename TOut, int POLY8, int MAXW, bool YOUT, bool CONV = false, bool CKPT = false>
__global__ void __launch_bounds__(32 * (MAXW + 1), 1)
scan_fwd_tmem_kernel(const ScanArgs a, const __grid_constant__ TmMaps maps, const int W, const int S) {
    extern __shared__ __align__(1024) unsigned char smem[];
    // tokens per tensor-memory load: 4 (32 columns) where registers allow two
    // such sets without spilling, 2 (16 columns) in the larger instantiations
    constexpr int TOK = (MAXW <= 11 || !MS_TMEM_DB) ? 4 : 2;
    constexpr bool SPLAT = MS_TMEM_SPLAT && !MS_TMEM_SCALAR && MAXW <= 11;  // matches TmLayout::splat()
    const TmLayout lay{W, S, (int)sizeof(TIn)};
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int cwc = lay.cwc();
    const int64_t dblocks = (a.dim + cwc - 1) / cwc;
    const int64_t b = blockIdx.x / dblocks;
    const int64_t dbase = (blockIdx.x % dblocks) * cwc;
    const int64_t L = a.L;
    const int ntiles = (int)((L + kT - 1) / kT);
    const bool has_z = YOUT && a.z != nullptr;

    auto bar = [&](int i) { return sa(smem) + (uint32_t)(8 * i); };
    const uint32_t full0 = 0, empty0 = (uint32_t)S, mma0 = (uint32_t)(2 * S), tfree0 = (uint32_t)(2 * S + 2);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + lay.abort_slot());
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + lay.tmem_slot());

    // ---- set-up: barriers, the selection matrix S, the zero parts of V
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            bar_init(bar(full0 + s), 1);
            bar_init(bar(empty0 + s), (uint32_t)W + 1);
        }
        for (int i = 0; i < 2; ++i) {
            bar_init(bar(mma0 + i), 1);
            bar_init(bar(tfree0 + i), (uint32_t)W);
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // S[m][k] = 1 when k % 4 == m % 4 and k < 12 (three parts of a value), else 0
    for (int i = threadIdx.x; i < 128 * 2; i += blockDim.x) {
        const int r = i >> 1, kc = i & 1;
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int k0 = 8 * kc + 2 * q;
            const float e0 = (k0 < 12 && (k0 & 3) == (r & 3)) ? 1.0f : 0.0f;
            const float e1 = (k0 + 1 < 12 && ((k0 + 1) & 3) == (r & 3)) ? 1.0f : 0.0f;
            w[q] = pack_bf16(e0, e1);
        }
        *reinterpret_cast<uint4 *>(smem + lay.asel() + op_off(r, kc)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    // V: both buffers start at zero (the producer rewrites the used parts every tile)
    for (int i = threadIdx.x; i < 2 * 8192 / 16; i += blockDim.x)
        *reinterpret_cast<uint4 *>(smem + lay.op(0) + 16 * i) = make_uint4(0u, 0u, 0u, 0u);
    if (warp == W) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(sa(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = *tmem_slot;
#ifdef MS_DEBUG
    {
        uint32_t dyn;
        asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn));
        (void)MS_CHECK(a.status, (uint32_t)lay.total() <= dyn && W >= 1 && W <= MAXW && S >= 2 && (int)blockDim.x == 32 * (W + 1));
    }
#endif

    const uint32_t chan_bytes = (uint32_t)lay.chan_tile(), bc_bytes = (uint32_t)lay.bc_tile();
    const uint32_t tile_tx = (has_z ? 3u : 2u) * chan_bytes + 2u * bc_bytes;

    if (warp == W) {
        // =============================== producer warp ===============================
        int issued = 0;  // tiles whose loads were issued
        auto issue = [&](int k) {
            const int s = k % S;
            const uint32_t st = sa(smem + lay.stage(s));
            const uint32_t fb = bar(full0 + s);
            bar_expect_tx(fb, tile_tx);
            const int x = k * kT;
            tma_load3(st, &maps.u, x, (int)dbase, (int)b, fb);
            tma_load3(st + chan_bytes, &maps.dl, x, (int)dbase, (int)b, fb);
            if (has_z) tma_load3(st + 2 * chan_bytes, &maps.z, x, (int)dbase, (int)b, fb);
            tma_load3(st + 3 * chan_bytes, &maps.B, x, 0, (int)b, fb);
            tma_load3(st + 3 * chan_bytes + bc_bytes, &maps.C, x, 0, (int)b, fb);
        };
        if (lane == 0)
            for (int k = 0; k < S - 1 && k < ntiles; ++k) issue(k);
        issued = ntiles < S - 1 ? ntiles : S - 1;
        int mmas = 0;      // MMAs issued
        int consumed = 0;  // tiles whose full barrier this warp has passed
        bool ok = true;
        // loads of tile k + S - 1 into the stage tile k - 1 used, once every
        // compute warp has read that tile's u, delta, z
        auto prefetch = [&](int k) -> bool {
            bool good = true;
            const int kk = k + S - 1;
            if (kk < ntiles) {
                if (lane == 0) {
                    if (kk >= S) good = bar_wait(bar(empty0 + kk % S), (uint32_t)(((kk - S) / S) & 1));
                    if (good) issue(kk);
                }
                good = __shfl_sync(0xffffffffu, good ? 1 : 0, 0) != 0;
                if (good) issued = kk + 1;
            }
            return good;
        };
        for (int k = 0; k < ntiles && ok; ++k) {
            if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
            if (!MS_TMEM_MMA_FIRST) {
                ok = prefetch(k);
                if (!ok) break;
            }
            // (1) tile k's B/C -> V[k % 2], once MMA k - 2 has finished reading it
            const int s = k % S, vb = k & 1;
            ok = bar_wait(bar(full0 + s), (uint32_t)((k / S) & 1));
            if (ok && k >= 2) ok = bar_wait(bar(mma0 + vb), (uint32_t)(((k - 2) >> 1) & 1));
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            consumed = k + 1;
            {
                const unsigned char *Bs = smem + lay.stage(s) + 3 * chan_bytes;
                const unsigned char *Cs = Bs + bc_bytes;
                unsigned char *V = smem + lay.op(vb);
                // row r = 8t + v: lane handles rows lane, lane + 32, ... (8 rows)
#pragma unroll 2
                for (int r = lane; r < 256; r += 32) {
                    const int t = r >> 3, v = r & 7;
                    if (!MS_CHECK(a.status, op_off(r, 1) + 16 <= 8192 && t < kT)) continue;
                    if constexpr (sizeof(TIn) == 2) {
                        // bf16 inputs: exact in one part (columns 0..3; 4..11 stay
                        // zero), moved as raw 16-bit values
                        const uint16_t *src = reinterpret_cast<const uint16_t *>(v < 4 ? Bs : Cs) + (v & 3) * kT + t;
                        const uint32_t e0 = src[0], e1 = src[4 * kT], e2 = src[8 * kT], e3 = src[12 * kT];
                        *reinterpret_cast<uint2 *>(V + op_off(r, 0)) = make_uint2(e0 | (e1 << 16), e2 | (e3 << 16));
                    } else {
                        // fp32 inputs: v = hi + mid + lo, each part bf16 (exact: 3 x 8 bits)
                        float val[4], hi[4], mid[4], lo[4];
#pragma unroll
                        for (int k4 = 0; k4 < 4; ++k4) {
                            val[k4] = bc_value<TIn>(Bs, Cs, t, k4, v);
                            hi[k4] = __bfloat162float(__float2bfloat16_rn(val[k4]));
                            const float r1 = val[k4] - hi[k4];
                            mid[k4] = __bfloat162float(__float2bfloat16_rn(r1));
                            lo[k4] = __bfloat162float(__float2bfloat16_rn(r1 - mid[k4]));
                        }
                        *reinterpret_cast<uint4 *>(V + op_off(r, 0)) =
                            make_uint4(pack_bf16(hi[0], hi[1]), pack_bf16(hi[2], hi[3]), pack_bf16(mid[0], mid[1]),
                                       pack_bf16(mid[2], mid[3]));
                        *reinterpret_cast<uint2 *>(V + op_off(r, 1)) =
                            make_uint2(pack_bf16(lo[0], lo[1]), pack_bf16(lo[2], lo[3]));
                    }
                }
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) {
                bar_arrive(bar(empty0 + s));  // this warp is done with the stage's B/C
                // (2) D[vb] = S x V[vb]^T once the compute warps have read tile k - 2's columns
                if (k >= 2) ok = bar_wait(bar(tfree0 + vb), (uint32_t)(((k - 2) >> 1) & 1));
                if (ok) {
                    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                    const uint64_t da = mat_desc(sa(smem + lay.asel()), 128u, 256u);
                    const uint64_t db = mat_desc(sa(smem + lay.op(vb)), 128u, 256u);
                    const uint32_t dcol = tmem + (uint32_t)(vb * kBufCols);
                    asm volatile(
                        "{\n\t.reg .pred p;\n\t"
                        "setp.ne.b32 p, %4, 0;\n\t"
                        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(dcol),
                        "l"(da), "l"(db), "r"(kIdesc), "r"(0u), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
                        : "memory");
                    asm volatile(
                        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                            bar(mma0 + vb))
                        : "memory");
                }
            }
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok) break;
            mmas = k + 1;
            if (MS_TMEM_MMA_FIRST) {
                ok = prefetch(k);
                if (!ok) break;
            }
        }
        if (!ok && lane == 0) report_abort(a, abort_flag);
        // drain: loads issued but not consumed here, and the last MMAs
        if (lane == 0) {
            for (int k = consumed; k < issued; ++k) bar_wait(bar(full0 + k % S), (uint32_t)((k / S) & 1));
            for (int k = (mmas >= 2 ? mmas - 2 : 0); k < mmas; ++k)
                bar_wait(bar(mma0 + (k & 1)), (uint32_t)((k >> 1) & 1));
        }
        __syncwarp();
    } else {
        // =============================== compute warps ===============================
        const int c = lane >> 2, g = lane & 3;
        const int cc = warp * kCW + c;           // channel within the CTA
        const int64_t d = dbase + cc;
        const bool active = d < a.dim;
        const int64_t dd = active ? d : 0;
        const int n0 = 4 * g;
        f2 A2[2], h[2];
        float amax2;  // max |A| log2(e) over the channel's 16 states (after the shuffles below)
        {
            const float4 Av = *reinterpret_cast<const float4 *>(a.A + dd * 16 + n0);
            A2[0] = f2_make(Av.x * kLog2e, Av.y * kLog2e);
            A2[1] = f2_make(Av.z * kLog2e, Av.w * kLog2e);
            amax2 = kLog2e * fmaxf(fmaxf(fabsf(Av.x), fabsf(Av.y)), fmaxf(fabsf(Av.z), fabsf(Av.w)));
            float4 hv = make_float4(0.f, 0.f, 0.f, 0.f);
            if (a.h0 != nullptr && active) hv = *reinterpret_cast<const float4 *>(a.h0 + (b * a.dim + d) * 16 + n0);
            h[0] = f2_make(hv.x, hv.y);
            h[1] = f2_make(hv.z, hv.w);
        }
        amax2 = fmaxf(amax2, __shfl_xor_sync(0xffffffffu, amax2, 1));
        amax2 = fmaxf(amax2, __shfl_xor_sync(0xffffffffu, amax2, 2));
        const float Dd = a.D ? __ldg(a.D + dd) : 0.0f;
        const float bias = a.bias ? __ldg(a.bias + dd) : 0.0f;
        const bool sp = a.softplus != 0;
        // Conv front-end: taps right-aligned in cw (cw[3] weights the current
        // token) and the 3 inputs before this lane's next chunk (the channel's
        // last lane's copy feeds lane g = 0 of the next tile)
        float cw[4] = {0.0f, 0.0f, 0.0f, 0.0f}, cb = 0.0f;
        float keep[3] = {0.0f, 0.0f, 0.0f};
        TIn *uo_row = nullptr;
        if constexpr (CONV) {
            const int Wc = a.conv_width;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int src = k - (4 - Wc);
                if (src >= 0) cw[k] = __ldg(a.conv_w + dd * Wc + src);
            }
            cb = a.conv_b ? __ldg(a.conv_b + dd) : 0.0f;
            if (a.conv_x0 != nullptr && active) {
                const TIn *x0 = static_cast<const TIn *>(a.conv_x0) + (b * a.dim + d) * (Wc - 1);
#pragma unroll
                for (int j = 1; j <= 3; ++j)
                    if (Wc - 1 - j >= 0) keep[3 - j] = ld_in<TIn>(x0 + (Wc - 1 - j));
            }
            if (a.u_out != nullptr) uo_row = static_cast<TIn *>(a.u_out) + b * a.uo_sb + dd * a.uo_sd;
        }
        float *xd = reinterpret_cast<float *>(smem + lay.xch(warp));   // [8][kRow] Delta (or the pairs)
        float *xu = xd + kCW * kRow;                                     // [8][kRow] Delta*u
        float *pr = xd + (SPLAT ? kCW * kRowS : 2 * kCW * kRow);         // [8*4][kRow] partial readouts
        TOut *y_row = static_cast<TOut *>(a.y) + b * a.y_sb + dd * a.y_sd;
        const uint32_t trow = (uint32_t)(32 * (warp & 3)) << 16;        // this warp's accumulator lanes

        bool ok = true;
        float dsum_acc = 0.0f;  // this lane's tokens' Delta (first pass of a split)
        constexpr bool FUSED = MS_TMEM_FUSED && YOUT && MAXW <= 11 && !SPLAT && !MS_TMEM_SCALAR && TOK == 4;
        if constexpr (FUSED) {
            constexpr int kWords = 8 * (int)sizeof(TIn) / 4;  // one 8-token chunk in 32-bit words
            // raw inputs of chunk g of channel c from a stage, as stored
            auto load_raw = [&](int k, uint32_t(&uw)[kWords], uint32_t(&dw)[kWords], uint32_t(&zw)[kWords]) {
                const unsigned char *st = smem + lay.stage(k % S);
                int off = (cc * kT + 8 * g) * (int)sizeof(TIn);
                if (!MS_CHECK(a.status, off + 8 * (int)sizeof(TIn) <= (int)chan_bytes && cc < cwc)) off = 0;
#pragma unroll
                for (int q = 0; q < kWords / 4; ++q) {
                    const uint4 U = *reinterpret_cast<const uint4 *>(st + off + 16 * q);
                    const uint4 Dl = *reinterpret_cast<const uint4 *>(st + chan_bytes + off + 16 * q);
                    uw[4 * q] = U.x; uw[4 * q + 1] = U.y; uw[4 * q + 2] = U.z; uw[4 * q + 3] = U.w;
                    dw[4 * q] = Dl.x; dw[4 * q + 1] = Dl.y; dw[4 * q + 2] = Dl.z; dw[4 * q + 3] = Dl.w;
                    if (has_z) {
                        const uint4 Z = *reinterpret_cast<const uint4 *>(st + 2 * chan_bytes + off + 16 * q);
                        zw[4 * q] = Z.x; zw[4 * q + 1] = Z.y; zw[4 * q + 2] = Z.z; zw[4 * q + 3] = Z.w;
                    } else {
                        zw[4 * q] = zw[4 * q + 1] = zw[4 * q + 2] = zw[4 * q + 3] = 0u;
                    }
                }
            };
            auto elem = [&](const uint32_t(&w)[kWords], int j) -> float {
                if constexpr (sizeof(TIn) == 4) return __uint_as_float(w[j]);
                else return (j & 1) ? bf16_hi(w[j >> 1]) : bf16_lo(w[j >> 1]);
            };
            // token j of the chunk: Delta, Delta*u, silu(z), D*u*silu(z)
            auto prol = [&](const uint32_t(&uw)[kWords], const uint32_t(&dw)[kWords], const uint32_t(&zw)[kWords],
                            int j, bool live, float &dl, float &dlu, float &gate, float &dug) {
                const float u = elem(uw, j);
                const float v = elem(dw, j) + bias;
                dl = live ? (sp ? softplus_f(v) : v) : 0.0f;  // past the end: the state is left alone
                dlu = dl * u;
                gate = has_z ? silu_f(elem(zw, j)) : 1.0f;
                dug = Dd * u * gate;
            };
            auto write_x = [&](const float(&dl)[8], const float(&dlu)[8]) {
                float4 *pd = reinterpret_cast<float4 *>(xd + c * kRow + 8 * g);
                float4 *pu = reinterpret_cast<float4 *>(xu + c * kRow + 8 * g);
                pd[0] = make_float4(dl[0], dl[1], dl[2], dl[3]);
                pd[1] = make_float4(dl[4], dl[5], dl[6], dl[7]);
                pu[0] = make_float4(dlu[0], dlu[1], dlu[2], dlu[3]);
                pu[1] = make_float4(dlu[4], dlu[5], dlu[6], dlu[7]);
            };
            float gate[8], dug[8];  // the current tile's chunk
            uint32_t uw[kWords], dw[kWords], zw[kWords];
            if (ntiles > 0) {
                ok = __all_sync(0xffffffffu, bar_wait(bar(full0), 0u));
                if (ok) {
                    load_raw(0, uw, dw, zw);
                    __syncwarp();
                    if (lane == 0) bar_arrive(bar(empty0));  // this warp is done with stage 0
                    float dl[8], dlu[8];
                    const bool live = 8 * g < L;
#pragma unroll
                    for (int j = 0; j < 8; ++j) prol(uw, dw, zw, j, live, dl[j], dlu[j], gate[j], dug[j]);
                    write_x(dl, dlu);
                    __syncwarp();
                }
            }
            for (int k = 0; k < ntiles && ok; ++k) {
                if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
                const int vb = k & 1;
                const int64_t t0 = (int64_t)k * kT;
                const bool has_next = k + 1 < ntiles;
                const bool live_next = t0 + kT + 8 * g < L;
                // the next tile's raw inputs, into registers; its stage is then free
                if (has_next) {
                    ok = __all_sync(0xffffffffu, bar_wait(bar(full0 + (k + 1) % S), (uint32_t)(((k + 1) / S) & 1)));
                    if (!ok) break;
                    load_raw(k + 1, uw, dw, zw);
                    __syncwarp();
                    if (lane == 0) bar_arrive(bar(empty0 + (k + 1) % S));
                }
                ok = __all_sync(0xffffffffu, bar_wait(bar(mma0 + vb), (uint32_t)((k >> 1) & 1)));
                if (!ok) break;
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                const uint32_t tcol = tmem + trow + (uint32_t)(vb * kBufCols);
                float dln[8], dlun[8], gaten[8], dugn[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    uint32_t bc[32];
                    (void)MS_CHECK(a.status, vb * kBufCols + 32 * (j + 1) <= kTmemCols && 4 * c + g < 32);
                    tmem_ld32(tcol + (uint32_t)(32 * j), bc);
                    const float4 dl4 = *reinterpret_cast<const float4 *>(xd + c * kRow + 4 * j);
                    const float4 du4 = *reinterpret_cast<const float4 *>(xu + c * kRow + 4 * j);
                    // the next tile's token j (independent of this group's chains)
                    if (has_next) prol(uw, dw, zw, j, live_next, dln[j], dlun[j], gaten[j], dugn[j]);
                    tmem_wait(bc);
                    const float dls[4] = {dl4.x, dl4.y, dl4.z, dl4.w};
                    const float dus[4] = {du4.x, du4.y, du4.z, du4.w};
                    float part[4];
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        const f2 dl2 = f2_splat(dls[t]);
                        const f2 du2 = f2_splat(dus[t]);
                        f2 acc = 0ull;
#pragma unroll
                        for (int p = 0; p < 2; ++p) {
                            const f2 Bp = f2_make(__uint_as_float(bc[8 * t + 2 * p]), __uint_as_float(bc[8 * t + 2 * p + 1]));
                            const f2 Cp = f2_make(__uint_as_float(bc[8 * t + 4 + 2 * p]), __uint_as_float(bc[8 * t + 5 + 2 * p]));
                            const f2 x = f2_mul(A2[p], dl2);
                            const bool poly = (2 * t + p) < POLY8;
                            f2 ab;
                            if (poly) {
                                ab = exp2_poly2(x);
                            } else {
                                float xa, xb;
                                f2_split(x, xa, xb);
                                ab = f2_make(exp2_mufu(xa), exp2_mufu(xb));
                            }
                            h[p] = f2_fma(ab, h[p], f2_mul(du2, Bp));
                            acc = p == 0 ? f2_mul(Cp, h[p]) : f2_fma(Cp, h[p], acc);
                        }
                        float lo, hi;
                        f2_split(acc, lo, hi);
                        part[t] = lo + hi;
                    }
                    *reinterpret_cast<float4 *>(pr + (c * 4 + g) * kRow + 4 * j) =
                        make_float4(part[0], part[1], part[2], part[3]);
                }
                // tensor-memory buffer vb is read: release it to the producer
                asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
                __syncwarp();
                if (lane == 0) bar_arrive(bar(tfree0 + vb));
                // ---- epilogue of this tile: chunk g of channel c
                float ys[8];
                {
                    const float4 *p0 = reinterpret_cast<const float4 *>(pr + (c * 4) * kRow + 8 * g);
                    float4 a0 = p0[0], a1 = p0[1];
#pragma unroll
                    for (int q = 1; q < 4; ++q) {
                        const float4 *pq = reinterpret_cast<const float4 *>(pr + (c * 4 + q) * kRow + 8 * g);
                        const float4 b0 = pq[0], b1 = pq[1];
                        a0.x += b0.x; a0.y += b0.y; a0.z += b0.z; a0.w += b0.w;
                        a1.x += b1.x; a1.y += b1.y; a1.z += b1.z; a1.w += b1.w;
                    }
                    ys[0] = a0.x; ys[1] = a0.y; ys[2] = a0.z; ys[3] = a0.w;
                    ys[4] = a1.x; ys[5] = a1.y; ys[6] = a1.z; ys[7] = a1.w;
                }
                const bool live = t0 + 8 * g < L;
                if (active && live && MS_CHECK(a.status, t0 + 8 * g + 8 <= L && d < a.dim)) {
                    float yo[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) yo[j] = fmaf(ys[j], gate[j], dug[j]);
                    TOut *yp = y_row + t0 + 8 * g;
                    if constexpr (sizeof(TOut) == 4) {
                        float4 *pp = reinterpret_cast<float4 *>(yp);
                        __stcs(pp, make_float4(yo[0], yo[1], yo[2], yo[3]));
                        __stcs(pp + 1, make_float4(yo[4], yo[5], yo[6], yo[7]));
                    } else {
                        __stcs(reinterpret_cast<uint4 *>(yp), make_uint4(pack_bf16(yo[0], yo[1]), pack_bf16(yo[2], yo[3]),
                                                                         pack_bf16(yo[4], yo[5]), pack_bf16(yo[6], yo[7])));
                    }
                }
                // every lane is past this tile's Delta rows and partials
                __syncwarp();
                if (has_next) {
                    write_x(dln, dlun);
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        gate[j] = gaten[j];
                        dug[j] = dugn[j];
                    }
                    __syncwarp();
                }
            }
        }
        for (int k = 0; k < ntiles && !FUSED; ++k) {
            if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
            const int s = k % S, vb = k & 1;
            const int64_t t0 = (int64_t)k * kT;
            // Training (the 12-warp instantiation, and the CKPT instantiations of the
            // wider ones): the state before this 64-token block, for the backward's
            // recompute ([batch, dim, ceil(L / 64), 16] fp32; this lane's 4 states)
            if ((MAXW == kMaxWSmall || CKPT) && a.ckpt != nullptr && t0 % kCkptTokens == 0 && active) {
                float h0a, h0b, h1a, h1b;
                f2_split(h[0], h0a, h0b);
                f2_split(h[1], h1a, h1b);
                const int64_t nck = (L + kCkptTokens - 1) / kCkptTokens;
                *reinterpret_cast<float4 *>(a.ckpt + ((b * a.dim + d) * nck + t0 / kCkptTokens) * 16 + n0) =
                    make_float4(h0a, h0b, h1a, h1b);
            }
            ok = __all_sync(0xffffffffu, bar_wait(bar(full0 + s), (uint32_t)((k / S) & 1)));
            if (!ok) break;
            // ---- prologue: chunk g of channel c (tokens 8g..8g+7 of the tile)
            const unsigned char *st = smem + lay.stage(s);
            float uv[8], dv[8], zv[8];
            {
                int off = (cc * kT + 8 * g) * (int)sizeof(TIn);
                if (!MS_CHECK(a.status, off + 8 * (int)sizeof(TIn) <= (int)chan_bytes && cc < cwc)) off = 0;
                if constexpr (sizeof(TIn) == 2) {
                    const uint4 U = *reinterpret_cast<const uint4 *>(st + off);
                    const uint4 Dl = *reinterpret_cast<const uint4 *>(st + chan_bytes + off);
                    const uint32_t uw[4] = {U.x, U.y, U.z, U.w}, dw[4] = {Dl.x, Dl.y, Dl.z, Dl.w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uv[2 * q] = bf16_lo(uw[q]);
                        uv[2 * q + 1] = bf16_hi(uw[q]);
                        dv[2 * q] = bf16_lo(dw[q]);
                        dv[2 * q + 1] = bf16_hi(dw[q]);
                    }
                    if (has_z) {
                        const uint4 Z = *reinterpret_cast<const uint4 *>(st + 2 * chan_bytes + off);
                        const uint32_t zw[4] = {Z.x, Z.y, Z.z, Z.w};
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            zv[2 * q] = bf16_lo(zw[q]);
                            zv[2 * q + 1] = bf16_hi(zw[q]);
                        }
                    }
                } else {
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const float4 U = *reinterpret_cast<const float4 *>(st + off + 16 * q);
                        const float4 Dl = *reinterpret_cast<const float4 *>(st + chan_bytes + off + 16 * q);
                        uv[4 * q] = U.x; uv[4 * q + 1] = U.y; uv[4 * q + 2] = U.z; uv[4 * q + 3] = U.w;
                        dv[4 * q] = Dl.x; dv[4 * q + 1] = Dl.y; dv[4 * q + 2] = Dl.z; dv[4 * q + 3] = Dl.w;
                        if (has_z) {
                            const float4 Z = *reinterpret_cast<const float4 *>(st + 2 * chan_bytes + off + 16 * q);
                            zv[4 * q] = Z.x; zv[4 * q + 1] = Z.y; zv[4 * q + 2] = Z.z; zv[4 * q + 3] = Z.w;
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) bar_arrive(bar(empty0 + s));  // this warp is done with the stage
            const bool live = t0 + 8 * g < L;  // L % 8 == 0: whole chunks are in or out
            if constexpr (CONV) {
                // u from the conv input x (the stage held x): the halo x[t-3..t-1] is the
                // previous lane's chunk tail, or for g = 0 the channel's last lane's tail
                // of the previous tile
                const bool last_lane = g == 3;
                const int src = g == 0 ? lane + 3 : lane - 1;
                const float h0 = __shfl_sync(0xffffffffu, last_lane ? keep[0] : uv[5], src);
                const float h1 = __shfl_sync(0xffffffffu, last_lane ? keep[1] : uv[6], src);
                const float h2 = __shfl_sync(0xffffffffu, last_lane ? keep[2] : uv[7], src);
                keep[0] = uv[5];
                keep[1] = uv[6];
                keep[2] = uv[7];
                float xs[11];
                xs[0] = h0;
                xs[1] = h1;
                xs[2] = h2;
#pragma unroll
                for (int j = 0; j < 8; ++j) xs[3 + j] = uv[j];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    float v = fmaf(cw[0], xs[j], cb);
                    v = fmaf(cw[1], xs[j + 1], v);
                    v = fmaf(cw[2], xs[j + 2], v);
                    v = fmaf(cw[3], xs[j + 3], v);
                    uv[j] = a.conv_silu ? silu_f(v) : v;
                }
                if (uo_row != nullptr && active && live) store8_in<TIn>(uo_row + t0 + 8 * g, a.vec_uout != 0, uv);
            }
            float gate[8], dug[8];
            // every exponent |Delta A| log2(e) of the warp's tile within the
            // series' range: the tile's decays come from the expm1 series
            bool series_tile = false;
            {
                float dl[8], dlu[8], dmax = 0.0f;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float v = dv[j] + bias;
                    dl[j] = live ? (sp ? softplus_f(v) : v) : 0.0f;  // past the end: the state is left alone
                    dmax = fmaxf(dmax, fabsf(dl[j]));
                    dlu[j] = dl[j] * uv[j];
                    if constexpr (YOUT) {
                        gate[j] = has_z ? silu_f(zv[j]) : 1.0f;
                        dug[j] = Dd * uv[j] * gate[j];
                    } else {
                        dsum_acc += dl[j];
                    }
                }
                if constexpr (POLY8 == 8 && MS_TMEM_SERIES) series_tile = __all_sync(0xffffffffu, dmax * amax2 <= Expm1Series::kMaxArg);
                if constexpr (SPLAT) {
                    float4 *px = reinterpret_cast<float4 *>(xd + c * kRowS + 4 * (8 * g));
#pragma unroll
                    for (int j = 0; j < 8; ++j) px[j] = make_float4(dl[j], dl[j], dlu[j], dlu[j]);
                } else {
                    float4 *pd = reinterpret_cast<float4 *>(xd + c * kRow + 8 * g);
                    float4 *pu = reinterpret_cast<float4 *>(xu + c * kRow + 8 * g);
                    pd[0] = make_float4(dl[0], dl[1], dl[2], dl[3]);
                    pd[1] = make_float4(dl[4], dl[5], dl[6], dl[7]);
                    pu[0] = make_float4(dlu[0], dlu[1], dlu[2], dlu[3]);
                    pu[1] = make_float4(dlu[4], dlu[5], dlu[6], dlu[7]);
                }
            }
            __syncwarp();
            // ---- the tile's B/C in tensor memory
            ok = __all_sync(0xffffffffu, bar_wait(bar(mma0 + vb), (uint32_t)((k >> 1) & 1)));
            if (!ok) break;
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            // ---- states: groups of TOK tokens; the tensor-memory load and the
            // Delta / Delta*u loads of the next group are in flight while a
            // group computes (two register sets, used alternately)
            const uint32_t tcol = tmem + trow + (uint32_t)(vb * kBufCols);
            uint32_t bcA[8 * TOK], bcB[8 * TOK];
            f2 dlA[TOK], duA[TOK], dlB[TOK], duB[TOK];
            auto fetch = [&](int j, uint32_t(&bc)[8 * TOK], f2(&dl)[TOK], f2(&du)[TOK]) {
                (void)MS_CHECK(a.status, vb * kBufCols + 8 * TOK * (j + 1) <= kTmemCols && 4 * c + g < 32);
                tmem_ld<8 * TOK>(tcol + (uint32_t)(8 * TOK * j), bc);
                if constexpr (SPLAT) {
                    // (Delta, Delta, Delta*u, Delta*u) per token: both pairs in one load
#pragma unroll
                    for (int t = 0; t < TOK; ++t) lds_f2x2(xd + c * kRowS + 4 * (TOK * j + t), dl[t], du[t]);
                } else {
                    float dls[TOK], dus[TOK];
                    lds_vec<TOK>(xd + c * kRow + TOK * j, dls);
                    lds_vec<TOK>(xu + c * kRow + TOK * j, dus);
#pragma unroll
                    for (int t = 0; t < TOK; ++t) {
                        dl[t] = f2_splat(dls[t]);
                        du[t] = f2_splat(dus[t]);
                    }
                }
            };
            // series: a tile whose decays all come from the expm1 series
            // (h += (A_bar - 1) h + Delta u B); the callers pass a constant
            auto group = [&](bool series, int j, const uint32_t(&bc)[8 * TOK], const f2(&dl2s)[TOK],
                             const f2(&du2s)[TOK]) {
                float part[TOK];
                if constexpr (MS_TMEM_SCALAR) {
                    // the pairs hold (Delta, Delta) and (Delta*u, Delta*u): use one half
                    float hs[4], As[4];
                    f2_split(h[0], hs[0], hs[1]);
                    f2_split(h[1], hs[2], hs[3]);
                    f2_split(A2[0], As[0], As[1]);
                    f2_split(A2[1], As[2], As[3]);
#pragma unroll
                    for (int t = 0; t < TOK; ++t) {
                        float dl, du, unused;
                        f2_split(dl2s[t], dl, unused);
                        f2_split(du2s[t], du, unused);
                        float acc = 0.0f;
#pragma unroll
                        for (int n = 0; n < 4; ++n) {
                            const float x = As[n] * dl;
                            const bool poly = (2 * ((TOK * j + t) & 3) + (n >> 1)) < POLY8;
                            const float ab = poly ? exp2_poly(x) : exp2_mufu(x);
                            hs[n] = fmaf(ab, hs[n], du * __uint_as_float(bc[8 * t + n]));
                            if constexpr (YOUT) acc = fmaf(__uint_as_float(bc[8 * t + 4 + n]), hs[n], acc);
                        }
                        part[t] = acc;
                    }
                    h[0] = f2_make(hs[0], hs[1]);
                    h[1] = f2_make(hs[2], hs[3]);
                    if constexpr (YOUT) sts_vec<TOK>(pr + (c * 4 + g) * kRow + TOK * j, part);
                    return;
                }
#pragma unroll
                for (int t = 0; t < TOK; ++t) {
                    const f2 dl2 = dl2s[t];
                    const f2 du2 = du2s[t];
                    // this token's exponents within the series' range on every lane of the warp
                    bool ser_t = false;
                    if constexpr (POLY8 == 8 && MS_TMEM_SERIES) {
                        float d0, d1;
                        f2_split(dl2, d0, d1);
                        ser_t = series || __all_sync(0xffffffffu, fabsf(d0) * amax2 <= Expm1Series::kMaxArg);
                    }
                    f2 acc = 0ull;
#pragma unroll
                    for (int p = 0; p < 2; ++p) {
                        const f2 Bp =
                            f2_make(__uint_as_float(bc[8 * t + 2 * p]), __uint_as_float(bc[8 * t + 2 * p + 1]));
                        const f2 x = f2_mul(A2[p], dl2);
                        if (POLY8 == 8 && ser_t) {
                            h[p] = f2_fma(exp2m1_series2(x), h[p], f2_fma(du2, Bp, h[p]));
                        } else {
                            // a fixed share of the (token, pair) slots of every 4 tokens on the polynomial
                            const bool poly = (2 * ((TOK * j + t) & 3) + p) < POLY8;
                            f2 ab;
                            if (poly) {
                                ab = exp2_poly2(x);
                            } else {
                                float xa, xb;
                                f2_split(x, xa, xb);
                                ab = f2_make(exp2_mufu(xa), exp2_mufu(xb));
                            }
                            h[p] = f2_fma(ab, h[p], f2_mul(du2, Bp));
                        }
                        if constexpr (YOUT) {
                            const f2 Cp = f2_make(__uint_as_float(bc[8 * t + 4 + 2 * p]),
                                                  __uint_as_float(bc[8 * t + 5 + 2 * p]));
                            acc = p == 0 ? f2_mul(Cp, h[p]) : f2_fma(Cp, h[p], acc);
                        }
                    }
                    float lo, hi;
                    f2_split(acc, lo, hi);
                    part[t] = lo + hi;
                }
                if constexpr (YOUT) sts_vec<TOK>(pr + (c * 4 + g) * kRow + TOK * j, part);
            };
            // the y-less pass keeps the loop rolled (unrolled it spills)
            constexpr int kUnr = YOUT ? kUnrollGroups : 1;
            auto run_tile = [&](bool sc) {
                constexpr int NG = kT / TOK;
                if constexpr (!MS_TMEM_DB && MS_TMEM_LD64 && MAXW <= 11 && YOUT) {
                    uint32_t bc2[16 * TOK];
#pragma unroll
                    for (int j = 0; j < NG; j += 2) {
                        static_assert(TOK == 4 && !SPLAT, "single loads: 4 tokens, plain Delta rows");
                        (void)MS_CHECK(a.status, vb * kBufCols + 32 * (j + 2) <= kTmemCols && 4 * c + g < 32);
                        float dls0[TOK], dus0[TOK], dls1[TOK], dus1[TOK];
                        lds_vec<TOK>(xd + c * kRow + TOK * j, dls0);
                        lds_vec<TOK>(xu + c * kRow + TOK * j, dus0);
                        lds_vec<TOK>(xd + c * kRow + TOK * (j + 1), dls1);
                        lds_vec<TOK>(xu + c * kRow + TOK * (j + 1), dus1);
                        tmem_ld64_sync(tcol + (uint32_t)(32 * j), bc2);
#pragma unroll
                        for (int t = 0; t < TOK; ++t) {
                            dlA[t] = f2_splat(dls0[t]);
                            duA[t] = f2_splat(dus0[t]);
                            dlB[t] = f2_splat(dls1[t]);
                            duB[t] = f2_splat(dus1[t]);
                        }
                        group(sc, j, *reinterpret_cast<const uint32_t(*)[8 * TOK]>(bc2), dlA, duA);
                        group(sc, j + 1, *reinterpret_cast<const uint32_t(*)[8 * TOK]>(bc2 + 8 * TOK), dlB, duB);
                    }
                } else if constexpr (!MS_TMEM_DB) {
#pragma unroll kUnr
                    for (int j = 0; j < NG; ++j) {
                        static_assert(TOK == 4 && !SPLAT, "single loads: 4 tokens, plain Delta rows");
                        (void)MS_CHECK(a.status, vb * kBufCols + 32 * (j + 1) <= kTmemCols && 4 * c + g < 32);
                        float dls[TOK], dus[TOK];
                        lds_vec<TOK>(xd + c * kRow + TOK * j, dls);
                        lds_vec<TOK>(xu + c * kRow + TOK * j, dus);
                        tmem_ld32_sync(tcol + (uint32_t)(32 * j), bcA);
#pragma unroll
                        for (int t = 0; t < TOK; ++t) {
                            dlA[t] = f2_splat(dls[t]);
                            duA[t] = f2_splat(dus[t]);
                        }
                        group(sc, j, bcA, dlA, duA);
                    }
                } else {
                fetch(0, bcA, dlA, duA);
                tmem_wait<8 * TOK>(bcA);
#pragma unroll 1
                for (int j = 0; j < NG; j += 2) {
                    fetch(j + 1, bcB, dlB, duB);
                    group(sc, j, bcA, dlA, duA);
                    tmem_wait<8 * TOK>(bcB);
                    if (j + 2 < NG) fetch(j + 2, bcA, dlA, duA);
                    group(sc, j + 1, bcB, dlB, duB);
                    if (j + 2 < NG) tmem_wait<8 * TOK>(bcA);
                }
                }
            };
            if (POLY8 == 8 && series_tile) run_tile(true);
            else run_tile(false);
            // tensor-memory buffer vb is read: release it to the producer
            asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
            __syncwarp();
            if (lane == 0) bar_arrive(bar(tfree0 + vb));
            if constexpr (!YOUT) continue;
            // ---- epilogue: chunk g of channel c
            float ys[8];
            {
                const float4 *p0 = reinterpret_cast<const float4 *>(pr + (c * 4) * kRow + 8 * g);
                float4 a0 = p0[0], a1 = p0[1];
#pragma unroll
                for (int q = 1; q < 4; ++q) {
                    const float4 *pq = reinterpret_cast<const float4 *>(pr + (c * 4 + q) * kRow + 8 * g);
                    const float4 b0 = pq[0], b1 = pq[1];
                    a0.x += b0.x; a0.y += b0.y; a0.z += b0.z; a0.w += b0.w;
                    a1.x += b1.x; a1.y += b1.y; a1.z += b1.z; a1.w += b1.w;
                }
                ys[0] = a0.x; ys[1] = a0.y; ys[2] = a0.z; ys[3] = a0.w;
                ys[4] = a1.x; ys[5] = a1.y; ys[6] = a1.z; ys[7] = a1.w;
            }
            __syncwarp();
            if (active && live && MS_CHECK(a.status, t0 + 8 * g + 8 <= L && d < a.dim)) {
                float yo[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) yo[j] = fmaf(ys[j], gate[j], dug[j]);
                TOut *yp = y_row + t0 + 8 * g;
                if constexpr (sizeof(TOut) == 4) {
                    float4 *p = reinterpret_cast<float4 *>(yp);
                    __stcs(p, make_float4(yo[0], yo[1], yo[2], yo[3]));
                    __stcs(p + 1, make_float4(yo[4], yo[5], yo[6], yo[7]));
                } else {
                    __stcs(reinterpret_cast<uint4 *>(yp), make_uint4(pack_bf16(yo[0], yo[1]), pack_bf16(yo[2], yo[3]),
                                                                     pack_bf16(yo[4], yo[5]), pack_bf16(yo[6], yo[7])));
                }
            }
        }
        if (!ok && lane == 0) report_abort(a, abort_flag);
        if constexpr (!YOUT) {
            // the channel's 4 lanes hold disjoint token chunks: sum them
            dsum_acc += __shfl_xor_sync(0xffffffffu, dsum_acc, 1);
            dsum_acc += __shfl_xor_sync(0xffffffffu, dsum_acc, 2);
            if (ok && active && g == 0 && a.dsum != nullptr) a.dsum[b * a.dim + d] = dsum_acc;
        }
        if (ok && active && a.last != nullptr) {
            float h0a, h0b, h1a, h1b;
            f2_split(h[0], h0a, h0b);
            f2_split(h[1], h1a, h1b);
            *reinterpret_cast<float4 *>(a.last + (b * a.dim + d) * 16 + n0) = make_float4(h0a, h0b, h1a, h1b);
        }
    }

    // ---- tear-down: every thread arrives here (waits above are bounded)
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == W) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
    }
}

// ------------------------------------------------------------------ host ----

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

// 3-D map over [outer][mid][L] elements: box {32 tokens, rows, 1}.
bool encode3(CUtensorMap *m, const void *base, bool bf16, int64_t L, int64_t mid, int64_t mid_stride, int64_t outer,
             int64_t outer_stride, int rows) {
    PfnEncodeTiled fn = encode_fn();
    if (!fn) return false;
    const int es = bf16 ? 2 : 4;
    const int64_t ms = mid_stride * es;
    const int64_t os = outer > 1 ? outer_stride * es : ms * mid;
    const cuuint64_t dims[3] = {(cuuint64_t)L, (cuuint64_t)mid, (cuuint64_t)outer};
    const cuuint64_t strides[2] = {(cuuint64_t)ms, (cuuint64_t)os};
    const cuuint32_t box[3] = {(cuuint32_t)kT, (cuuint32_t)rows, 1u};
    const cuuint32_t estr[3] = {1u, 1u, 1u};
    return fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3,
              const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool al16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr int kSmemLimit = 227 * 1024;
constexpr int kOneCtaSmem = 116 * 1024;

// Compute warps per CTA: the fewest that put every (batch row, channel
// block) CTA in one wave on the SMs, at most kMaxWLarge and at most what two
// stages of the input dtype leave room for in shared memory.
int choose_w(int64_t batch, int64_t dim, int num_sms, int in_bytes) {
    const int64_t units = (dim + kCW - 1) / kCW;
    int wmax = kMaxWLarge;
    while (wmax > 1 && TmLayout{wmax, 2, in_bytes}.total() > kSmemLimit) --wmax;
    int64_t w = (batch * units + num_sms - 1) / num_sms;
    if (w < 1) w = 1;
    while (w < wmax && batch * ((units + w - 1) / w) > num_sms) ++w;
    if (w > wmax) w = wmax;
    if (w > units) w = units;
    return (int)w;
}

template <typename TIn, typename TOut, int POLY8, int MAXW, bool YOUT, bool CONV = false, bool CKPT = false>
cudaError_t launch_tm(const ScanArgs &a, const TmMaps &maps, int W, int S, cudaStream_t stream) {
    const TmLayout lay{W, S, (int)sizeof(TIn)};
    static SmemOptIn opt_in;
    cudaError_t e = opt_in.ensure(
        reinterpret_cast<const void *>(scan_fwd_tmem_kernel<TIn, TOut, POLY8, MAXW, YOUT, CONV, CKPT>), kSmemLimit);
    if (e != cudaSuccess) return e;
    const int64_t blocks = a.batch * ((a.dim + lay.cwc() - 1) / lay.cwc());
    if (blocks <= 0) return cudaSuccess;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    // At least half of an SM's shared memory: one CTA per SM, so the CTA's
    // 512 tensor-memory columns are always free when it allocates them.
    const int smem = lay.total() > kOneCtaSmem ? lay.total() : kOneCtaSmem;
    scan_fwd_tmem_kernel<TIn, TOut, POLY8, MAXW, YOUT, CONV, CKPT>
        <<<(unsigned)blocks, 32 * (W + 1), smem, stream>>>(a, maps, W, S);
    return cudaGetLastError();
}

template <typename TIn, typename TOut, int POLY8, bool YOUT = true, bool CONV = false>
cudaError_t launch_w(const ScanArgs &a, const TmMaps &maps, int W, int S, cudaStream_t stream) {
    if (W <= kMaxWSmall) return launch_tm<TIn, TOut, POLY8, kMaxWSmall, YOUT, CONV>(a, maps, W, S, stream);
    if (W <= kMaxWMid) return launch_tm<TIn, TOut, POLY8, kMaxWMid, YOUT, CONV>(a, maps, W, S, stream);
    return launch_tm<TIn, TOut, POLY8, kMaxWLarge, YOUT, CONV>(a, maps, W, S, stream);
}

// Training forward of a layer wider than the 12-warp instantiation covers
// (the automatic plan's exponentials only: every one on MUFU for bf16 inputs,
// on the FMA-pipe polynomial for fp32).
template <typename TIn, typename TOut, int POLY8>
cudaError_t launch_ckpt_wide(const ScanArgs &a, const TmMaps &maps, int W, int S, cudaStream_t stream) {
    if (W <= kMaxWMid) return launch_tm<TIn, TOut, POLY8, kMaxWMid, true, false, true>(a, maps, W, S, stream);
    return launch_tm<TIn, TOut, POLY8, kMaxWLarge, true, false, true>(a, maps, W, S, stream);
}

// First pass of a sequence split (no y): the exponentials as for y.
template <typename TIn>
cudaError_t launch_pass1(const ScanArgs &a, const TmMaps &maps, int W, int S, int poly8, cudaStream_t stream) {
    return poly8 == 0 ? launch_w<TIn, float, 0, false>(a, maps, W, S, stream)
                      : launch_w<TIn, float, 8, false>(a, maps, W, S, stream);
}

template <typename TIn, typename TOut>
cudaError_t launch_poly(const ScanArgs &a, const TmMaps &maps, int W, int S, int poly8, cudaStream_t stream) {
    switch (poly8) {
        case 0: return launch_w<TIn, TOut, 0>(a, maps, W, S, stream);
        case 2: return launch_w<TIn, TOut, 2>(a, maps, W, S, stream);
        case 4: return launch_w<TIn, TOut, 4>(a, maps, W, S, stream);
        default: return launch_w<TIn, TOut, 8>(a, maps, W, S, stream);
    }
}

}  // namespace

bool scan_tmem_shape_ok(const ScanArgs &a, bool in_bf16, int out_bytes) {
    if (a.N != 16 || a.L < 8 || a.L % 8 != 0 || a.batch < 1 || a.dim < 1) return false;
    if (a.L > 0x7fffffffLL || a.dim > 0x7fffffffLL || a.batch > 0x7fffffffLL) return false;
    const int es = in_bf16 ? 2 : 4;
    const int64_t st[10] = {a.u_sd, a.u_sb, a.dl_sd, a.dl_sb, a.z_sd, a.z_sb, a.B_sn, a.B_sb, a.C_sn, a.C_sb};
    for (int i = 0; i < 5; ++i)
        if ((st[2 * i] * es) % 16 != 0 || (a.batch > 1 && (st[2 * i + 1] * es) % 16 != 0)) return false;
    return (a.y_sd * out_bytes) % 16 == 0 && (a.y_sb * out_bytes) % 16 == 0;
}

bool scan_tmem_applies(const ScanArgs &a, bool in_bf16, int out_bytes) {
    if (!scan_tmem_shape_ok(a, in_bf16, out_bytes)) return false;
    // the training forward's saved states: with y, unsplit, no conv front-end, rows
    // 16-byte aligned
    if (a.ckpt) {
        if (MS_TMEM_FUSED || a.y == nullptr || a.dsum != nullptr || a.conv_w != nullptr || !al16(a.ckpt)) return false;
    }
    if (a.conv_w && (a.y == nullptr || a.dsum != nullptr)) return false;  // the conv front-end writes y, unsplit
    // either y (and no Delta sums), or the first pass of a split: no y, the
    // Delta sums and the end states
    if (a.y ? a.dsum != nullptr : (a.dsum == nullptr || a.last == nullptr)) return false;
    if (a.dsum && (reinterpret_cast<uintptr_t>(a.dsum) & 3u)) return false;
    const void *in[5] = {a.u, a.delta, a.z, a.B, a.C};
    for (int i = 0; i < 5; ++i)
        if (in[i] != nullptr && !al16(in[i])) return false;
    if ((a.y && !al16(a.y)) || !al16(a.A) || (a.h0 && !al16(a.h0)) || (a.last && !al16(a.last))) return false;
    return encode_fn() != nullptr;
}

cudaError_t launch_scan_fwd_tmem(const ScanArgs &a, const ScanPlan &plan, bool in_bf16, bool out_bf16, int num_sms,
                                 cudaStream_t stream) {
    const int es = in_bf16 ? 2 : 4;
    const int W = choose_w(a.batch, a.dim, num_sms, es);
    int S = 3;
    while (S > 2 && TmLayout{W, S, es}.total() > kSmemLimit) --S;
    if (TmLayout{W, S, es}.total() > kSmemLimit) return cudaErrorInvalidConfiguration;
    const int rows = kCW * W;
    TmMaps maps;
    const bool zmap = a.z != nullptr;
    if (!encode3(&maps.u, a.u, in_bf16, a.L, a.dim, a.u_sd, a.batch, a.u_sb, rows) ||
        !encode3(&maps.dl, a.delta, in_bf16, a.L, a.dim, a.dl_sd, a.batch, a.dl_sb, rows) ||
        (zmap && !encode3(&maps.z, a.z, in_bf16, a.L, a.dim, a.z_sd, a.batch, a.z_sb, rows)) ||
        !encode3(&maps.B, a.B, in_bf16, a.L, 16, a.B_sn, a.batch, a.B_sb, 16) ||
        !encode3(&maps.C, a.C, in_bf16, a.L, 16, a.C_sn, a.batch, a.C_sb, 16))
        return cudaErrorInvalidValue;
    if (!zmap) maps.z = maps.u;  // never loaded
    const int poly8 = plan.poly8;
    if (a.conv_w != nullptr) {
        // the conv front-end: every exponential on MUFU for bf16 inputs, on the
        // FMA pipe for fp32 (the automatic plans)
        if (poly8 != (in_bf16 ? 0 : 8)) return cudaErrorInvalidValue;
        if (in_bf16) {
            return out_bf16 ? launch_w<__nv_bfloat16, __nv_bfloat16, 0, true, true>(a, maps, W, S, stream)
                            : launch_w<__nv_bfloat16, float, 0, true, true>(a, maps, W, S, stream);
        }
        return out_bf16 ? launch_w<float, __nv_bfloat16, 8, true, true>(a, maps, W, S, stream)
                        : launch_w<float, float, 8, true, true>(a, maps, W, S, stream);
    }
    if (a.ckpt != nullptr && W > kMaxWSmall) {
        // the training forward of a wider layer: its own instantiations, the automatic plan
        if (poly8 != (in_bf16 ? kTmemPoly8Bf16 : 8)) return cudaErrorInvalidValue;
        if (in_bf16) {
            return out_bf16 ? launch_ckpt_wide<__nv_bfloat16, __nv_bfloat16, kTmemPoly8Bf16>(a, maps, W, S, stream)
                            : launch_ckpt_wide<__nv_bfloat16, float, kTmemPoly8Bf16>(a, maps, W, S, stream);
        }
        return out_bf16 ? launch_ckpt_wide<float, __nv_bfloat16, 8>(a, maps, W, S, stream)
                        : launch_ckpt_wide<float, float, 8>(a, maps, W, S, stream);
    }
    if (a.y == nullptr)
        return in_bf16 ? launch_pass1<__nv_bfloat16>(a, maps, W, S, poly8, stream)
                       : launch_pass1<float>(a, maps, W, S, poly8, stream);
    if (in_bf16) {
        return out_bf16 ? launch_poly<__nv_bfloat16, __nv_bfloat16>(a, maps, W, S, poly8, stream)
                        : launch_poly<__nv_bfloat16, float>(a, maps, W, S, poly8, stream);
    }
    return out_bf16 ? launch_poly<float, __nv_bfloat16>(a, maps, W, S, poly8, stream)
                    : launch_poly<float, float>(a, maps, W, S, poly8, stream);
}

}  // namespace ms
