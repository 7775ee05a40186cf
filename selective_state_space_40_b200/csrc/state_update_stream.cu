// state_update_stream.cu -- selective state update (decode) as a bulk-copy
// stream on sm_100a.
//
// Same step as state_update.cu (one token from the stored fp32 state; blog
// 'Mamba-1/2/3 Markdown図解', section 2: generation is the recurrent update of
// the same model), organised for HBM streaming: a persistent CTA walks tiles
// of kTC consecutive channels of one batch row. The tile's state rows (kTC x 64
// bytes) and its x, delta, z values arrive by bulk copies (TMA engine) into a
// ring of kStages shared-memory stages tracked by mbarriers; the compute
// threads update the state in place in shared memory; a producer warp writes
// the state and y back by bulk copies once every compute warp is done with a
// stage, and refills the stage once those stores have read it. Loads run up
// to kStages tiles ahead, so the copy engine, not the threads, keeps the HBM
// requests in flight, and no compute thread waits on the store path. No
// cluster multicast is used.
//
// Used when the state rows are dense (16 fp32 per channel, 16-byte aligned),
// d_state is 16, dim is a multiple of kTC and every row start is 16-byte
// aligned; otherwise state_update.cu runs.

#include <cstdint>

#include "mambascan.h"
#include "ms_device.cuh"
#include "ms_internal.h"

namespace ms {

namespace {

// Tile size, block size and ring depth (compile-time; defaults measured best).
#ifndef MS_STREAM_TC
#define MS_STREAM_TC 128
#endif
#ifndef MS_STREAM_THREADS
#define MS_STREAM_THREADS 256
#endif
#ifndef MS_STREAM_STAGES
#define MS_STREAM_STAGES 4
#endif
constexpr int kTC = MS_STREAM_TC;                    // channels per tile
constexpr int kComputeThreads = MS_STREAM_THREADS;   // 4 lanes per channel
constexpr int kThreads = kComputeThreads + 32;       // + one producer warp
constexpr int kStages = MS_STREAM_STAGES;
static_assert(kTC * 4 % kComputeThreads == 0, "whole channels per pass");
constexpr uint32_t kSpinLimit = 1u << 20;  // try_wait rounds before giving up

__device__ __forceinline__ uint32_t saddr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(saddr(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(saddr(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(saddr(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_wait_n(uint64_t *bar, uint32_t parity, uint32_t limit) {
    const uint32_t a = saddr(bar);
    for (uint32_t i = 0; i < limit; ++i) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(a), "r"(parity)
            : "memory");
        if (done) return true;
    }
    return false;
}
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity) { return mbar_wait_n(bar, parity, kSpinLimit); }
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            saddr(dst)),
        "l"(src), "r"(bytes), "r"(saddr(bar))
        : "memory");
}
__device__ __forceinline__ void bulk_store(void *dst, const void *src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(saddr(src)),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until at most N committed store groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

template <typename TIn, typename TOut>
struct StreamSmem {
    static constexpr int kStateBytes = kTC * 16 * 4;
    static constexpr int kInBytes = kTC * (int)sizeof(TIn);
    static constexpr int kYBytes = kTC * (int)sizeof(TOut);
    static constexpr int kStageBytes = kStateBytes + 3 * kInBytes + ((kYBytes + 15) & ~15);
    static constexpr int kOffStages = 128;  // mbarriers first (full[kStages], done[kStages])
    static constexpr int kTotal = kOffStages + kStages * kStageBytes;
};

template <typename TIn, typename TOut>
__global__ void __launch_bounds__(kThreads)
state_update_stream_kernel(const UpdateArgs a) {
    using Sm = StreamSmem<TIn, TOut>;
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem);  // stage s loaded
    uint64_t *done = full + kStages;                       // stage s computed (one arrival per compute warp)
    auto stage = [&](int s) { return smem + Sm::kOffStages + s * Sm::kStageBytes; };

    const int64_t tiles_per_row = a.dim / kTC;
    const int64_t ntiles = a.batch * tiles_per_row;
    // this CTA's tiles: blockIdx.x, blockIdx.x + gridDim.x, ...
    const int64_t my_tiles = blockIdx.x < ntiles ? (ntiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    auto tile_of = [&](int64_t i) { return (int64_t)blockIdx.x + i * (int64_t)gridDim.x; };
    const bool has_z = a.z != nullptr;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int q = lane & 3;        // states 4q..4q+3
    const int n0 = 4 * q;

    // Bytes of one tile's loads (state + x + delta [+ z]).
    const uint32_t tile_bytes = Sm::kStateBytes + (has_z ? 3 : 2) * Sm::kInBytes;

    auto issue = [&](int s, int64_t tile) {
        const int64_t b = tile / tiles_per_row;
        const int64_t d0 = (tile % tiles_per_row) * kTC;
        unsigned char *st = stage(s);
        mbar_arrive_expect_tx(&full[s], tile_bytes);
        bulk_load(st, a.state + b * a.st_sb + d0 * 16, Sm::kStateBytes, &full[s]);
        bulk_load(st + Sm::kStateBytes, static_cast<const TIn *>(a.x) + b * a.x_sb + d0, Sm::kInBytes, &full[s]);
        bulk_load(st + Sm::kStateBytes + Sm::kInBytes, static_cast<const TIn *>(a.delta) + b * a.dl_sb + d0,
                  Sm::kInBytes, &full[s]);
        if (has_z)
            bulk_load(st + Sm::kStateBytes + 2 * Sm::kInBytes, static_cast<const TIn *>(a.z) + b * a.z_sb + d0,
                      Sm::kInBytes, &full[s]);
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&done[s], kComputeThreads / 32);
        }
        fence_mbar_init();
    }
    // Back-to-back steps: this grid may have been launched while the previous
    // kernel on the stream still runs (programmatic dependent launch). Let the
    // next step's grid get scheduled now, and wait here until everything the
    // previous kernel wrote (the state) is complete and visible. Without that
    // launch attribute both instructions do nothing.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    __syncthreads();

    if (warp == kComputeThreads / 32) {
        // ---- producer warp (lane 0): loads run kStages tiles ahead; a tile's
        // state and y go back by bulk stores once every compute warp is done
        // with it, and its stage is refilled once those stores have read it.
        if (lane == 0) {
            int64_t issued = 0, stored = 0;
            for (; issued < kStages && issued < my_tiles; ++issued) issue((int)issued, tile_of(issued));
            bool ok = true;
            for (int64_t i = 0; i < my_tiles; ++i) {
                const int s = (int)(i % kStages);
                ok = mbar_wait(&done[s], (uint32_t)((i / kStages) & 1));
                if (!ok) break;
                const int64_t tile = tile_of(i);
                const int64_t b = tile / tiles_per_row;
                const int64_t d0 = (tile % tiles_per_row) * kTC;
                unsigned char *st = stage(s);
                bulk_store(a.state + b * a.st_sb + d0 * 16, st, Sm::kStateBytes);
                bulk_store(static_cast<TOut *>(a.y) + b * a.y_sb + d0, st + Sm::kStateBytes + 3 * Sm::kInBytes,
                           Sm::kYBytes);
                bulk_commit();
                stored = i + 1;
                if (issued < my_tiles) {
                    bulk_wait_read<0>();  // this stage's stores have read it
                    issue(s, tile_of(issued));
                    ++issued;
                }
            }
            if (!ok) {
                if (a.status) atomicOr(a.status, MS_ERR_TIMEOUT);
                // Drain (bounded) the loads this CTA may still have in flight.
                for (int64_t k = stored; k < issued; ++k)
                    mbar_wait(&full[k % kStages], (uint32_t)((k / kStages) & 1));
            }
            bulk_wait_all();
        }
        return;
    }

    // ---- compute warps: 4 lanes per channel, 4 states each
    for (int64_t i = 0; i < my_tiles; ++i) {
        const int s = (int)(i % kStages);
        const int64_t tile = tile_of(i);
        const int64_t b = tile / tiles_per_row;
        const int64_t d0 = (tile % tiles_per_row) * kTC;
        // the tile's parameters (global, L2-resident) load while the stage may still be in flight
        float Bv[4], Cv[4];
        {
            const TIn *Bb = static_cast<const TIn *>(a.B) + b * a.B_sb + n0;
            const TIn *Cb = static_cast<const TIn *>(a.C) + b * a.C_sb + n0;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                Bv[k] = Elem<TIn>::load(Bb + k);
                Cv[k] = Elem<TIn>::load(Cb + k);
            }
        }
        constexpr int kHalves = kTC * 4 / kComputeThreads;
        float4 Av[kHalves];
        float biasv[kHalves], Dv[kHalves];
#pragma unroll
        for (int half = 0; half < kHalves; ++half) {
            const int64_t d = d0 + (threadIdx.x >> 2) + half * (kComputeThreads / 4);
            Av[half] = __ldg(reinterpret_cast<const float4 *>(a.A + d * 16 + n0));
            biasv[half] = a.bias ? __ldg(a.bias + d) : 0.0f;
            Dv[half] = a.D ? __ldg(a.D + d) : 0.0f;
        }
        const bool ok = __all_sync(0xffffffffu, mbar_wait(&full[s], (uint32_t)((i / kStages) & 1)));
        if (!ok) {
            if (lane == 0 && a.status) atomicOr(a.status, MS_ERR_TIMEOUT);
            break;
        }
        unsigned char *st = stage(s);
        float *sstate = reinterpret_cast<float *>(st);
        const TIn *sx = reinterpret_cast<const TIn *>(st + Sm::kStateBytes);
        const TIn *sdl = sx + kTC;
        const TIn *sz = sdl + kTC;
        TOut *sy = reinterpret_cast<TOut *>(st + Sm::kStateBytes + 3 * Sm::kInBytes);
        // Per-channel scalars are evaluated once per warp instruction stream: lane
        // (slot, q) takes Delta = softplus(delta + bias) of its slot's channel in
        // half q % kHalves and the quad reads each half's value by shuffle; after
        // the state update, lane q < kHalves finishes half q's y (D x, silu(z)).
        static_assert(kHalves <= 4, "one lane of the quad per half");
        float dt_mine;
        {
            const int hm = q % kHalves;
            float bias_m = biasv[0];
#pragma unroll
            for (int hh = 1; hh < kHalves; ++hh)
                if (hm == hh) bias_m = biasv[hh];
            const int clm = (threadIdx.x >> 2) + hm * (kComputeThreads / 4);
            const float v = (MS_CHECK(a.status, clm < kTC) ? to_f32(sdl[clm]) : 0.0f) + bias_m;
            dt_mine = a.softplus ? softplus_f(v) : v;
        }
        float accs[kHalves], xs[kHalves];
#pragma unroll
        for (int half = 0; half < kHalves; ++half) {
            const int cl = (threadIdx.x >> 2) + half * (kComputeThreads / 4);  // channel within the tile
            const int64_t d = d0 + cl;
            const float dt = __shfl_sync(0xffffffffu, dt_mine, (lane & ~3) | half);
            accs[half] = 0.0f;
            xs[half] = 0.0f;
            if (!MS_CHECK(a.status, cl < kTC && d < a.dim)) continue;
            float4 hv = *reinterpret_cast<const float4 *>(sstate + cl * 16 + n0);
            float h[4] = {hv.x, hv.y, hv.z, hv.w};
            const float A[4] = {Av[half].x, Av[half].y, Av[half].z, Av[half].w};
            const float x = to_f32(sx[cl]);
            const float dx = dt * x;
            const float dtl = dt * kLog2e;
            float acc = 0.0f;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                h[k] = fmaf(exp2_mufu(dtl * A[k]), h[k], dx * Bv[k]);
                acc = fmaf(Cv[k], h[k], acc);
            }
            acc += __shfl_xor_sync(0xffffffffu, acc, 1);
            acc += __shfl_xor_sync(0xffffffffu, acc, 2);
            *reinterpret_cast<float4 *>(sstate + cl * 16 + n0) = make_float4(h[0], h[1], h[2], h[3]);
            accs[half] = acc;
            xs[half] = x;
        }
        if (q < kHalves) {
            float acc = accs[0], x = xs[0], Dh = Dv[0];
#pragma unroll
            for (int hh = 1; hh < kHalves; ++hh)
                if (q == hh) {
                    acc = accs[hh];
                    x = xs[hh];
                    Dh = Dv[hh];
                }
            const int cl = (threadIdx.x >> 2) + q * (kComputeThreads / 4);
            if (MS_CHECK(a.status, cl < kTC && d0 + cl < a.dim)) {
                float yv = acc + Dh * x;
                if (has_z) yv *= silu_f(to_f32(sz[cl]));
                Elem<TOut>::store(sy + cl, yv);
            }
        }
        fence_proxy_async();  // this thread's shared writes -> visible to the copy engine
        __syncwarp();
        if (lane == 0) mbar_arrive(&done[s]);
    }
}

template <typename TIn, typename TOut>
cudaError_t launch_t(const UpdateArgs &a, cudaStream_t stream) {
    using Sm = StreamSmem<TIn, TOut>;
    static SmemOptIn opt_in;
    cudaError_t e = opt_in.ensure(reinterpret_cast<const void *>(state_update_stream_kernel<TIn, TOut>), Sm::kTotal);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148, per_sm = 1;
    e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, state_update_stream_kernel<TIn, TOut>, kThreads,
                                                  Sm::kTotal);
    if (per_sm < 1) per_sm = 1;
    const int64_t ntiles = a.batch * (a.dim / kTC);
    const int64_t grid = ntiles < (int64_t)sms * per_sm ? ntiles : (int64_t)sms * per_sm;
    if (grid <= 0) return cudaSuccess;
    // programmatic dependent launch: the grid is scheduled while the previous
    // kernel on the stream drains; the kernel waits (griddepcontrol.wait)
    // before it reads any memory
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = Sm::kTotal;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, state_update_stream_kernel<TIn, TOut>, a);
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

namespace {

// Test hook for the timeout path: one thread waits, with the bounded wait the
// stream kernel uses, on a barrier that nothing completes (no arrival is ever
// made); when the wait gives up it records MS_ERR_TIMEOUT and the kernel ends.
__global__ void bounded_wait_probe_kernel(int *status, uint32_t rounds) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
        if (!mbar_wait_n(&bar, 0, rounds)) atomicOr(status, MS_ERR_TIMEOUT);
    }
}

}  // namespace

#ifdef MS_DEBUG
namespace {
__device__ int g_bounds_probe[16];
__global__ void bounds_probe_kernel(int index, int *status) {
    if (MS_CHECK(status, index >= 0 && index < 16)) g_bounds_probe[index] = index + 1;
}
}  // namespace

cudaError_t launch_bounds_probe(int index, int *status, cudaStream_t stream) {
    bounds_probe_kernel<<<1, 1, 0, stream>>>(index, status);
    return cudaGetLastError();
}
#endif

cudaError_t launch_bounded_wait_probe(int *status, uint32_t rounds, cudaStream_t stream) {
    bounded_wait_probe_kernel<<<1, 32, 0, stream>>>(status, rounds);
    return cudaGetLastError();
}

bool state_update_stream_applies(const UpdateArgs &a, int in_bytes, int out_bytes) {
    if (a.N != 16 || a.st_sd != 16 || a.dim % kTC != 0) return false;
    if (!aligned16(a.state) || (a.st_sb * 4) % 16 != 0) return false;
    const void *rows[4] = {a.x, a.delta, a.z, a.y};
    const int64_t sbs[4] = {a.x_sb, a.dl_sb, a.z_sb, a.y_sb};
    const int es[4] = {in_bytes, in_bytes, in_bytes, out_bytes};
    for (int k = 0; k < 4; ++k) {
        if (rows[k] == nullptr) continue;
        if (!aligned16(rows[k]) || (sbs[k] * es[k]) % 16 != 0) return false;
    }
    return aligned16(a.A);
}

cudaError_t launch_state_update_stream(const UpdateArgs &a, bool in_bf16, bool out_bf16, cudaStream_t stream) {
    if (in_bf16) {
        return out_bf16 ? launch_t<__nv_bfloat16, __nv_bfloat16>(a, stream)
                        : launch_t<__nv_bfloat16, float>(a, stream);
    }
    return out_bf16 ? launch_t<float, __nv_bfloat16>(a, stream) : launch_t<float, float>(a, stream);
}

}  // namespace ms
