// ssd_update.cu -- Mamba-2 SSD layer, one-token state update (decode) on sm_100a.
//
// 'Mamba-1/2/3 Markdown図解' blog, section 3: decoding runs the recurrent view
// of the SSD model, one state update per token. For batch row b and head h
// (state S [P x N] fp32, group g of B and C):
//   Delta = softplus(dt + dt_bias),  S = exp(Delta A_h) S + Delta x B^T,
//   y = S C + D x
// The state is read and written once (the step's traffic); one CTA of 8
// warps per (b, h): lane l owns columns n in [4l, 4l+4) (one 16-byte access
// per row), warps stride over the rows p with every row's load in flight at
// once, and each row's readout C . S is a warp sum. Back-to-back steps overlap
// through programmatic dependent launch.

#include <cstdint>

#include "ms_device.cuh"
#include "ms_internal.h"

namespace ms {

namespace {

constexpr int kUW = 8;  // warps per CTA

template <typename T>
__device__ __forceinline__ float ldv(const T *p) {
    if constexpr (sizeof(T) == 4) return __ldg(reinterpret_cast<const float *>(p));
    else return bf16_bits_to_f32(__ldg(reinterpret_cast<const unsigned short *>(p)));
}

constexpr int kRowsPerWarp = 8;  // rows of the state a warp has in flight (P <= 64)

template <typename TIn, typename TOut>
__global__ void __launch_bounds__(kUW * 32) ssd_update_kernel(const SsdUpdArgs a) {
    // Back-to-back steps: this grid may have been scheduled while the previous
    // kernel on the stream still runs (programmatic dependent launch). Let the
    // next grid be scheduled, and wait until everything the previous kernel wrote
    // is complete and visible before reading any memory. Without that launch
    // attribute both instructions do nothing.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t b = blockIdx.x / a.H, h = blockIdx.x % a.H;
    const int64_t g = h / (a.H / a.G);
    const int P = a.P;
    constexpr int N = 128;
    // debug build: the grid covers exactly batch x H, and g names one of the G groups
    if (!MS_CHECK(a.status, b < a.batch && g < a.G)) return;
    const float v = ldv(static_cast<const TIn *>(a.dt) + b * a.dt_sb + h) + (a.dt_bias ? __ldg(a.dt_bias + h) : 0.0f);
    const float dl = a.softplus ? softplus_f(v) : v;
    const float decay = exp2_mufu(dl * __ldg(a.A + h) * kLog2e);
    const float Dh = a.D ? __ldg(a.D + h) : 0.0f;
    const TIn *Bp = static_cast<const TIn *>(a.B) + b * a.B_sb + g * a.B_sg + 4 * lane;
    const TIn *Cp = static_cast<const TIn *>(a.C) + b * a.C_sb + g * a.C_sg + 4 * lane;
    float Bv[4], Cv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        Bv[i] = dl * ldv(Bp + i);
        Cv[i] = ldv(Cp + i);
    }
    const TIn *xr = static_cast<const TIn *>(a.x) + b * a.x_sb + h * a.x_sh;
    TOut *yr = static_cast<TOut *>(a.y) + b * a.y_sb + h * a.y_sh;
    float *st = a.state + b * a.st_sb + h * a.st_sh + 4 * lane;
    // rows p = warp + kUW i; every load of the warp's rows issued before any store
    for (int p0 = warp; p0 < P; p0 += kUW * kRowsPerWarp) {
        float4 sv[kRowsPerWarp];
        float xv[kRowsPerWarp];
#pragma unroll
        for (int i = 0; i < kRowsPerWarp; ++i) {
            const int p = p0 + kUW * i;
            if (p < P) {
                sv[i] = *reinterpret_cast<const float4 *>(st + (int64_t)p * N);
                xv[i] = ldv(xr + p);
            }
        }
        float part[kRowsPerWarp];
#pragma unroll
        for (int i = 0; i < kRowsPerWarp; ++i) {
            const int p = p0 + kUW * i;
            part[i] = 0.0f;
            if (p < P) {
                float4 s = sv[i];
                s.x = fmaf(decay, s.x, xv[i] * Bv[0]);
                s.y = fmaf(decay, s.y, xv[i] * Bv[1]);
                s.z = fmaf(decay, s.z, xv[i] * Bv[2]);
                s.w = fmaf(decay, s.w, xv[i] * Bv[3]);
                *reinterpret_cast<float4 *>(st + (int64_t)p * N) = s;
                part[i] = Cv[0] * s.x + Cv[1] * s.y + Cv[2] * s.z + Cv[3] * s.w;
            }
        }
        // the rows' readouts summed over the warp by a reduce-scatter: lanes with
        // bit 4 keep rows 4..7 and pass 0..3 (then bits 3, 2 halve the rest), the
        // last two levels sum within groups of 4 lanes; lane l ends with the sum
        // of row r = 4 b4 + 2 b3 + b2 (b = the bits of l)
        static_assert(kRowsPerWarp == 8, "reduce-scatter of 8 rows over 32 lanes");
#pragma unroll
        for (int lvl = 0; lvl < 3; ++lvl) {
            const int w = 4 >> lvl;                 // values kept after this level
            const bool hi = (lane >> (4 - lvl)) & 1;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                if (j < w) {
                    const float send = hi ? part[j] : part[w + j];
                    const float keep = hi ? part[w + j] : part[j];
                    part[j] = keep + __shfl_xor_sync(0xffffffffu, send, 16 >> lvl);
                }
            }
        }
        part[0] += __shfl_xor_sync(0xffffffffu, part[0], 2);
        part[0] += __shfl_xor_sync(0xffffffffu, part[0], 1);
        const int r = ((lane >> 4) & 1) * 4 + ((lane >> 3) & 1) * 2 + ((lane >> 2) & 1);
        float xr_ = xv[0];
#pragma unroll
        for (int i = 1; i < kRowsPerWarp; ++i)
            if (r == i) xr_ = xv[i];
        const int pr = p0 + kUW * r;
        if ((lane & 3) == 0 && pr < P && MS_CHECK(a.status, r < kRowsPerWarp))
            Elem<TOut>::store(yr + pr, part[0] + Dh * xr_);
    }
}

template <typename TIn, typename TOut>
cudaError_t launch_t(const SsdUpdArgs &a, cudaStream_t stream) {
    const int64_t blocks = a.batch * a.H;
    if (blocks <= 0) return cudaSuccess;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    // programmatic dependent launch: the grid is scheduled while the previous
    // kernel on the stream drains; the kernel waits (griddepcontrol.wait) before
    // it reads any memory
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)blocks);
    cfg.blockDim = dim3(kUW * 32);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, ssd_update_kernel<TIn, TOut>, a);
}

}  // namespace

cudaError_t launch_ssd_update(const SsdUpdArgs &a, bool in_bf16, bool out_bf16, cudaStream_t stream) {
    if (in_bf16) return out_bf16 ? launch_t<__nv_bfloat16, __nv_bfloat16>(a, stream)
                                 : launch_t<__nv_bfloat16, float>(a, stream);
    return out_bf16 ? launch_t<float, __nv_bfloat16>(a, stream) : launch_t<float, float>(a, stream);
}

}  // namespace ms
