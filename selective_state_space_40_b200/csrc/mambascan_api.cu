// mambascan_api.cu -- the extern "C" entry points of libmambascan.so: host-side
// argument checks, launch planning and status codes. The operations are
// described in include/mambascan.h.

#include <climits>
#include <cstdint>
#include <mutex>
#include <cuda_runtime.h>

#include "mambascan.h"
#include "ms_internal.h"

static_assert(MS_CKPT_TOKENS == ms::kCkptTokens, "saved-state interval of the ABI and the kernels");

// Fixed scratch of mamba_scan_bwd_noalloc: saved states recomputed by the
// backward (one copy per device, placed by the module loader; never freed).
static __device__ __align__(256) unsigned char g_bwd_scratch[MS_BWD_NOALLOC_MAX_BYTES];

namespace {

bool aligned(const void *p, size_t n) { return (reinterpret_cast<uintptr_t>(p) % n) == 0; }

// Largest element offset b*sb + d*sd + t for the given extents, or -1 on
// int64 overflow (extents are >= 1 here, strides >= 0).
int64_t max_offset3(int64_t n0, int64_t s0, int64_t n1, int64_t s1, int64_t n2) {
    __int128 o = (__int128)(n0 - 1) * s0 + (__int128)(n1 - 1) * s1 + (n2 - 1);
    if (o > (__int128)INT64_MAX / 4) return -1;
    return (int64_t)o;
}

int elem_bytes(int32_t dt) { return dt == MS_BF16 ? 2 : 4; }

int num_sms_current() {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms > 0 ? sms : 148;
}

bool vec_ok(const void *p, int64_t sb, int64_t sd, int es) {
    return p == nullptr || (aligned(p, 16) && (sb * es) % 16 == 0 && (sd * es) % 16 == 0);
}

}  // namespace

namespace ms {

namespace {
using PfnCtxGetCurrent = int (*)(void **);
using PfnCtxGetId = int (*)(void *, unsigned long long *);
PfnCtxGetCurrent g_ctx_get_current = nullptr;
PfnCtxGetId g_ctx_get_id = nullptr;
std::once_flag g_ctx_fns_once;
}  // namespace

uint64_t current_context_id() {
    std::call_once(g_ctx_fns_once, [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &f, 12000, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_ctx_get_current = reinterpret_cast<PfnCtxGetCurrent>(f);
        f = nullptr;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &f, 12000, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_ctx_get_id = reinterpret_cast<PfnCtxGetId>(f);
        cudaGetLastError();
    });
    if (!g_ctx_get_current || !g_ctx_get_id) return 0;
    void *ctx = nullptr;
    if (g_ctx_get_current(&ctx) != 0 || ctx == nullptr) return 0;
    unsigned long long id = 0;
    if (g_ctx_get_id(ctx, &id) != 0) return 0;
    return (uint64_t)id + 1;
}

cudaError_t SmemOptIn::ensure(const void *func, int bytes) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t ctx = current_context_id();
    if (ctx != 0 && dev >= 0 && dev < 64 && ctx_[dev].load(std::memory_order_acquire) == ctx) return cudaSuccess;
    e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    // the attribute call has made the device's primary context current
    const uint64_t now = current_context_id();
    if (now != 0 && dev >= 0 && dev < 64) ctx_[dev].store(now, std::memory_order_release);
    return cudaSuccess;
}

}  // namespace ms

extern "C" {

const char *mamba_status_string(int code) {
    switch (code) {
        case MS_OK: return "ok";
        case MS_ERR_NULL: return "a required pointer is NULL";
        case MS_ERR_DTYPE: return "unsupported dtype code";
        case MS_ERR_SHAPE: return "invalid sizes (negative, dstate outside [1,16], or offset overflow)";
        case MS_ERR_STRIDE: return "negative stride";
        case MS_ERR_ALIGN: return "pointer not aligned to its element size";
        case MS_ERR_WORKSPACE: return "workspace argument inconsistent";
        case MS_ERR_CUDA: return "CUDA runtime error (no device or launch failure)";
        case MS_ERR_TIMEOUT: return "device wait timed out";
        case MS_ERR_DEVICE: return "device is not compute capability 10.0";
        case MS_ERR_SCRATCH: return "needs more scratch than the library's fixed buffer holds";
        case MS_ERR_BOUNDS: return "a device bounds check failed (debug build)";
        default: return "unknown status code";
    }
}

int mamba_debug_bounded_wait(uint32_t rounds, int *dev_status, ms_stream_t stream) {
    if (!dev_status) return MS_ERR_NULL;
    if (rounds < 1 || rounds > (1u << 20)) return MS_ERR_SHAPE;
    if (!aligned(dev_status, 4)) return MS_ERR_ALIGN;
    if (ms::launch_bounded_wait_probe(dev_status, rounds, (cudaStream_t)stream) != cudaSuccess) {
        cudaGetLastError();
        return MS_ERR_CUDA;
    }
    return MS_OK;
}

int mamba_debug_build(void) {
#ifdef MS_DEBUG
    return 1;
#else
    return 0;
#endif
}

int mamba_debug_bounds_probe(int32_t index, int *dev_status, ms_stream_t stream) {
    if (!dev_status) return MS_ERR_NULL;
    if (!aligned(dev_status, 4)) return MS_ERR_ALIGN;
#ifdef MS_DEBUG
    if (ms::launch_bounds_probe(index, dev_status, (cudaStream_t)stream) != cudaSuccess) {
        cudaGetLastError();
        return MS_ERR_CUDA;
    }
    return MS_OK;
#else
    (void)index;
    (void)stream;
    return MS_ERR_SHAPE;
#endif
}

int mamba_device_check(void) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return MS_ERR_CUDA;
    }
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
        cudaGetLastError();
        return MS_ERR_CUDA;
    }
    return (major == 10 && minor == 0) ? MS_OK : MS_ERR_DEVICE;
}

static int check_scan(const void *u, const void *delta, const float *A, const void *B, const void *C,
                      const float *D, const void *z, const float *delta_bias, const float *h0, void *y,
                      float *last, const ms_scan_dims *dm) {
    if (!dm) return MS_ERR_NULL;
    if ((dm->in_dtype != MS_F32 && dm->in_dtype != MS_BF16) ||
        (dm->out_dtype != MS_F32 && dm->out_dtype != MS_BF16))
        return MS_ERR_DTYPE;
    if (dm->batch < 0 || dm->dim < 0 || dm->seqlen < 0 || dm->dstate < 1 || dm->dstate > MS_MAX_DSTATE)
        return MS_ERR_SHAPE;
    if (dm->u_sb < 0 || dm->u_sd < 0 || dm->delta_sb < 0 || dm->delta_sd < 0 || dm->z_sb < 0 ||
        dm->z_sd < 0 || dm->y_sb < 0 || dm->y_sd < 0 || dm->B_sb < 0 || dm->B_sn < 0 || dm->C_sb < 0 ||
        dm->C_sn < 0)
        return MS_ERR_STRIDE;
    const bool channels = dm->batch > 0 && dm->dim > 0;
    if (!channels) return MS_OK;
    if (!A) return MS_ERR_NULL;
    if (dm->seqlen > 0 && (!u || !delta || !B || !C || !y)) return MS_ERR_NULL;
    const int ei = elem_bytes(dm->in_dtype), eo = elem_bytes(dm->out_dtype);
    if (!aligned(u, ei) || !aligned(delta, ei) || !aligned(B, ei) || !aligned(C, ei) ||
        (z && !aligned(z, ei)) || !aligned(y, eo) || !aligned(A, 4) || (D && !aligned(D, 4)) ||
        (delta_bias && !aligned(delta_bias, 4)) || (h0 && !aligned(h0, 4)) || (last && !aligned(last, 4)))
        return MS_ERR_ALIGN;
    if (dm->seqlen > 0) {
        const int64_t L = dm->seqlen;
        if (max_offset3(dm->batch, dm->u_sb, dm->dim, dm->u_sd, L) < 0 ||
            max_offset3(dm->batch, dm->delta_sb, dm->dim, dm->delta_sd, L) < 0 ||
            max_offset3(dm->batch, dm->z_sb, dm->dim, dm->z_sd, L) < 0 ||
            max_offset3(dm->batch, dm->y_sb, dm->dim, dm->y_sd, L) < 0 ||
            max_offset3(dm->batch, dm->B_sb, dm->dstate, dm->B_sn, L) < 0 ||
            max_offset3(dm->batch, dm->C_sb, dm->dstate, dm->C_sn, L) < 0)
            return MS_ERR_SHAPE;
    }
    if (max_offset3(dm->batch, dm->dim * dm->dstate, dm->dim, dm->dstate, dm->dstate) < 0)
        return MS_ERR_SHAPE;
    return MS_OK;
}

// Sequence split for layers with too few channels to fill the GPU: S
// segments of Ls tokens per batch row (the last one may be shorter). S = 1:
// no split. Each batch row is split on its own, so the parallel work of one
// pass is (S - 1) or S segments x dim channels.
struct SplitPlan {
    int64_t S, Ls;
};

static SplitPlan split_plan(const ms_scan_dims *d, int num_sms) {
    SplitPlan sp{1, d->seqlen};
    const int64_t ch = d->batch * d->dim, L = d->seqlen;
    if (ch <= 0 || d->dim <= 0 || L < 8192 || ch * 4 / 32 >= (int64_t)num_sms * 8) return sp;
    const int64_t target_warps = (int64_t)num_sms * 12;  // at 4 lanes per channel
    int64_t S0 = (target_warps * 8 + d->dim - 1) / d->dim;
    const int64_t cap = L / 1024 < 256 ? L / 1024 : 256;
    S0 = S0 > cap ? cap : S0;
    if (S0 < 2) return sp;
    // prefer a count that cuts L into equal segments of whole 64-token multiples
    for (int64_t s = S0; s <= 2 * S0 && s <= cap; ++s) {
        if (L % s == 0 && (L / s) % 64 == 0) {
            sp.S = s;
            sp.Ls = L / s;
            return sp;
        }
    }
    sp.Ls = ((L + S0 - 1) / S0 + 63) / 64 * 64;
    sp.S = (L + sp.Ls - 1) / sp.Ls;
    if (sp.S < 2) return SplitPlan{1, L};
    return sp;
}

// Workspace of a split, in floats per batch row (reused row after row): end
// states E [S-1, dim, N], Delta sums [S-1, dim], initial states Sin [S, dim,
// N], last states of the segments [S, dim, N]; each region 16-byte aligned.
static int64_t round4(int64_t v) { return (v + 3) / 4 * 4; }
static int64_t split_ws_floats(const ms_scan_dims *d, const SplitPlan &sp) {
    if (sp.S < 2) return 0;
    const int64_t cn = d->dim * d->dstate;
    return round4((sp.S - 1) * cn) + round4((sp.S - 1) * d->dim) + round4(sp.S * cn) + round4(sp.S * cn);
}

size_t mamba_scan_workspace_size(const ms_scan_dims *dims) {
    if (!dims || dims->dstate < 1 || dims->dstate > MS_MAX_DSTATE) return 0;
    const SplitPlan sp = split_plan(dims, num_sms_current());
    return (size_t)split_ws_floats(dims, sp) * sizeof(float);
}

static bool plan_valid(const ms_scan_plan *p) {
    const int g = p->lanes_per_channel, c = p->chunks_per_lane, q = p->poly8, e = p->engine;
    if (e == MS_ENGINE_TMEM) return g == 4 && c == 1 && (q == 0 || q == 2 || q == 4 || q == 8);
    return e == MS_ENGINE_REGISTER && (g == 1 || g == 2 || g == 4 || g == 8) && (c == 1 || (c == 2 && g != 8)) &&
           (q == 0 || q == 2 || q == 4 || q == 8);
}

// The plan a call without an explicit plan runs: the tensor-memory kernel
// where it applies (sizes, strides, alignment and outputs), else the
// register-prefetch kernel with its own heuristic.
static ms::ScanPlan auto_plan_args(const ms::ScanArgs &a, bool in_bf16, bool out_bf16, bool check_pointers) {
    ms::ScanPlan pl = ms::plan_scan(a, in_bf16, num_sms_current());
    const int eo = out_bf16 ? 2 : 4;
    if (check_pointers ? ms::scan_tmem_applies(a, in_bf16, eo) : ms::scan_tmem_shape_ok(a, in_bf16, eo)) {
        pl.engine = MS_ENGINE_TMEM;
        pl.lanes_per_channel = 4;
        pl.chunks_per_lane = 1;
        pl.poly8 = in_bf16 ? ms::kTmemPoly8Bf16 : 8;
    }
    return pl;
}

static ms::ScanArgs dims_args(const ms_scan_dims *dims) {
    ms::ScanArgs a{};
    a.batch = dims->batch;
    a.dim = dims->dim;
    a.L = dims->seqlen;
    a.N = (int)dims->dstate;
    a.u_sb = dims->u_sb; a.u_sd = dims->u_sd;
    a.dl_sb = dims->delta_sb; a.dl_sd = dims->delta_sd;
    a.z_sb = dims->z_sb; a.z_sd = dims->z_sd;
    a.y_sb = dims->y_sb; a.y_sd = dims->y_sd;
    a.B_sb = dims->B_sb; a.B_sn = dims->B_sn; a.C_sb = dims->C_sb; a.C_sn = dims->C_sn;
    return a;
}

static ms::ScanPlan auto_plan(const ms_scan_dims *dims) {
    return auto_plan_args(dims_args(dims), dims->in_dtype == MS_BF16, dims->out_dtype == MS_BF16, false);
}

int mamba_scan_choose_plan(const ms_scan_dims *dims, ms_scan_plan *plan) {
    if (!dims || !plan) return MS_ERR_NULL;
    int rc = check_scan(nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                        nullptr, nullptr, dims);
    if (rc != MS_OK && rc != MS_ERR_NULL) return rc;
    const ms::ScanPlan p = auto_plan(dims);
    plan->lanes_per_channel = p.lanes_per_channel;
    plan->chunks_per_lane = p.chunks_per_lane;
    plan->poly8 = p.poly8;
    plan->engine = p.engine;
    return MS_OK;
}

int mamba_scan_fwd(const void *u, const void *delta, const float *A, const void *B, const void *C,
                   const float *D, const void *z, const float *delta_bias, int softplus_flag,
                   const float *initial_state, void *y, float *last_state, const ms_scan_dims *dims,
                   void *workspace, size_t workspace_bytes, int *dev_status, ms_stream_t stream) {
    return mamba_scan_fwd_plan(u, delta, A, B, C, D, z, delta_bias, softplus_flag, initial_state, y,
                               last_state, dims, workspace, workspace_bytes, dev_status, stream, nullptr);
}

// Conv front-end arguments of mamba_conv_scan_fwd (all null for the plain scan).
struct ConvIn {
    const float *w, *b;
    const void *x0;
    void *u_out;
    const ms_conv_dims *cd;
};

static int check_conv(const ConvIn &cv, const ms_scan_dims *dm) {
    if (!cv.cd) return MS_ERR_NULL;
    const ms_conv_dims *cd = cv.cd;
    if (cd->width < 1 || cd->width > 4) return MS_ERR_SHAPE;
    if (cd->uout_sb < 0 || cd->uout_sd < 0) return MS_ERR_STRIDE;
    if (dm->batch == 0 || dm->dim == 0) return MS_OK;
    if (!cv.w) return MS_ERR_NULL;
    const int ei = elem_bytes(dm->in_dtype);
    if (!aligned(cv.w, 4) || (cv.b && !aligned(cv.b, 4)) || (cv.x0 && !aligned(cv.x0, ei)) ||
        (cv.u_out && !aligned(cv.u_out, ei)))
        return MS_ERR_ALIGN;
    if (dm->seqlen > 0 && cv.u_out &&
        max_offset3(dm->batch, cd->uout_sb, dm->dim, cd->uout_sd, dm->seqlen) < 0)
        return MS_ERR_SHAPE;
    if (max_offset3(dm->batch, dm->dim * cd->width, dm->dim, cd->width, cd->width) < 0) return MS_ERR_SHAPE;
    return MS_OK;
}

static int scan_common(const void *u, const void *delta, const float *A, const void *B, const void *C,
                       const float *D, const void *z, const float *delta_bias, int softplus_flag,
                       const float *initial_state, void *y, float *last_state, const ms_scan_dims *dims,
                       int *dev_status, ms_stream_t stream, const ms_scan_plan *plan, const ConvIn *cv,
                       float *ckpt = nullptr) {
    ms::ScanArgs a{};
    a.ckpt = ckpt;
    a.u = u; a.delta = delta; a.z = z; a.B = B; a.C = C;
    a.A = A; a.D = D; a.bias = delta_bias; a.h0 = initial_state;
    a.y = y; a.last = last_state; a.status = dev_status;
    a.batch = dims->batch; a.dim = dims->dim; a.L = dims->seqlen; a.N = (int)dims->dstate;
    a.u_sb = dims->u_sb; a.u_sd = dims->u_sd;
    a.dl_sb = dims->delta_sb; a.dl_sd = dims->delta_sd;
    a.z_sb = dims->z_sb; a.z_sd = dims->z_sd;
    a.y_sb = dims->y_sb; a.y_sd = dims->y_sd;
    a.B_sb = dims->B_sb; a.B_sn = dims->B_sn; a.C_sb = dims->C_sb; a.C_sn = dims->C_sn;
    a.softplus = softplus_flag ? 1 : 0;
    const int ei = elem_bytes(dims->in_dtype), eo = elem_bytes(dims->out_dtype);
    a.vec_in = vec_ok(u, dims->u_sb, dims->u_sd, ei) && vec_ok(delta, dims->delta_sb, dims->delta_sd, ei) &&
               vec_ok(z, dims->z_sb, dims->z_sd, ei);
    a.vec_out = vec_ok(y, dims->y_sb, dims->y_sd, eo);
    if (cv) {
        a.conv_w = cv->w;
        a.conv_b = cv->b;
        a.conv_x0 = cv->x0;
        a.u_out = cv->u_out;
        a.uo_sb = cv->cd->uout_sb;
        a.uo_sd = cv->cd->uout_sd;
        a.conv_width = (int)cv->cd->width;
        a.conv_silu = cv->cd->silu ? 1 : 0;
        a.vec_uout = vec_ok(cv->u_out, a.uo_sb, a.uo_sd, ei);
    }

    const bool in_bf16 = dims->in_dtype == MS_BF16, out_bf16 = dims->out_dtype == MS_BF16;
    ms::ScanPlan pl = auto_plan_args(a, in_bf16, out_bf16, true);
    if (plan) {
        pl.lanes_per_channel = plan->lanes_per_channel;
        pl.chunks_per_lane = plan->chunks_per_lane;
        pl.poly8 = plan->poly8;
        pl.engine = plan->engine;
        if (pl.engine == MS_ENGINE_TMEM && !ms::scan_tmem_applies(a, in_bf16, eo)) return MS_ERR_SHAPE;
    }
    cudaError_t e = ms::launch_scan_fwd(a, pl, in_bf16, out_bf16, (cudaStream_t)stream);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return MS_ERR_CUDA;
    }
    return MS_OK;
}

// The scan of one batch row split into segments (see split_plan): pass 1
// scans segments 0..S-2 from zero for their end states and Delta sums, the
// carries are chained, pass 2 scans every segment from its true initial
// state. Exact up to rounding: the recurrence is linear in the state.
static int scan_split(const void *u, const void *delta, const float *A, const void *B, const void *C,
                      const float *D, const void *z, const float *delta_bias, int softplus_flag,
                      const float *initial_state, void *y, float *last_state, const ms_scan_dims *dims,
                      const SplitPlan &sp, float *ws, int *dev_status, ms_stream_t stream) {
    const int ei = elem_bytes(dims->in_dtype), eo = elem_bytes(dims->out_dtype);
    const int64_t dim = dims->dim, N = dims->dstate, L = dims->seqlen, S = sp.S, Ls = sp.Ls, cn = dim * N;
    float *E = ws;
    float *dsum = E + round4((S - 1) * cn);
    float *Sin = dsum + round4((S - 1) * dim);
    float *Slast = Sin + round4(S * cn);
    const int64_t S_full = (S * Ls == L) ? S : S - 1;  // segments of exactly Ls tokens
    const cudaStream_t st = (cudaStream_t)stream;
    auto at = [](const void *p, int64_t elems, int es) -> const void * {
        return p ? static_cast<const char *>(p) + elems * es : nullptr;
    };
    for (int64_t b = 0; b < dims->batch; ++b) {
        const void *ub = at(u, b * dims->u_sb, ei), *db = at(delta, b * dims->delta_sb, ei);
        const void *zb = at(z, b * dims->z_sb, ei), *Bb = at(B, b * dims->B_sb, ei), *Cb = at(C, b * dims->C_sb, ei);
        void *yb = static_cast<char *>(y) + b * dims->y_sb * eo;
        // a run of `nseg` segments starting at segment k0 as a batch of scans
        auto segments = [&](int64_t k0, int64_t nseg, int64_t len, const float *h0, void *yv, float *last,
                            float *ds) -> int {
            const int64_t off = k0 * Ls;
            ms::ScanArgs a{};
            a.u = at(ub, off, ei); a.delta = at(db, off, ei); a.z = at(zb, off, ei);
            a.B = at(Bb, off, ei); a.C = at(Cb, off, ei);
            a.A = A; a.D = D; a.bias = delta_bias; a.h0 = h0;
            a.y = yv ? static_cast<char *>(yv) + off * eo : nullptr;
            a.last = last; a.status = dev_status; a.dsum = ds;
            a.batch = nseg; a.dim = dim; a.L = len; a.N = (int)N;
            a.u_sb = Ls; a.u_sd = dims->u_sd; a.dl_sb = Ls; a.dl_sd = dims->delta_sd;
            a.z_sb = Ls; a.z_sd = dims->z_sd; a.y_sb = Ls; a.y_sd = dims->y_sd;
            a.B_sb = Ls; a.B_sn = dims->B_sn; a.C_sb = Ls; a.C_sn = dims->C_sn;
            a.softplus = softplus_flag ? 1 : 0;
            a.vec_in = vec_ok(a.u, Ls, a.u_sd, ei) && vec_ok(a.delta, Ls, a.dl_sd, ei) && vec_ok(a.z, Ls, a.z_sd, ei);
            a.vec_out = a.y == nullptr || vec_ok(a.y, Ls, a.y_sd, eo);
            const ms::ScanPlan pl = auto_plan_args(a, dims->in_dtype == MS_BF16, dims->out_dtype == MS_BF16, true);
            return ms::launch_scan_fwd(a, pl, dims->in_dtype == MS_BF16, dims->out_dtype == MS_BF16, st) ==
                           cudaSuccess
                       ? MS_OK
                       : MS_ERR_CUDA;
        };
        const float *h0b = initial_state ? initial_state + b * cn : nullptr;
        // pass 1: end states and Delta sums of segments 0..S-2, from zero
        if (segments(0, S - 1, Ls, nullptr, nullptr, E, dsum) != MS_OK) return MS_ERR_CUDA;
        if (ms::launch_carry_combine(E, dsum, A, h0b, Sin, dim, (int)N, S, st) != cudaSuccess) return MS_ERR_CUDA;
        // pass 2: every segment from its initial state
        float *lastb = last_state ? last_state + b * cn : nullptr;
        if (segments(0, S_full, Ls, Sin, yb, Slast, nullptr) != MS_OK) return MS_ERR_CUDA;
        if (S_full < S) {
            if (segments(S - 1, 1, L - (S - 1) * Ls, Sin + (S - 1) * cn, yb, lastb, nullptr) != MS_OK)
                return MS_ERR_CUDA;
        } else if (lastb) {
            if (cudaMemcpyAsync(lastb, Slast + (S - 1) * cn, cn * sizeof(float), cudaMemcpyDeviceToDevice, st) !=
                cudaSuccess)
                return MS_ERR_CUDA;
        }
    }
    return MS_OK;
}

int mamba_scan_fwd_plan(const void *u, const void *delta, const float *A, const void *B, const void *C,
                        const float *D, const void *z, const float *delta_bias, int softplus_flag,
                        const float *initial_state, void *y, float *last_state, const ms_scan_dims *dims,
                        void *workspace, size_t workspace_bytes, int *dev_status, ms_stream_t stream,
                        const ms_scan_plan *plan) {
    if (plan && !plan_valid(plan)) return MS_ERR_SHAPE;
    int rc = check_scan(u, delta, A, B, C, D, z, delta_bias, initial_state, y, last_state, dims);
    if (rc != MS_OK) return rc;
    if (workspace_bytes < mamba_scan_workspace_size(dims) || (workspace_bytes > 0 && !workspace))
        return MS_ERR_WORKSPACE;
    if (dims->batch == 0 || dims->dim == 0) return MS_OK;
    if (dims->seqlen == 0 && !last_state) return MS_OK;
    if (!plan) {
        const SplitPlan sp = split_plan(dims, num_sms_current());
        if (sp.S > 1) {
            if (!aligned(workspace, 16)) return MS_ERR_ALIGN;
            rc = scan_split(u, delta, A, B, C, D, z, delta_bias, softplus_flag, initial_state, y, last_state, dims, sp,
                            static_cast<float *>(workspace), dev_status, stream);
            if (rc != MS_OK) cudaGetLastError();
            return rc;
        }
    }
    return scan_common(u, delta, A, B, C, D, z, delta_bias, softplus_flag, initial_state, y, last_state,
                       dims, dev_status, stream, plan, nullptr);
}

int mamba_conv_scan_fwd(const void *x, const float *conv_w, const float *conv_b, const void *conv_x0,
                        void *u_out, const ms_conv_dims *cdims, const void *delta, const float *A,
                        const void *B, const void *C, const float *D, const void *z,
                        const float *delta_bias, int softplus_flag, const float *initial_state,
                        void *y, float *last_state, const ms_scan_dims *dims,
                        const ms_scan_plan *plan, int *dev_status, ms_stream_t stream) {
    if (plan && (!plan_valid(plan) || plan->engine != MS_ENGINE_REGISTER || plan->chunks_per_lane != 1 ||
                 (plan->poly8 != 0 && plan->poly8 != 8)))
        return MS_ERR_SHAPE;
    int rc = check_scan(x, delta, A, B, C, D, z, delta_bias, initial_state, y, last_state, dims);
    if (rc != MS_OK) return rc;
    const ConvIn cv{conv_w, conv_b, conv_x0, u_out, cdims};
    rc = check_conv(cv, dims);
    if (rc != MS_OK) return rc;
    if (dims->batch == 0 || dims->dim == 0) return MS_OK;
    if (dims->seqlen == 0 && !last_state) return MS_OK;
    return scan_common(x, delta, A, B, C, D, z, delta_bias, softplus_flag, initial_state, y, last_state,
                       dims, dev_status, stream, plan, &cv);
}

size_t mamba_scan_ckpt_size(const ms_scan_dims *dims) {
    if (!dims || dims->batch <= 0 || dims->dim <= 0 || dims->seqlen <= 0 || dims->dstate <= 0) return 0;
    const int64_t nck = (dims->seqlen + ms::kCkptTokens - 1) / ms::kCkptTokens;
    return (size_t)dims->batch * (size_t)dims->dim * (size_t)nck * (size_t)dims->dstate * sizeof(float);
}

int mamba_scan_fwd_train(const void *u, const void *delta, const float *A, const void *B, const void *C,
                         const float *D, const void *z, const float *delta_bias, int softplus_flag,
                         const float *initial_state, void *y, float *last_state, float *ckpt,
                         const ms_scan_dims *dims, int *dev_status, ms_stream_t stream) {
    int rc = check_scan(u, delta, A, B, C, D, z, delta_bias, initial_state, y, last_state, dims);
    if (rc != MS_OK) return rc;
    if (dims->batch == 0 || dims->dim == 0) return MS_OK;
    if (dims->seqlen > 0 && !ckpt) return MS_ERR_NULL;
    if (ckpt && !aligned(ckpt, 4)) return MS_ERR_ALIGN;
    if (dims->seqlen == 0 && !last_state) return MS_OK;
    return scan_common(u, delta, A, B, C, D, z, delta_bias, softplus_flag, initial_state, y, last_state,
                       dims, dev_status, stream, nullptr, nullptr, ckpt);
}

size_t mamba_scan_bwd_workspace_size(const ms_scan_dims *dims) { return mamba_scan_ckpt_size(dims); }

int mamba_scan_bwd(const void *u, const void *delta, const float *A, const void *B, const void *C,
                   const float *D, const void *z, const float *delta_bias, int softplus_flag,
                   const float *initial_state, const float *ckpt, const void *dout, const float *dlast,
                   float *du, float *ddelta, float *dA, float *dB, float *dC, float *dD, float *dz,
                   float *ddelta_bias, float *dinitial_state, const ms_scan_dims *dims, void *workspace,
                   size_t workspace_bytes, int *dev_status, ms_stream_t stream) {
    // dout takes y's place in the forward checks (its dtype and strides).
    int rc = check_scan(u, delta, A, B, C, D, z, delta_bias, initial_state, const_cast<void *>(dout), nullptr,
                        dims);
    if (rc != MS_OK) return rc;
    const int64_t nb = dims->batch, nd = dims->dim, N = dims->dstate, L = dims->seqlen;
    if (nb == 0 || nd == 0) return MS_OK;
    if (!dA || (L > 0 && (!du || !ddelta || !dB || !dC))) return MS_ERR_NULL;
    const float *outs[] = {du, ddelta, dA, dB, dC, dD, dz, ddelta_bias, dinitial_state, ckpt, dlast};
    for (const float *p : outs)
        if (p && !aligned(p, 4)) return MS_ERR_ALIGN;
    if (max_offset3(nb, nd * L, nd, L, L > 0 ? L : 1) < 0 || max_offset3(nb, N * L, N, L, L > 0 ? L : 1) < 0)
        return MS_ERR_SHAPE;
    const size_t ck_bytes = mamba_scan_ckpt_size(dims);
    if (!ckpt && L > 0 && (workspace_bytes < ck_bytes || !workspace)) return MS_ERR_WORKSPACE;
    if (!ckpt && L > 0 && !aligned(workspace, 4)) return MS_ERR_ALIGN;

    const cudaStream_t st = (cudaStream_t)stream;
    // sums are accumulated: start from zero
    const size_t fl = sizeof(float);
    cudaError_t e = cudaMemsetAsync(dA, 0, (size_t)(nd * N) * fl, st);
    if (e == cudaSuccess && L > 0) e = cudaMemsetAsync(dB, 0, (size_t)(nb * N * L) * fl, st);
    if (e == cudaSuccess && L > 0) e = cudaMemsetAsync(dC, 0, (size_t)(nb * N * L) * fl, st);
    if (e == cudaSuccess && dD) e = cudaMemsetAsync(dD, 0, (size_t)nd * fl, st);
    if (e == cudaSuccess && ddelta_bias) e = cudaMemsetAsync(ddelta_bias, 0, (size_t)nd * fl, st);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return MS_ERR_CUDA;
    }
    if (L > 0 && !ckpt) {
        // recompute the saved states: the forward without y
        float *wck = static_cast<float *>(workspace);
        rc = scan_common(u, delta, A, B, C, D, z, delta_bias, softplus_flag, initial_state, nullptr, nullptr,
                         dims, dev_status, stream, nullptr, nullptr, wck);
        if (rc != MS_OK) return rc;
        ckpt = wck;
    }
    ms::BwdArgs a{};
    a.u = u; a.delta = delta; a.z = z; a.B = B; a.C = C;
    a.A = A; a.D = D; a.bias = delta_bias; a.ckpt = ckpt; a.dlast = dlast; a.dout = dout;
    a.du = du; a.ddelta = ddelta; a.dz = z ? dz : nullptr; a.dA = dA; a.dB = dB; a.dC = dC; a.dD = dD;
    a.dbias = ddelta_bias; a.dh0 = dinitial_state; a.status = dev_status;
    a.batch = nb; a.dim = nd; a.L = L; a.N = (int)N;
    a.u_sb = dims->u_sb; a.u_sd = dims->u_sd; a.dl_sb = dims->delta_sb; a.dl_sd = dims->delta_sd;
    a.z_sb = dims->z_sb; a.z_sd = dims->z_sd; a.y_sb = dims->y_sb; a.y_sd = dims->y_sd;
    a.B_sb = dims->B_sb; a.B_sn = dims->B_sn; a.C_sb = dims->C_sb; a.C_sn = dims->C_sn;
    a.softplus = softplus_flag ? 1 : 0;
    {
        const int ei = elem_bytes(dims->in_dtype), eo = elem_bytes(dims->out_dtype);
        a.vec_in = vec_ok(u, dims->u_sb, dims->u_sd, ei) && vec_ok(delta, dims->delta_sb, dims->delta_sd, ei) &&
                   vec_ok(z, dims->z_sb, dims->z_sd, ei);
        a.vec_out = vec_ok(dout, dims->y_sb, dims->y_sd, eo);
        a.vec_bc = aligned(dB, 16) && aligned(dC, 16) && (L % 4) == 0;
    }
    e = ms::launch_scan_bwd(a, dims->in_dtype == MS_BF16, dims->out_dtype == MS_BF16, st);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return MS_ERR_CUDA;
    }
    return MS_OK;
}

// Device address of g_bwd_scratch on the current device: looked up with the
// device current on the first call, and again whenever the device's context
// has changed since (after a device reset the module is loaded anew and the
// array may sit elsewhere), or when the context's id cannot be read.
static int bwd_scratch(void **p) {
    static std::mutex mtx;
    static void *addr[64] = {};
    static uint64_t ctx_of[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return MS_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lock(mtx);
    const uint64_t ctx = ms::current_context_id();
    if (addr[dev] == nullptr || ctx == 0 || ctx != ctx_of[dev]) {
        void *a = nullptr;
        if (cudaGetSymbolAddress(&a, g_bwd_scratch) != cudaSuccess || a == nullptr) {
            cudaGetLastError();
            return MS_ERR_CUDA;
        }
        addr[dev] = a;
        ctx_of[dev] = ms::current_context_id();  // the lookup made the primary context current
    }
    *p = addr[dev];
    return MS_OK;
}

int mamba_scan_bwd_noalloc(const void *u, const void *delta, const float *A, const void *B, const void *C,
                           const float *D, const void *z, const float *delta_bias, int softplus_flag,
                           const float *initial_state, const void *dout, const float *dlast, float *du,
                           float *ddelta, float *dA, float *dB, float *dC, float *dD, float *dz,
                           float *ddelta_bias, float *dinitial_state, const ms_scan_dims *dims,
                           int *dev_status, ms_stream_t stream) {
    int rc = check_scan(u, delta, A, B, C, D, z, delta_bias, initial_state, const_cast<void *>(dout), nullptr,
                        dims);
    if (rc != MS_OK) return rc;
    if (dims->batch == 0 || dims->dim == 0) return MS_OK;
    const size_t need = mamba_scan_bwd_workspace_size(dims);
    if (need > MS_BWD_NOALLOC_MAX_BYTES) return MS_ERR_SCRATCH;
    void *scratch = nullptr;
    if (need > 0) {
        rc = bwd_scratch(&scratch);
        if (rc != MS_OK) return rc;
    }
    return mamba_scan_bwd(u, delta, A, B, C, D, z, delta_bias, softplus_flag, initial_state, nullptr, dout, dlast,
                          du, ddelta, dA, dB, dC, dD, dz, ddelta_bias, dinitial_state, dims, scratch,
                          need > 0 ? MS_BWD_NOALLOC_MAX_BYTES : 0, dev_status, stream);
}

size_t mamba2_ssd_workspace_size(const ms_ssd_dims *dm) {
    if (!dm || dm->batch < 0 || dm->nheads < 1) return 0;
    return ms::ssd_tc_workspace_size(dm->batch, dm->nheads);
}

int mamba2_ssd_fwd(const void *x, const void *dt, const float *A, const void *B, const void *C, const float *D,
                   const float *dt_bias, int softplus_flag, const float *initial_state, void *y, float *final_state,
                   const ms_ssd_dims *dm, void *workspace, size_t workspace_bytes, int *dev_status,
                   ms_stream_t stream) {
    if (!dm) return MS_ERR_NULL;
    if ((dm->in_dtype != MS_F32 && dm->in_dtype != MS_BF16) || (dm->out_dtype != MS_F32 && dm->out_dtype != MS_BF16))
        return MS_ERR_DTYPE;
    if (dm->batch < 0 || dm->seqlen < 0 || dm->nheads < 1 || dm->ngroups < 1 || dm->nheads % dm->ngroups != 0 ||
        dm->headdim < 1 || dm->dstate < 1)
        return MS_ERR_SHAPE;
    if (dm->x_sb < 0 || dm->x_sl < 0 || dm->x_sh < 0 || dm->dt_sb < 0 || dm->dt_sl < 0 || dm->B_sb < 0 ||
        dm->B_sl < 0 || dm->B_sg < 0 || dm->C_sb < 0 || dm->C_sl < 0 || dm->C_sg < 0 || dm->y_sb < 0 ||
        dm->y_sl < 0 || dm->y_sh < 0)
        return MS_ERR_STRIDE;
    if (!ms::ssd_shape_supported(dm->headdim, dm->dstate)) return MS_ERR_SHAPE;
    if (dm->in_dtype != MS_BF16) return MS_ERR_DTYPE;
    if (dm->batch == 0) return MS_OK;
    if (!A) return MS_ERR_NULL;
    if (dm->seqlen > 0 && (!x || !dt || !B || !C || !y)) return MS_ERR_NULL;
    const int eo = elem_bytes(dm->out_dtype);
    auto rows16 = [](const void *p, int64_t s1, int64_t s2, int64_t s3) {
        return p == nullptr || (aligned(p, 16) && (s1 * 2) % 16 == 0 && (s2 * 2) % 16 == 0 && (s3 * 2) % 16 == 0);
    };
    if (!rows16(x, dm->x_sb, dm->x_sl, dm->x_sh) || !rows16(B, dm->B_sb, dm->B_sl, dm->B_sg) ||
        !rows16(C, dm->C_sb, dm->C_sl, dm->C_sg) || (dt && !aligned(dt, 2)) || !aligned(A, 4) ||
        (D && !aligned(D, 4)) || (dt_bias && !aligned(dt_bias, 4)) || (initial_state && !aligned(initial_state, 4)) ||
        (final_state && !aligned(final_state, 4)) ||
        (y && (!aligned(y, 2 * eo) || dm->y_sb % 2 || dm->y_sl % 2 || dm->y_sh % 2)))
        return MS_ERR_ALIGN;
    if (dm->seqlen > 0) {
        const int64_t L = dm->seqlen, H = dm->nheads, G = dm->ngroups;
        if (max_offset3(dm->batch, dm->x_sb, L, dm->x_sl, 1) < 0 || max_offset3(H, dm->x_sh, 1, 0, 64) < 0 ||
            max_offset3(dm->batch, dm->y_sb, L, dm->y_sl, 1) < 0 || max_offset3(H, dm->y_sh, 1, 0, 64) < 0 ||
            max_offset3(dm->batch, dm->dt_sb, L, dm->dt_sl, H) < 0 ||
            max_offset3(dm->batch, dm->B_sb, L, dm->B_sl, 1) < 0 || max_offset3(G, dm->B_sg, 1, 0, 128) < 0 ||
            max_offset3(dm->batch, dm->C_sb, L, dm->C_sl, 1) < 0 || max_offset3(G, dm->C_sg, 1, 0, 128) < 0)
            return MS_ERR_SHAPE;
    }
    if (dm->seqlen == 0) {
        // no tokens: the final state is the initial one
        if (!final_state) return MS_OK;
        const size_t bytes = (size_t)dm->batch * dm->nheads * dm->headdim * dm->dstate * sizeof(float);
        cudaError_t e = initial_state ? (initial_state == final_state
                                             ? cudaSuccess
                                             : cudaMemcpyAsync(final_state, initial_state, bytes,
                                                               cudaMemcpyDeviceToDevice, (cudaStream_t)stream))
                                      : cudaMemsetAsync(final_state, 0, bytes, (cudaStream_t)stream);
        if (e != cudaSuccess) {
            cudaGetLastError();
            return MS_ERR_CUDA;
        }
        return MS_OK;
    }
    const size_t need = ms::ssd_tc_workspace_size(dm->batch, dm->nheads);
    if (!workspace || workspace_bytes < need) return MS_ERR_WORKSPACE;
    if (!aligned(workspace, 16)) return MS_ERR_ALIGN;
    ms::SsdArgs a{};
    a.x = x; a.dt = dt; a.B = B; a.C = C; a.A = A; a.D = D; a.dt_bias = dt_bias; a.s0 = initial_state;
    a.y = y; a.s_last = final_state;
    a.batch = dm->batch; a.L = dm->seqlen; a.H = dm->nheads; a.G = dm->ngroups;
    a.x_sb = dm->x_sb; a.x_sl = dm->x_sl; a.x_sh = dm->x_sh; a.dt_sb = dm->dt_sb; a.dt_sl = dm->dt_sl;
    a.B_sb = dm->B_sb; a.B_sl = dm->B_sl; a.B_sg = dm->B_sg; a.C_sb = dm->C_sb; a.C_sl = dm->C_sl;
    a.C_sg = dm->C_sg; a.y_sb = dm->y_sb; a.y_sl = dm->y_sl; a.y_sh = dm->y_sh;
    a.softplus = softplus_flag ? 1 : 0;
    a.status = dev_status;
    cudaError_t e = ms::launch_ssd_fwd_tc(a, dm->out_dtype == MS_BF16, workspace, num_sms_current(), (cudaStream_t)stream);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return MS_ERR_CUDA;
    }
    return MS_OK;
}

size_t mamba2_ssd_chunk_cb_size(const ms_ssd_dims *dm) {
    if (!dm || dm->batch < 0 || dm->seqlen < 0 || dm->ngroups < 1) return 0;
    return (size_t)dm->batch * (size_t)dm->ngroups * (size_t)((dm->seqlen + 31) / 32) * 32 * 32 * sizeof(float);
}

int mamba2_ssd_chunk_cb(const void *B, const void *C, float *cb, const ms_ssd_dims *dm, int *dev_status,
                        ms_stream_t stream) {
    if (!dm) return MS_ERR_NULL;
    if (dm->in_dtype != MS_BF16) return MS_ERR_DTYPE;
    if (dm->batch < 0 || dm->seqlen < 0 || dm->ngroups < 1 || !ms::ssd_cb_shape_supported(dm->dstate))
        return MS_ERR_SHAPE;
    if (dm->B_sb < 0 || dm->B_sl < 0 || dm->B_sg < 0 || dm->C_sb < 0 || dm->C_sl < 0 || dm->C_sg < 0)
        return MS_ERR_STRIDE;
    if (dm->batch == 0 || dm->seqlen == 0) return MS_OK;
    if (!B || !C || !cb) return MS_ERR_NULL;
    auto rows16 = [](const void *p, int64_t s1, int64_t s2, int64_t s3) {
        return aligned(p, 16) && (s1 * 2) % 16 == 0 && (s2 * 2) % 16 == 0 && (s3 * 2) % 16 == 0;
    };
    if (!rows16(B, dm->B_sb, dm->B_sl, dm->B_sg) || !rows16(C, dm->C_sb, dm->C_sl, dm->C_sg) || !aligned(cb, 16))
        return MS_ERR_ALIGN;
    const int64_t L = dm->seqlen, G = dm->ngroups;
    if (max_offset3(dm->batch, dm->B_sb, L, dm->B_sl, 1) < 0 || max_offset3(G, dm->B_sg, 1, 0, 128) < 0 ||
        max_offset3(dm->batch, dm->C_sb, L, dm->C_sl, 1) < 0 || max_offset3(G, dm->C_sg, 1, 0, 128) < 0)
        return MS_ERR_SHAPE;
    ms::SsdCbArgs a{};
    a.B = B; a.C = C; a.cb = cb; a.status = dev_status;
    a.batch = dm->batch; a.L = L; a.G = G;
    a.B_sb = dm->B_sb; a.B_sl = dm->B_sl; a.B_sg = dm->B_sg;
    a.C_sb = dm->C_sb; a.C_sl = dm->C_sl; a.C_sg = dm->C_sg;
    if (ms::launch_ssd_chunk_cb(a, (cudaStream_t)stream) != cudaSuccess) {
        cudaGetLastError();
        return MS_ERR_CUDA;
    }
    return MS_OK;
}

int mamba2_ssd_state_update(float *state, const void *x, const void *dt, const float *A, const void *B,
                            const void *C, const float *D, const float *dt_bias, int softplus_flag, void *y,
                            const ms_ssd_update_dims *dm, int *dev_status, ms_stream_t stream) {
    if (!dm) return MS_ERR_NULL;
    if ((dm->in_dtype != MS_F32 && dm->in_dtype != MS_BF16) || (dm->out_dtype != MS_F32 && dm->out_dtype != MS_BF16))
        return MS_ERR_DTYPE;
    if (dm->batch < 0 || dm->nheads < 1 || dm->ngroups < 1 || dm->nheads % dm->ngroups != 0 || dm->headdim < 1 ||
        dm->headdim > INT32_MAX || dm->dstate != 128)
        return MS_ERR_SHAPE;
    if (dm->x_sb < 0 || dm->x_sh < 0 || dm->dt_sb < 0 || dm->B_sb < 0 || dm->B_sg < 0 || dm->C_sb < 0 ||
        dm->C_sg < 0 || dm->y_sb < 0 || dm->y_sh < 0 || dm->state_sb < 0 || dm->state_sh < 0)
        return MS_ERR_STRIDE;
    if (dm->batch == 0) return MS_OK;
    if (!state || !x || !dt || !A || !B || !C || !y) return MS_ERR_NULL;
    const int ei = elem_bytes(dm->in_dtype), eo = elem_bytes(dm->out_dtype);
    if (!aligned(state, 16) || dm->state_sb % 4 || dm->state_sh % 4 || !aligned(x, ei) || !aligned(dt, ei) ||
        !aligned(B, ei) || !aligned(C, ei) || !aligned(y, eo) || !aligned(A, 4) || (D && !aligned(D, 4)) ||
        (dt_bias && !aligned(dt_bias, 4)))
        return MS_ERR_ALIGN;
    const int64_t H = dm->nheads, G = dm->ngroups, P = dm->headdim;
    if (max_offset3(dm->batch, dm->state_sb, H, dm->state_sh, P * 128) < 0 ||
        max_offset3(dm->batch, dm->x_sb, H, dm->x_sh, P) < 0 || max_offset3(dm->batch, dm->y_sb, H, dm->y_sh, P) < 0 ||
        max_offset3(dm->batch, dm->dt_sb, 1, 0, H) < 0 || max_offset3(dm->batch, dm->B_sb, G, dm->B_sg, 128) < 0 ||
        max_offset3(dm->batch, dm->C_sb, G, dm->C_sg, 128) < 0)
        return MS_ERR_SHAPE;
    ms::SsdUpdArgs a{};
    a.state = state; a.x = x; a.dt = dt; a.B = B; a.C = C; a.A = A; a.D = D; a.dt_bias = dt_bias; a.y = y;
    a.status = dev_status;
    a.batch = dm->batch; a.H = H; a.G = G; a.P = (int)P;
    a.x_sb = dm->x_sb; a.x_sh = dm->x_sh; a.dt_sb = dm->dt_sb; a.B_sb = dm->B_sb; a.B_sg = dm->B_sg;
    a.C_sb = dm->C_sb; a.C_sg = dm->C_sg; a.y_sb = dm->y_sb; a.y_sh = dm->y_sh;
    a.st_sb = dm->state_sb; a.st_sh = dm->state_sh;
    a.softplus = softplus_flag ? 1 : 0;
    cudaError_t e = ms::launch_ssd_update(a, dm->in_dtype == MS_BF16, dm->out_dtype == MS_BF16, (cudaStream_t)stream);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return MS_ERR_CUDA;
    }
    return MS_OK;
}

int mamba_state_update(float *state, const void *x, const void *delta, const float *A, const void *B,
                       const void *C, const float *D, const void *z, const float *delta_bias,
                       int softplus_flag, void *y, const ms_update_dims *dm, int *dev_status,
                       ms_stream_t stream) {
    if (!dm) return MS_ERR_NULL;
    if ((dm->in_dtype != MS_F32 && dm->in_dtype != MS_BF16) ||
        (dm->out_dtype != MS_F32 && dm->out_dtype != MS_BF16))
        return MS_ERR_DTYPE;
    if (dm->batch < 0 || dm->dim < 0 || dm->dstate < 1 || dm->dstate > MS_MAX_DSTATE) return MS_ERR_SHAPE;
    if (dm->batch > 65535 || dm->dim > (int64_t)(INT32_MAX / 4)) return MS_ERR_SHAPE;
    if (dm->x_sb < 0 || dm->delta_sb < 0 || dm->z_sb < 0 || dm->y_sb < 0 || dm->B_sb < 0 || dm->C_sb < 0 ||
        dm->state_sb < 0 || dm->state_sd < 0)
        return MS_ERR_STRIDE;
    if (dm->batch == 0 || dm->dim == 0) return MS_OK;
    if (!state || !x || !delta || !A || !B || !C || !y) return MS_ERR_NULL;
    const int ei = elem_bytes(dm->in_dtype), eo = elem_bytes(dm->out_dtype);
    if (!aligned(state, 4) || !aligned(x, ei) || !aligned(delta, ei) || !aligned(B, ei) || !aligned(C, ei) ||
        (z && !aligned(z, ei)) || !aligned(y, eo) || !aligned(A, 4) || (D && !aligned(D, 4)) ||
        (delta_bias && !aligned(delta_bias, 4)))
        return MS_ERR_ALIGN;
    if (max_offset3(dm->batch, dm->x_sb, 1, 0, dm->dim) < 0 || max_offset3(dm->batch, dm->delta_sb, 1, 0, dm->dim) < 0 ||
        max_offset3(dm->batch, dm->z_sb, 1, 0, dm->dim) < 0 || max_offset3(dm->batch, dm->y_sb, 1, 0, dm->dim) < 0 ||
        max_offset3(dm->batch, dm->B_sb, 1, 0, dm->dstate) < 0 || max_offset3(dm->batch, dm->C_sb, 1, 0, dm->dstate) < 0 ||
        max_offset3(dm->batch, dm->state_sb, dm->dim, dm->state_sd, dm->dstate) < 0)
        return MS_ERR_SHAPE;

    ms::UpdateArgs a{};
    a.state = state; a.x = x; a.delta = delta; a.z = z; a.B = B; a.C = C;
    a.A = A; a.D = D; a.bias = delta_bias; a.y = y; a.status = dev_status;
    a.batch = dm->batch; a.dim = dm->dim; a.N = (int)dm->dstate;
    a.x_sb = dm->x_sb; a.dl_sb = dm->delta_sb; a.z_sb = dm->z_sb; a.y_sb = dm->y_sb;
    a.B_sb = dm->B_sb; a.C_sb = dm->C_sb; a.st_sb = dm->state_sb; a.st_sd = dm->state_sd;
    a.softplus = softplus_flag ? 1 : 0;
    a.vec_state = aligned(state, 16) && (dm->state_sb % 4) == 0 && (dm->state_sd % 4) == 0;
    a.vec_A = aligned(A, 16) && (dm->dstate % 4) == 0;
    a.vec_bc = aligned(B, 4 * ei) && aligned(C, 4 * ei) && (dm->B_sb % 4) == 0 && (dm->C_sb % 4) == 0;
    const bool ib = dm->in_dtype == MS_BF16, ob = dm->out_dtype == MS_BF16;
    cudaError_t e = ms::state_update_stream_applies(a, ei, eo)
                        ? ms::launch_state_update_stream(a, ib, ob, (cudaStream_t)stream)
                        : ms::launch_state_update(a, ib, ob, (cudaStream_t)stream);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return MS_ERR_CUDA;
    }
    return MS_OK;
}

}  // extern "C"
