// ms_internal.h -- argument blocks passed from the C-ABI layer to the kernel
// launchers (not part of the public ABI).
#pragma once

#include <atomic>
#include <cstdint>
#include <cuda_runtime.h>

namespace ms {

struct ScanArgs {
    const void *u, *delta, *z, *B, *C;
    const float *A, *D, *bias, *h0;
    void *y;
    float *last;
    int *status;
    int64_t batch, dim, L;
    int N;
    int64_t u_sb, u_sd, dl_sb, dl_sd, z_sb, z_sd, y_sb, y_sd;
    int64_t B_sb, B_sn, C_sb, C_sn;
    int softplus;
    int vec_in;   // u/delta/z rows 16-byte aligned: vector loads allowed
    int vec_out;  // y rows 16-byte aligned: vector stores allowed
    // Causal conv front-end (conv_w == nullptr: u is read as given). With the
    // front-end, `u` points at the conv input x.
    const float *conv_w, *conv_b;  // [dim, conv_width], [dim]
    const void *conv_x0;           // [batch, dim, conv_width - 1] in the input dtype, or null
    void *u_out;                   // [batch, dim, L] in the input dtype, or null
    int64_t uo_sb, uo_sd;
    int conv_width;                // 1..4
    int conv_silu;
    int vec_uout;                  // u_out rows 16-byte aligned
    // Training: the state before every kCkptTokens-token block, [batch, dim,
    // ceil(L / kCkptTokens), N] fp32 (null: not written). y may be null then.
    float *ckpt;
    // Sequence split: sum of Delta over the sequence per channel, [batch, dim]
    // (null: not written). Like ckpt, it selects the saved-state kernels.
    float *dsum;
};

// Carry combine of a sequence split into S segments for one batch row:
// Sin[0] = h0 (or 0), Sin[k+1] = exp(A dsum[k]) Sin[k] + E[k], with E[k] the
// end state of segment k scanned from zero and dsum[k] its sum of Delta.
cudaError_t launch_carry_combine(const float *E, const float *dsum, const float *A, const float *h0, float *Sin,
                                 int64_t dim, int N, int64_t S, cudaStream_t stream);

// Tokens between two saved states of the forward (the backward recomputes
// each block from its saved state).
constexpr int kCkptTokens = 64;

// The automatic plan of the tensor-memory kernel: exponentials on the FMA-pipe
// polynomial, in eighths. bf16 inputs take every one on MUFU (the polynomial
// costs more issue than it frees); fp32 inputs take every one from the
// polynomial (unbiased near 1, see ms_device.cuh).
constexpr int kTmemPoly8Bf16 = 0;

// Arguments of the backward kernel (gradients are fp32, dense).
struct BwdArgs {
    const void *u, *delta, *z, *B, *C;  // input dtype
    const float *A, *D, *bias, *ckpt, *dlast;
    const void *dout;                   // output dtype, strides y_sb / y_sd
    float *du, *ddelta, *dz, *dA, *dB, *dC, *dD, *dbias, *dh0;
    int *status;  // device status word of the debug build's bounds checks, or null
    int64_t batch, dim, L;
    int N;
    int64_t u_sb, u_sd, dl_sb, dl_sd, z_sb, z_sd, y_sb, y_sd;
    int64_t B_sb, B_sn, C_sb, C_sn;
    int softplus;
    int vec_in;   // u/delta/z rows 16-byte aligned
    int vec_out;  // dout rows 16-byte aligned
    int vec_bc;   // dB/dC rows allow 16-byte atomics (L % 4 == 0, aligned base)
};

// Arguments of the Mamba-2 SSD forward (bf16 x, dt, B, C; fp32 A, D, dt_bias,
// states). Element strides; the innermost dimension of every array is dense.
struct SsdArgs {
    const void *x, *dt, *B, *C;
    const float *A, *D, *dt_bias, *s0;
    void *y;
    float *s_last;
    int64_t batch, L, H, G;
    int64_t x_sb, x_sl, x_sh, dt_sb, dt_sl, B_sb, B_sl, B_sg, C_sb, C_sl, C_sg, y_sb, y_sl, y_sh;
    int softplus;
    int *status;
};
bool ssd_shape_supported(int64_t headdim, int64_t dstate);

// Chunk-parallel SSD forward on the tcgen05 tensor cores: per-launch state
// of the chunk hand-off (flags [batch * H] then the ticket counter, zeroed
// before the launch; the running state [batch, H, P / 4, N, 4] in the workspace),
// the index of the last chunk, the number of work items, the heads per work
// item, and how y is stored.
struct SsdTcArgs {
    int *flags;
    int *counter;
    float *state;
    int64_t last_chunk;
    int64_t items;
    int hb;
    int y_vec16;  // y rows take 16-byte stores
    int y_tma;    // y is written by tensor stores through the kernel's y map
    int cb_tma;   // the C and B tiles are read by tensor copies through the kernel's maps
};
int ssd_tc_head_block(int64_t batch, int64_t seqlen, int64_t nheads, int64_t ngroups, int num_sms);
size_t ssd_tc_workspace_size(int64_t batch, int64_t nheads);
cudaError_t launch_ssd_fwd_tc(const SsdArgs &a, bool out_bf16, void *workspace, int num_sms, cudaStream_t stream);

// Arguments of the per-chunk C B^T of the SSD layer (bf16 B, C with dstate
// 128; cb [batch, G, ceil(L / 32), 32, 32] fp32, dense).
struct SsdCbArgs {
    const void *B, *C;
    float *cb;
    int *status;
    int64_t batch, L, G;
    int64_t B_sb, B_sl, B_sg, C_sb, C_sl, C_sg;
};
bool ssd_cb_shape_supported(int64_t dstate);
cudaError_t launch_ssd_chunk_cb(const SsdCbArgs &a, cudaStream_t stream);

// Arguments of the Mamba-2 SSD one-token state update (state [b, H, P, 128]
// fp32, each head's [P, 128] block dense).
struct SsdUpdArgs {
    float *state;
    const void *x, *dt, *B, *C;
    const float *A, *D, *dt_bias;
    void *y;
    int *status;  // device status word of the debug build's bounds checks, or null
    int64_t batch, H, G;
    int P;
    int64_t x_sb, x_sh, dt_sb, B_sb, B_sg, C_sb, C_sg, y_sb, y_sh, st_sb, st_sh;
    int softplus;
};
cudaError_t launch_ssd_update(const SsdUpdArgs &a, bool in_bf16, bool out_bf16, cudaStream_t stream);

// Launch shape chosen on the host for one scan call.
struct ScanPlan {
    int lanes_per_channel;  // G: lanes sharing one channel (1, 2, 4, 8), 16/G states each
    int chunks_per_lane;    // CH: 8-token chunks per lane per tile (1, 2; 1 when G = 8)
    int poly8;              // eighths of the exponentials evaluated on the FMA pipe
    int engine;             // 0: register-prefetch kernel; 1: TMA + tensor-memory kernel (G = 4)
};

struct UpdateArgs {
    float *state;
    const void *x, *delta, *z, *B, *C;
    const float *A, *D, *bias;
    void *y;
    int *status;
    int64_t batch, dim;
    int N;
    int64_t x_sb, dl_sb, z_sb, y_sb, B_sb, C_sb, st_sb, st_sd;
    int softplus;
    int vec_state;  // state: 16-byte aligned groups of 4 states
    int vec_A;      // A: 16-byte aligned groups of 4 states
    int vec_bc;     // B, C: groups of 4 states aligned for one vector load
};

// in_bf16/out_bf16 select the element types. Return a cudaError_t.
cudaError_t launch_scan_fwd(const ScanArgs &a, const ScanPlan &plan, bool in_bf16, bool out_bf16,
                            cudaStream_t stream);
cudaError_t launch_state_update(const UpdateArgs &a, bool in_bf16, bool out_bf16,
                                cudaStream_t stream);

// Bulk-copy stream variant of the decode step (dense 16-state rows, dim a
// multiple of 128, 16-byte aligned rows).
bool state_update_stream_applies(const UpdateArgs &a, int in_bytes, int out_bytes);
cudaError_t launch_state_update_stream(const UpdateArgs &a, bool in_bf16, bool out_bf16, cudaStream_t stream);
// One CTA waits `rounds` bounded tries on a barrier nothing completes, then
// ORs MS_ERR_TIMEOUT into *status (tests the device timeout path).
cudaError_t launch_bounded_wait_probe(int *status, uint32_t rounds, cudaStream_t stream);
#ifdef MS_DEBUG
// One thread writes element `index` of a 16-int device array through
// MS_CHECK (debug build only).
cudaError_t launch_bounds_probe(int index, int *status, cudaStream_t stream);
#endif

cudaError_t launch_scan_bwd(const BwdArgs &a, bool in_bf16, bool out_bf16, cudaStream_t stream);

// Plan for a call (host heuristic from sizes, strides and dtypes).
ScanPlan plan_scan(const ScanArgs &a, bool in_bf16, int num_sms);

// The TMA + tensor-memory scan kernel (scan_fwd_tmem.cu): sizes and strides
// it takes (d_state 16, L a multiple of 8, 16-byte rows), and the full check
// including pointer alignment and the outputs requested.
bool scan_tmem_shape_ok(const ScanArgs &a, bool in_bf16, int out_bytes);
bool scan_tmem_applies(const ScanArgs &a, bool in_bf16, int out_bytes);
cudaError_t launch_scan_fwd_tmem(const ScanArgs &a, const ScanPlan &plan, bool in_bf16, bool out_bf16, int num_sms,
                                 cudaStream_t stream);

// Unique id of the calling thread's current CUDA context, never 0; 0 when it
// cannot be read. A device reset replaces the primary context, so caches of
// per-context facts (kernel attributes, device addresses of symbols) are
// keyed on this id and redone when it changes.
uint64_t current_context_id();

// Raises a kernel's dynamic shared memory limit to `bytes` once per device
// and context (cudaFuncSetAttribute is repeated when the context changed or
// its id cannot be read).
class SmemOptIn {
  public:
    cudaError_t ensure(const void *func, int bytes);

  private:
    std::atomic<uint64_t> ctx_[64] = {};  // per device: context the attribute was set in
};

}  // namespace ms
