/*
 * mambascan.h -- C ABI of libmambascan.so: the Mamba selective scan (forward)
 * and the single-token selective state update, as hand-written CUDA for
 * NVIDIA B200 (sm_100a).
 *
 * What is computed. For every batch row b and channel d, with Delta_t the step
 * size of token t:
 *     Delta_t = softplus(delta[b,d,t] + delta_bias[d])   (plain sum when the
 *                                                         softplus flag is 0)
 *     A_bar   = exp(Delta_t * A[d,n])                     per state n
 *     h_t[n]  = A_bar * h_{t-1}[n] + Delta_t * B[b,n,t] * u[b,d,t]
 *     y[b,d,t] = (sum_n C[b,n,t] * h_t[n] + D[d] * u[b,d,t]) * silu(z[b,d,t])
 * with silu(z) = z * sigmoid(z). Sources: the 'Mamba (deep learning)' wiki
 * page, paragraph on state space models (A_bar = exp(Delta*A); Delta, B, C made
 * functions of the input), and the 'Mamba-1/2/3 Markdown図解' blog, section 1
 * (h_t = A_bar_t h_{t-1} + B_bar_t x_t, y_t = C_t h_t) and section 2 (the block
 * gates the SSM output with a second branch; training/prefill runs the scan
 * while one-token generation runs the recurrent update of the same model).
 * The input term B_bar_t x_t is read as Delta_t * B_t * u_t, the bias is added
 * before softplus, and D is applied inside the gate: the pages leave those
 * steps open and this library fixes that reading.
 *
 * Conventions common to every entry point:
 *  - All array pointers are device pointers owned by the caller. Calls are
 *    re-entrant and asynchronous on the given stream (NULL = the legacy
 *    default stream). The library's only process-wide state is (a) per-device
 *    caches of kernel attributes and symbol addresses, keyed on the CUDA
 *    context and set up under a lock, and (b) the fixed device scratch of
 *    mamba_scan_bwd_noalloc (below), which calls of that entry point share.
 *  - Strides are in ELEMENTS, and the innermost stride is always 1.
 *  - Arguments are checked on the host before anything touches the GPU; a
 *    failed check returns its MS_ERR_* code and launches nothing.
 *  - dev_status (optional device int): the kernels OR device-detected error
 *    codes into it; the caller zeroes it before the call.
 *  - There is no CPU fallback: without a usable sm_100 device a call returns
 *    MS_ERR_CUDA or MS_ERR_DEVICE.
 */
#ifndef MAMBASCAN_H
#define MAMBASCAN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st *ms_stream_t;

/* Element types of the token-indexed arrays. A, D, delta_bias and every state
   array are always fp32. */
enum { MS_F32 = 0, MS_BF16 = 1 };

/* Status codes. */
enum {
    MS_OK = 0,
    MS_ERR_NULL = 1,      /* a required pointer is NULL                          */
    MS_ERR_DTYPE = 2,     /* in_dtype / out_dtype not MS_F32 or MS_BF16          */
    MS_ERR_SHAPE = 3,     /* negative size, dstate outside [1, 16], or a size    */
                          /* whose element offsets overflow int64                */
    MS_ERR_STRIDE = 4,    /* negative stride                                     */
    MS_ERR_ALIGN = 5,     /* pointer not aligned to its element size             */
    MS_ERR_WORKSPACE = 6, /* workspace argument inconsistent                     */
    MS_ERR_CUDA = 7,      /* a CUDA runtime call failed (no device, launch error)*/
    MS_ERR_TIMEOUT = 8,   /* device: a bounded wait gave up                      */
    MS_ERR_DEVICE = 9,    /* device is not compute capability 10.0 (B200)        */
    MS_ERR_SCRATCH = 10,  /* needs more scratch than the library's fixed buffer  */
    MS_ERR_BOUNDS = 11    /* device, debug build: an index failed a bounds check */
};

/* Maximum d_state the kernels support (Mamba-1 layers use 16). */
#define MS_MAX_DSTATE 16

/*
 * Sizes and strides of one selective-scan call.
 *   u, delta, z, y : [batch, dim, seqlen]   element (b,d,t) at b*x_sb + d*x_sd + t
 *   B, C           : [batch, dstate, seqlen] element (b,n,t) at b*x_sb + n*x_sn + t
 *                    (one group: every channel of a batch row shares B and C)
 *   A              : [dim, dstate] dense;  D, delta_bias : [dim] dense
 *   initial_state, last_state : [batch, dim, dstate] dense fp32
 */
typedef struct {
    int64_t batch, dim, dstate, seqlen;
    int64_t u_sb, u_sd;
    int64_t delta_sb, delta_sd;
    int64_t z_sb, z_sd;
    int64_t y_sb, y_sd;
    int64_t B_sb, B_sn;
    int64_t C_sb, C_sn;
    int32_t in_dtype;  /* u, delta, z, B, C */
    int32_t out_dtype; /* y */
} ms_scan_dims;

/*
 * Workspace bytes mamba_scan_fwd needs for these dims. Usually 0: the scan
 * keeps its state in registers and its tiles in shared memory. When there are
 * too few channels to fill the GPU (batch x dim below ~9,500 on 148 SMs) and
 * the sequence is long (seqlen >= 8192), mamba_scan_fwd splits every batch
 * row's sequence into segments scanned in parallel: a first pass scans the
 * segments from zero for their end states and Delta sums, the carries are
 * chained (the recurrence is linear in the state), and a second pass scans
 * every segment from its true initial state. The workspace (16-byte
 * aligned) holds the segments' states; mamba_scan_fwd_plan with an explicit
 * plan never splits.
 */
size_t mamba_scan_workspace_size(const ms_scan_dims *dims);

/*
 * Selective scan forward over whole sequences (prefill / training forward).
 *   u, delta, B, C   required; delta is the raw step before bias and softplus.
 *   A                required, fp32 [dim, dstate]; real diagonal transition
 *                    (Mamba-1), usually negative.
 *   D, delta_bias    optional fp32 [dim] (NULL = 0).
 *   z                optional gate input (NULL = no gate).
 *   softplus_flag    nonzero: Delta = softplus(delta + bias); zero: delta + bias.
 *   initial_state    optional fp32 [batch, dim, dstate] (NULL = zero state):
 *                    the state before token 0, so that a sequence can be scanned
 *                    in pieces (the state is the only thing carried).
 *   y                required output [batch, dim, seqlen] in out_dtype.
 *   last_state       optional fp32 [batch, dim, dstate] output: the state after
 *                    token seqlen-1 (equal to initial_state, or 0, if seqlen = 0).
 *   workspace        device scratch of mamba_scan_workspace_size() bytes, or
 *                    NULL with workspace_bytes = 0 when that size is 0.
 * Returns MS_OK or an MS_ERR_* code.
 */
int mamba_scan_fwd(const void *u, const void *delta, const float *A, const void *B,
                   const void *C, const float *D, const void *z, const float *delta_bias,
                   int softplus_flag, const float *initial_state, void *y, float *last_state,
                   const ms_scan_dims *dims, void *workspace, size_t workspace_bytes,
                   int *dev_status, ms_stream_t stream);

/*
 * Launch shape of the scan kernel. mamba_scan_fwd picks one from the sizes;
 * mamba_scan_fwd_plan takes it from the caller (tuning and tests). Any valid
 * plan gives the same result up to fp32 rounding.
 *   lanes_per_channel  1, 2, 4 or 8: lanes sharing one channel, each holding
 *                      16/lanes_per_channel of its states.
 *   chunks_per_lane    1 or 2 (1 when lanes_per_channel is 8): 8-token
 *                      chunks each lane prepares per tile; a tile is
 *                      8 * lanes_per_channel * chunks_per_lane tokens.
 *   poly8              0, 2, 4 or 8: eighths of the exponentials computed by
 *                      a polynomial on the FMA pipe instead of the MUFU unit.
 *   engine             MS_ENGINE_REGISTER: the kernel that prefetches each
 *                      lane's token chunks into registers and stages B/C in
 *                      shared memory (any sizes and strides, every option).
 *                      MS_ENGINE_TMEM: token tiles streamed by the TMA engine
 *                      into a shared-memory ring and B/C broadcast to the
 *                      lanes through tensor memory by one tcgen05 product per
 *                      32-token tile (lanes_per_channel 4, chunks_per_lane 1;
 *                      needs dstate 16, seqlen a multiple of 8, 16-byte
 *                      aligned rows and pointers; not for the conv front-end
 *                      or the training forward). Finite B and C are assumed:
 *                      a non-finite value also spoils the other states of its
 *                      token in this engine.
 * mamba_scan_fwd uses MS_ENGINE_TMEM wherever it applies.
 */
enum { MS_ENGINE_REGISTER = 0, MS_ENGINE_TMEM = 1 };

typedef struct {
    int32_t lanes_per_channel;
    int32_t chunks_per_lane;
    int32_t poly8;
    int32_t engine;
} ms_scan_plan;

/* mamba_scan_fwd with an explicit plan (NULL = choose automatically).
   Returns MS_ERR_SHAPE for a plan value outside the lists above, or for
   MS_ENGINE_TMEM where that engine does not apply. */
int mamba_scan_fwd_plan(const void *u, const void *delta, const float *A, const void *B,
                        const void *C, const float *D, const void *z, const float *delta_bias,
                        int softplus_flag, const float *initial_state, void *y, float *last_state,
                        const ms_scan_dims *dims, void *workspace, size_t workspace_bytes,
                        int *dev_status, ms_stream_t stream, const ms_scan_plan *plan);

/* The plan mamba_scan_fwd would choose for these dims on the current device
   (written to *plan). Returns MS_OK or the code mamba_scan_fwd would return
   for invalid dims. */
int mamba_scan_choose_plan(const ms_scan_dims *dims, ms_scan_plan *plan);

/*
 * Scan with the block's causal conv front-end. In the Mamba-1 block (blog,
 * section 2, block diagram) the projected input passes a short causal
 * convolution along the tokens, one filter per channel, and silu before the
 * selective SSM. This entry point takes that convolution's input x and forms
 * the SSM input inside the scan's load stage (u never goes through HBM):
 *     u[b,d,t] = act(conv_b[d] + sum_{k=0}^{W-1} conv_w[d,k] * x[b,d,t-(W-1)+k])
 * with act = silu when silu is nonzero (identity otherwise) and x at t < 0
 * taken from conv_x0[b,d,t+W-1] (zero when conv_x0 is NULL). A sequence
 * scanned in pieces passes the previous piece's last W-1 inputs as conv_x0
 * and its last_state as initial_state. Everything after u is mamba_scan_fwd.
 */
typedef struct {
    int64_t width;            /* W: filter taps, 1..4 (conv_w[d, W-1] weights token t) */
    int64_t uout_sb, uout_sd; /* strides of u_out; inner stride 1 */
    int32_t silu;             /* nonzero: act = silu */
} ms_conv_dims;

/*
 *   x          required input of the convolution, [batch, dim, seqlen] in
 *              dims->in_dtype, strides dims->u_sb / dims->u_sd.
 *   conv_w     required fp32 [dim, W], dense.
 *   conv_b     optional fp32 [dim] (NULL = 0).
 *   conv_x0    optional [batch, dim, W-1] dense, in_dtype: inputs before token 0.
 *   u_out      optional output [batch, dim, seqlen], in_dtype: the computed u
 *              (rounded to in_dtype; the scan itself uses fp32 u).
 *   plan       NULL = automatic; a given plan must have chunks_per_lane 1 and
 *              poly8 0 or 8.
 * The other arguments are those of mamba_scan_fwd; no workspace is needed.
 * Returns MS_OK or an MS_ERR_* code (MS_ERR_SHAPE for W outside [1, 4] or a
 * plan outside the list above).
 */
int mamba_conv_scan_fwd(const void *x, const float *conv_w, const float *conv_b, const void *conv_x0,
                        void *u_out, const ms_conv_dims *cdims, const void *delta, const float *A,
                        const void *B, const void *C, const float *D, const void *z,
                        const float *delta_bias, int softplus_flag, const float *initial_state,
                        void *y, float *last_state, const ms_scan_dims *dims,
                        const ms_scan_plan *plan, int *dev_status, ms_stream_t stream);

/*
 * Training. The forward of a training step also saves the state before every
 * MS_CKPT_TOKENS-token block (fp32 [batch, dim, ceil(seqlen/64), dstate],
 * mamba_scan_ckpt_size() bytes); the backward recomputes each block from it.
 * The blog's section 2 describes training as running the same model through
 * the scan; the gradients are the reverse mode of the recurrence above.
 */
#define MS_CKPT_TOKENS 64

/* Bytes of the saved-state array for these dims (0 when seqlen is 0). */
size_t mamba_scan_ckpt_size(const ms_scan_dims *dims);

/*
 * mamba_scan_fwd that also writes the saved states into ckpt (required,
 * caller-owned, mamba_scan_ckpt_size() bytes, 4-byte aligned).
 */
int mamba_scan_fwd_train(const void *u, const void *delta, const float *A, const void *B,
                         const void *C, const float *D, const void *z, const float *delta_bias,
                         int softplus_flag, const float *initial_state, void *y, float *last_state,
                         float *ckpt, const ms_scan_dims *dims, int *dev_status, ms_stream_t stream);

/* Workspace bytes mamba_scan_bwd needs when it is given no saved states
   (it then recomputes them); 0 is enough when ckpt is given. */
size_t mamba_scan_bwd_workspace_size(const ms_scan_dims *dims);

/*
 * Gradients of the selective scan for a loss with dL/dy = dout and
 * dL/dlast_state = dlast. Inputs are those of the forward (same dims; dout
 * has y's dtype and strides). Gradients are fp32 and dense:
 *   du, ddelta, dz           [batch, dim, seqlen]   (dz only with z; NULL = skip)
 *   dB, dC                   [batch, dstate, seqlen]
 *   dA                       [dim, dstate]
 *   dD, ddelta_bias          [dim]                  (NULL = skip)
 *   dinitial_state           [batch, dim, dstate]   (NULL = skip): dL/d initial_state
 * dA, dB, dC, dD, ddelta_bias are sums over channels, batch rows or tokens,
 * accumulated with fp32 atomics (the library zeroes them first on the
 * stream), so their last bits may differ between runs; the others are
 * written directly. ckpt: the saved states of mamba_scan_fwd_train for the
 * same inputs, or NULL to have them recomputed into the workspace
 * (mamba_scan_bwd_workspace_size() bytes). dlast NULL = 0.
 * Returns MS_OK or an MS_ERR_* code (also MS_ERR_SHAPE for dstate > 16).
 */
int mamba_scan_bwd(const void *u, const void *delta, const float *A, const void *B, const void *C,
                   const float *D, const void *z, const float *delta_bias, int softplus_flag,
                   const float *initial_state, const float *ckpt, const void *dout, const float *dlast,
                   float *du, float *ddelta, float *dA, float *dB, float *dC, float *dD, float *dz,
                   float *ddelta_bias, float *dinitial_state, const ms_scan_dims *dims,
                   void *workspace, size_t workspace_bytes, int *dev_status, ms_stream_t stream);

/*
 * mamba_scan_bwd without saved states, without a caller workspace and without
 * any allocation. The pages have no counterpart: this is mamba_scan_bwd
 * packaged for callers that must not allocate device memory, such as a
 * serving or training runtime whose memory pool claimed the device's free
 * memory at start-up (a cudaMalloc there fails or defeats the pool's
 * accounting), or a latency-critical path where cudaMalloc/cudaFree may
 * synchronize the device and stall other streams. The recomputed saved
 * states go to a fixed scratch array of MS_BWD_NOALLOC_MAX_BYTES compiled
 * into the library as a file-scope __device__ array: every GPU that loads the
 * library holds it until the process exits.
 *  - Set-up: the first call on a device (and the first call after that
 *    device's context was replaced, e.g. by a device reset) looks up the
 *    array's device address with that device current, which may load the
 *    library's module. Make the first call on each device before any stream
 *    capture on it.
 *  - Calls needing more than MS_BWD_NOALLOC_MAX_BYTES of saved states
 *    (mamba_scan_bwd_workspace_size()) return MS_ERR_SCRATCH before any
 *    GPU work.
 *  - The array is shared by all calls on a device and keeps the last call's
 *    contents (every call rewrites what it reads; the accumulated gradients
 *    are zeroed on the stream as in mamba_scan_bwd). Two calls that overlap
 *    on one device (different streams, or host threads without ordering)
 *    race on it; calls on one stream, or ordered by events, are safe.
 *  - Nothing is allocated: no cudaMalloc, cudaFree or allocating library
 *    routine, on any call.
 * Arguments and results are those of mamba_scan_bwd with ckpt = NULL.
 */
#define MS_BWD_NOALLOC_MAX_BYTES ((size_t)96 << 20)

int mamba_scan_bwd_noalloc(const void *u, const void *delta, const float *A, const void *B, const void *C,
                           const float *D, const void *z, const float *delta_bias, int softplus_flag,
                           const float *initial_state, const void *dout, const float *dlast, float *du,
                           float *ddelta, float *dA, float *dB, float *dC, float *dD, float *dz,
                           float *ddelta_bias, float *dinitial_state, const ms_scan_dims *dims,
                           int *dev_status, ms_stream_t stream);

/*
 * Mamba-2 state space duality (SSD) layer, forward ('Mamba-1/2/3 Markdown図解'
 * blog, section 3: the same model has a recurrent view and a matrix view
 * computed chunk by chunk, matrix products inside a chunk and the state
 * passed between chunks; the transition is a scalar times the identity in a
 * head). For batch b, head h with head dim P and state N, and group
 * g = h / (nheads / ngroups) whose B and C it uses:
 *     Delta_t = softplus(dt[b,t,h] + dt_bias[h])   (plain sum when the flag is 0)
 *     S_t[p][n] = exp(Delta_t A[h]) S_{t-1}[p][n] + Delta_t x[b,t,h,p] B[b,t,g,n]
 *     y[b,t,h,p] = sum_n C[b,t,g,n] S_t[p][n] + D[h] x[b,t,h,p]
 * Layouts (element strides; the last dimension of each array is dense):
 *   x, y [batch, seqlen, nheads, headdim]; dt [batch, seqlen, nheads];
 *   B, C [batch, seqlen, ngroups, dstate]; A, D, dt_bias [nheads] fp32;
 *   initial_state, final_state [batch, nheads, headdim, dstate] fp32, dense.
 * This version runs headdim 64 and dstate 128 (the Mamba-2 layer sizes) with
 * bf16 x, dt, B, C (MS_ERR_SHAPE / MS_ERR_DTYPE otherwise); x, B, C rows must
 * be 16-byte aligned and y rows aligned to two elements (MS_ERR_ALIGN).
 * y is fp32 or bf16 (out_dtype). D, dt_bias, initial_state, final_state may
 * be NULL; initial_state may be the same array as final_state.
 * The chunks (128 tokens) run in parallel on the tcgen05 tensor cores; the
 * state entering a chunk is handed over from the previous chunk's work item
 * through the workspace.
 *   workspace        caller-owned device memory of mamba2_ssd_workspace_size()
 *                    bytes (batch x nheads running states of headdim x dstate
 *                    fp32 and batch x nheads + 1 counters), 16-byte aligned;
 *                    its contents need not be kept between calls, but two
 *                    calls in flight at once need two workspaces. Too small:
 *                    MS_ERR_WORKSPACE.
 *   dev_status       receives MS_ERR_TIMEOUT if a bounded wait inside the
 *                    kernel ran out (y and final_state are then undefined).
 */
typedef struct {
    int64_t batch, seqlen, nheads, headdim, dstate, ngroups;
    int64_t x_sb, x_sl, x_sh;
    int64_t dt_sb, dt_sl;
    int64_t B_sb, B_sl, B_sg;
    int64_t C_sb, C_sl, C_sg;
    int64_t y_sb, y_sl, y_sh;
    int32_t in_dtype, out_dtype;
} ms_ssd_dims;

size_t mamba2_ssd_workspace_size(const ms_ssd_dims *dims);
int mamba2_ssd_fwd(const void *x, const void *dt, const float *A, const void *B, const void *C,
                   const float *D, const float *dt_bias, int softplus_flag, const float *initial_state,
                   void *y, float *final_state, const ms_ssd_dims *dims, void *workspace,
                   size_t workspace_bytes, int *dev_status, ms_stream_t stream);

/*
 * Mamba-2 SSD layer: the intra-chunk products of the chunked matrix view
 * ('Mamba-1/2/3 Markdown図解' blog, section 3: inside a chunk the output is
 * built from the products C_t . B_s of the chunk's tokens), for chunks of 32
 * tokens, computed on the tcgen05 tensor cores once per group:
 *     cb[b][g][k][i][j] = sum_n C[b, 32k+i, g, n] B[b, 32k+j, g, n]
 * for i, j < 32 (tokens at or past seqlen count as zero). cb is [batch,
 * ngroups, ceil(seqlen / 32), 32, 32] fp32, dense, caller-owned device memory
 * of mamba2_ssd_chunk_cb_size() bytes, 16-byte aligned. B, C and their
 * fields of dims are as for mamba2_ssd_fwd (bf16, dstate 128, rows 16-byte
 * aligned: MS_ERR_DTYPE / MS_ERR_SHAPE / MS_ERR_ALIGN otherwise); the other
 * fields of dims are not read. dev_status receives MS_ERR_TIMEOUT if a
 * product did not complete within the kernel's bounded wait.
 */
size_t mamba2_ssd_chunk_cb_size(const ms_ssd_dims *dims);
int mamba2_ssd_chunk_cb(const void *B, const void *C, float *cb, const ms_ssd_dims *dims, int *dev_status,
                        ms_stream_t stream);

/*
 * Mamba-2 SSD layer, one token (decode): the recurrent view of the same model
 * (blog, section 3: generation updates the state once per token). For batch
 * row b, head h, group g = h / (nheads / ngroups):
 *     Delta = softplus(dt[b,h] + dt_bias[h])   (plain sum when the flag is 0)
 *     S[p][n] = exp(Delta A[h]) S[p][n] + Delta x[b,h,p] B[b,g,n]
 *     y[b,h,p] = sum_n C[b,g,n] S[p][n] + D[h] x[b,h,p]
 * state [batch, nheads, headdim, dstate] fp32 is read and overwritten; each
 * head's [headdim, dstate] block is dense, 16-byte aligned. x, y [batch,
 * nheads, headdim]; dt [batch, nheads]; B, C [batch, ngroups, dstate]
 * (innermost dimension dense). This version runs dstate 128 (MS_ERR_SHAPE
 * otherwise), any headdim; x, dt, B, C fp32 or bf16, y fp32 or bf16.
 */
typedef struct {
    int64_t batch, nheads, headdim, dstate, ngroups;
    int64_t x_sb, x_sh;
    int64_t dt_sb;
    int64_t B_sb, B_sg;
    int64_t C_sb, C_sg;
    int64_t y_sb, y_sh;
    int64_t state_sb, state_sh;
    int32_t in_dtype, out_dtype;
} ms_ssd_update_dims;

int mamba2_ssd_state_update(float *state, const void *x, const void *dt, const float *A, const void *B,
                            const void *C, const float *D, const float *dt_bias, int softplus_flag, void *y,
                            const ms_ssd_update_dims *dims, int *dev_status, ms_stream_t stream);

/*
 * Sizes and strides of one decode step.
 *   x, delta, z, y : [batch, dim]     element (b,d) at b*x_sb + d
 *   B, C           : [batch, dstate]  element (b,n) at b*x_sb + n
 *   state          : [batch, dim, dstate] fp32, element (b,d,n) at
 *                    b*state_sb + d*state_sd + n
 *   A [dim, dstate], D [dim], delta_bias [dim] dense fp32.
 */
typedef struct {
    int64_t batch, dim, dstate;
    int64_t x_sb, delta_sb, z_sb, y_sb;
    int64_t B_sb, C_sb;
    int64_t state_sb, state_sd;
    int32_t in_dtype;  /* x, delta, z, B, C */
    int32_t out_dtype; /* y */
} ms_update_dims;

/*
 * Selective state update: one token for every (b, d), the recurrent form used
 * for generation (blog, section 2). Reads the fp32 state, applies the same
 * step as the scan, writes the new state in place and y.
 *   state            required, read and overwritten.
 *   x, delta, A, B, C, y required; D, delta_bias, z optional as in the scan.
 * Returns MS_OK or an MS_ERR_* code.
 */
int mamba_state_update(float *state, const void *x, const void *delta, const float *A,
                       const void *B, const void *C, const float *D, const void *z,
                       const float *delta_bias, int softplus_flag, void *y,
                       const ms_update_dims *dims, int *dev_status, ms_stream_t stream);

/*
 * Test hook for device failure detection (the pages have no counterpart):
 * launches one CTA that waits, with the library's bounded barrier wait, on a
 * barrier that nothing completes. After `rounds` tries (1 .. 1048576) the
 * wait gives up, MS_ERR_TIMEOUT is ORed into *dev_status (required device
 * int) and the kernel ends; the context stays usable. This is the path every
 * bounded wait of the library takes when what it waits for never comes.
 * Returns MS_ERR_NULL / MS_ERR_SHAPE for bad arguments, else MS_OK or
 * MS_ERR_CUDA (the timeout itself is reported through *dev_status).
 */
int mamba_debug_bounded_wait(uint32_t rounds, int *dev_status, ms_stream_t stream);

/*
 * Debug build check (the pages have no counterpart). libmambascan_debug.so is
 * this library compiled with MS_DEBUG: its kernels test their shared-memory,
 * tensor-memory and global indexes against the buffers they address, and a
 * failing test ORs MS_ERR_BOUNDS into *dev_status and skips the access
 * instead of performing it (the stand-in for a memory checker on a pool where
 * none can run). This hook launches one thread that writes element `index` of
 * a 16-int device array through such a check: index in [0, 16) writes, any
 * other index is recorded and skipped. In the product library (not built with
 * MS_DEBUG) it launches nothing and returns MS_ERR_SHAPE.
 * Returns MS_ERR_NULL without dev_status, else MS_OK or MS_ERR_CUDA.
 */
int mamba_debug_bounds_probe(int32_t index, int *dev_status, ms_stream_t stream);

/* 1 when this library is the MS_DEBUG build, else 0. */
int mamba_debug_build(void);

/* Static English text for a status code (never NULL). */
const char *mamba_status_string(int code);

/* MS_OK when the current CUDA device is usable (compute capability 10.0);
   MS_ERR_CUDA when there is no device, MS_ERR_DEVICE for another GPU. */
int mamba_device_check(void);

#ifdef __cplusplus
}
#endif

#endif /* MAMBASCAN_H */
