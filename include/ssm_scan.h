/*
 * ssm_scan.h -- C ABI of the B200 (sm_100a) selective-SSM (S6) forward scan.
 *
 * The operation (Mamba "architecture-details" page, section "How S6 Works";
 * "Agent 229: SSM optimization patterns" page, section 7 "Selective Attention
 * Mechanism" for A_bar = exp(delta*A)): for every batch row b, channel d and
 * state n, walking t = 0 .. L-1 from h = 0,
 *
 *     dt      = softplus(delta[b,hd,t] + delta_bias[hd])     (or without softplus)
 *     h[n]    = exp(dt * A[d,n]) * h[n] + dt * B[b,g,n,t] * u[b,d,t]
 *     y       = sum_n C[b,g,n,t] * h[n] + D[d] * u[b,d,t]
 *     out     = y * silu(z[b,d,t]),     silu(z) = z / (1 + exp(-z))
 *
 * and the state after the last step is returned as last_state[b,d,:].
 * hd = d / (dim/nheads) is the channel's head (hd = d when nheads == dim) and
 * g = d / (dim/ngroups) its B/C group.  With nheads < dim, A holds one scalar
 * per head (A[hd] for every n), the layout of Mamba-2 ("SKILL" page, Mamba-2
 * section: headdim, ngroups, d_state=128).
 *
 * Arithmetic: fp32 in registers (state, dt, products), inputs and outputs in
 * the I/O dtype (fp32 or bf16, rounded to nearest even on output).
 *
 * Layouts -- every tensor is contiguous, row-major, in device memory owned by
 * the caller:
 *   u, z, out    (batch, dim, seqlen)          io dtype
 *   delta        (batch, nheads, seqlen)       io dtype
 *   B, C         (batch, ngroups, dstate, seqlen) io dtype
 *   A            (dim, dstate) fp32, or (nheads) fp32 when nheads < dim
 *   D            (dim) fp32                     nullable: no skip term
 *   delta_bias   (nheads) fp32                  nullable: zero bias
 *   z            nullable: no gate (out = y)
 *   last_state   (batch, dim, dstate) fp32      nullable: not written
 *
 * Errors: every call returns an ssm_status_t.  Argument checks happen on the
 * host before anything is launched; kernel-side conditions (a bounded wait
 * that ran out, a debug bounds check) are recorded in the plan's device status
 * word and read back with ssm_scan_device_status.  No call traps, asserts or
 * aborts on the device.
 */
#ifndef SSM_SCAN_H
#define SSM_SCAN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* The CUDA stream type, declared without including the CUDA headers:
 * a cudaStream_t converts to it as is; NULL is the legacy default stream. */
struct CUstream_st;
typedef struct CUstream_st* ssm_stream_t;

typedef enum {
    SSM_OK = 0,
    SSM_ERR_INVALID_ARG = 1, /* NULL required pointer, bad size, dims != plan dims, destroyed plan */
    SSM_ERR_UNSUPPORTED = 2, /* a shape or dtype no kernel here handles (e.g. dstate not in {8,16,32,64,128}) */
    SSM_ERR_CUDA = 3,        /* a CUDA runtime call failed (allocation, launch, copy) */
    SSM_ERR_TIMEOUT = 4,     /* device side: a bounded inter-CTA wait gave up */
    SSM_ERR_BOUNDS = 5       /* device side: a bounds or alignment check fired */
} ssm_status_t;

typedef enum { SSM_F32 = 0, SSM_BF16 = 1 } ssm_dtype_t;

/* Problem shape.  nheads == dim is the S6 layout (per-channel delta, A, bias);
 * nheads < dim gives one delta row, bias and scalar A per head.  dim must be a
 * multiple of nheads and of ngroups. */
typedef struct {
    int64_t batch;    /* B */
    int64_t dim;      /* D: channels (d_inner) */
    int64_t seqlen;   /* L */
    int64_t dstate;   /* N */
    int64_t nheads;   /* H: == dim for S6 */
    int64_t ngroups;  /* G: B/C groups */
    int32_t io_dtype; /* ssm_dtype_t of u, delta, z, B, C, out */
    int32_t reserved; /* must be 0 */
} ssm_dims_t;

typedef struct ssm_plan_s* ssm_plan_t;

/*
 * Create a plan for one problem shape on one device: validates the shape,
 * picks the kernel and allocates the plan's own device workspace (the status
 * word and the chunk-carry buffers).  The plan belongs to the caller until
 * ssm_scan_destroy.  Returns SSM_ERR_INVALID_ARG for a NULL out_plan or a bad
 * shape, SSM_ERR_UNSUPPORTED for a shape no kernel handles, SSM_ERR_CUDA when
 * the device cannot be used or the workspace cannot be allocated.
 */
int ssm_scan_plan(ssm_plan_t* out_plan, const ssm_dims_t* dims, int device);

/*
 * The forward scan (the operation above), asynchronous on `stream`.
 * `dims` must equal the plan's dims.  Pointers are device pointers owned by
 * the caller and are not kept after the call returns; `out` must not alias an
 * input.  softplus != 0 applies softplus to delta + delta_bias; with softplus
 * == 0, delta + delta_bias is dt itself and must be >= 0 (with A <= 0 every
 * exp(dt*A) is then <= 1; a dt*A above about 88 overflows fp32).
 * Allocates nothing.  One plan must not run on two streams at once.
 * Returns SSM_ERR_INVALID_ARG for a NULL required pointer (u, delta, A, B, C,
 * out) or mismatched dims, SSM_ERR_CUDA if the launch fails.
 */
int ssm_selective_scan_fwd(ssm_plan_t plan, const void* u, const void* delta, const float* A,
                           const void* B, const void* C, const float* D, const void* z,
                           const float* delta_bias, int softplus, const ssm_dims_t* dims, void* out,
                           float* last_state, ssm_stream_t stream);

/*
 * Same as ssm_selective_scan_fwd, starting from the state h0 (batch, dim, dstate)
 * fp32 instead of zero (h0 == NULL means zero).  Running [0, L1) and then
 * [L1, L) with h0 = the first call's last_state gives the same result as one
 * run over [0, L) ("Agent 229" page, section 9 "Chunked Computation": the final
 * state of a chunk is the initial state of the next).  h0 may alias last_state.
 */
int ssm_selective_scan_fwd_h0(ssm_plan_t plan, const void* u, const void* delta, const float* A,
                              const void* B, const void* C, const float* D, const void* z,
                              const float* delta_bias, int softplus, const ssm_dims_t* dims,
                              const float* h0, void* out, float* last_state, ssm_stream_t stream);

/*
 * The forward for training: ssm_selective_scan_fwd_h0 that also stores the states the
 * backward walks from, so that ssm_selective_scan_bwd_ckpt skips its recomputation pass
 * ("Agent 229" page, section 4 "Activation Recomputation": checkpoints at chunk
 * boundaries, recompute inside a chunk).  ckpt (device, fp32, required, 8-byte aligned,
 * caller-owned) receives (batch, dim, ceil(seqlen/8), dstate): element
 * [b][d][k][n] is the state h[n] of channel (b, d) entering step 8k (k = 0 holds h0, or
 * zero): the start of every 8-step window the backward recomputes, so that it rebuilds
 * none.  About batch*dim*seqlen*dstate/2 bytes.  Every other argument and output is
 * ssm_selective_scan_fwd_h0's, bit for bit.  Covered: the shapes the backward covers
 * (the S6 layout, nheads == dim, with dstate 16), on the register kernel; another shape, or
 * a plan forced onto the tensor-memory kernel, returns SSM_ERR_UNSUPPORTED.
 * SSM_ERR_INVALID_ARG as ssm_selective_scan_fwd, or for ckpt NULL.
 */
int ssm_selective_scan_fwd_ckpt(ssm_plan_t plan, const void* u, const void* delta, const float* A,
                                const void* B, const void* C, const float* D, const void* z,
                                const float* delta_bias, int softplus, const ssm_dims_t* dims,
                                const float* h0, void* out, float* last_state, float* ckpt,
                                ssm_stream_t stream);

/*
 * End-to-end variant: the same arguments as ssm_selective_scan_fwd but every
 * tensor pointer is HOST memory (pinned memory makes the copies asynchronous).
 * The plan allocates device copies on first use (kept until ssm_scan_destroy);
 * each call copies the inputs host->device, runs the scan and copies out (and
 * last_state, if given) device->host.  With batch >= 2 the batch rows are cut
 * into chunks (the largest divisor of batch up to 8) that are pipelined on three
 * streams the plan owns (copies in, scans through a plan for one chunk, copies
 * out), so the copies in both directions and the scans overlap; the call is
 * ordered after the work already on `stream`, and later work on `stream` waits
 * for it.  The host outputs are complete once `stream` is synchronised.
 */
int ssm_selective_scan_fwd_host(ssm_plan_t plan, const void* u, const void* delta, const float* A,
                                const void* B, const void* C, const float* D, const void* z,
                                const float* delta_bias, int softplus, const ssm_dims_t* dims,
                                void* out, float* last_state, ssm_stream_t stream);

/*
 * Plan options (mostly for tests).  Changing SEG_LEN, CONSUMER_WARPS, WORKERS,
 * STATES_PER_LANE or SSD re-plans the schedule (synchronises the device).
 *   SSM_OPT_SPIN_LIMIT         polls a chained wait makes before it gives up and
 *                              records SSM_ERR_TIMEOUT (default about 2M, i.e. ~1 s)
 *   SSM_OPT_INJECT_STALL       test hook, nonzero: every chained wait waits for a
 *                              flag that no worker ever sets, so it runs out and the
 *                              call reports SSM_ERR_TIMEOUT (outputs are then invalid);
 *                              0 switches it off
 *   SSM_OPT_SEG_LEN            force the segment length (rounded up to 32 steps);
 *                              0 = automatic
 *   SSM_OPT_CONSUMER_WARPS     force 4, 8, 12 or 16 consumer warps per CTA (16 exists
 *                              for dstate <= 16 with 2 states per lane, 12 for dstate
 *                              16 with 4); 0 = automatic
 *   SSM_OPT_WORKERS            cap the number of persistent CTAs; 0 = one per SM
 *   SSM_OPT_STATES_PER_LANE    force the states each lane holds (2 or 4 for dstate <= 16,
 *                              4 for dstate 32, dstate/8 above); 0 = automatic.  A
 *                              combination with CONSUMER_WARPS that no kernel has makes
 *                              the call return SSM_ERR_UNSUPPORTED and keeps the
 *                              previous setting.
 *   SSM_OPT_SSD                the chunked tensor-core (state-space-dual) path for bf16
 *                              I/O, nheads < dim with dim/nheads == 64, dstate 128 and
 *                              seqlen a multiple of 128: 0 = use it where it applies
 *                              (automatic), 1 = never (the scan kernel), 2 = required
 *                              (SSM_ERR_UNSUPPORTED for a shape it does not cover)
 *   SSM_OPT_TIME_LANES         force the time sub-chunks per 32-step block: 1 = the
 *                              state-parallel recurrence, 2 or 4 = sequence-parallel
 *                              blocks (lanes split the block in time and join their
 *                              sub-chunks by an associative scan; dstate <= 16);
 *                              0 = automatic
 *   SSM_OPT_TENSOR_MEMORY      the kernel that brings B and C to the lanes through
 *                              tensor memory (bf16 I/O, dstate 16, A per channel): 0 =
 *                              use it where it applies (automatic), 1 = never (the
 *                              register kernel), 2 = required (SSM_ERR_UNSUPPORTED for a
 *                              shape it does not cover)
 * Returns SSM_ERR_INVALID_ARG for an unknown option or a bad value.
 */
typedef enum {
    SSM_OPT_SPIN_LIMIT = 1,
    SSM_OPT_INJECT_STALL = 2,
    SSM_OPT_SEG_LEN = 3,
    SSM_OPT_CONSUMER_WARPS = 4,
    SSM_OPT_WORKERS = 5,
    SSM_OPT_STATES_PER_LANE = 6,
    SSM_OPT_SSD = 7,
    SSM_OPT_TIME_LANES = 8,
    SSM_OPT_TENSOR_MEMORY = 9
} ssm_option_t;
int ssm_scan_set_option(ssm_plan_t plan, int option, int64_t value);

/*
 * The plan's schedule: consumer warps per CTA, segment length (time steps per
 * work unit), channel tiles, segments per tile and persistent CTAs.  NULL
 * outputs are skipped.
 */
int ssm_scan_plan_schedule(ssm_plan_t plan, int* consumer_warps, int* seg_len, int* n_tiles, int* n_seg,
                           int* n_ctas);

/*
 * The forward scan without a plan and without any device allocation (no
 * counterpart in the pages: this is a deployment convenience).  For callers that
 * cannot call cudaMalloc -- code inside a framework that owns all device memory
 * through its own pre-reserved pool, or a hot path that must not take an
 * allocation's latency and failure mode.  Same arguments and layouts as
 * ssm_selective_scan_fwd, minus the plan; device pointers, current device.
 *   - Scratch comes from a fixed 8 MiB __device__ array held by every GPU that
 *     loads the library until exit; a problem whose workspace does not fit
 *     (about batch * dim * dstate * 4 bytes of carry states) returns
 *     SSM_ERR_UNSUPPORTED without launching anything.
 *   - The first call on a device looks up the array's address (once per device);
 *     make that first call before any stream capture.
 *   - Under CUDA's lazy module loading (the default) the array and the kernels
 *     are placed in device memory at that first call, not when the library is
 *     loaded: a caller that reserves all of its device memory for its own pool
 *     should make one warm-up call first, or run with CUDA_MODULE_LOADING=EAGER.
 *   - All calls share the array: each clears its counters, flags and status on
 *     its stream, and calls whose kernels overlap on the GPU race and must not
 *     be made.
 *   - Kernel-side conditions (a bounded wait that gave up: SSM_ERR_TIMEOUT, with
 *     out and last_state invalid) land in the array's status word; read them
 *     with ssm_selective_scan_noalloc_device_status before the next call.
 * Calls no cudaMalloc, cudaFree or other allocating routine.
 */
int ssm_selective_scan_fwd_noalloc(const void* u, const void* delta, const float* A, const void* B, const void* C,
                                   const float* D, const void* z, const float* delta_bias, int softplus,
                                   const ssm_dims_t* dims, void* out, float* last_state, ssm_stream_t stream);

/*
 * The kernel-side status of the last ssm_selective_scan_fwd_noalloc call on the
 * current device (no counterpart in the pages).  Waits for `stream`, returns the
 * status word of the shared scratch array (SSM_OK, or SSM_ERR_TIMEOUT when a
 * bounded wait gave up) and clears it.  Allocates nothing.  SSM_ERR_CUDA if the
 * copy or the synchronisation fails.
 */
int ssm_selective_scan_noalloc_device_status(ssm_stream_t stream);

/*
 * Test hook of the allocation-free entry point (no counterpart in the pages).
 * stall != 0 makes the chained waits of the following calls wait for a flag
 * that nothing sets, so that they give up and report SSM_ERR_TIMEOUT;
 * spin_limit (0 = default, else 1 .. 2^31-1; about 256 ns per unit) bounds
 * every device-side wait of those calls.  Host-side settings of this process.
 */
int ssm_selective_scan_noalloc_test_hooks(int stall, int64_t spin_limit);

/*
 * One step of the recurrence with the state kept in device memory: the
 * inference mode of the Mamba "architecture-details" page ("Parallel
 * Algorithm": the sequential, RNN-style mode; "Memory Efficiency": a
 * constant-size state and no cache of past inputs).  For every (b, d):
 *
 *     dt = softplus(delta[b,hd] + delta_bias[hd]),   h = state[b,d,:]
 *     h[n] = exp(dt * A[d,n]) * h[n] + dt * B[b,g,n] * u[b,d]
 *     out[b,d] = (sum_n C[b,g,n] * h[n] + D[d] * u[b,d]) * silu(z[b,d])
 *     state[b,d,:] = h                       (overwritten in place)
 *
 * This is exactly ssm_selective_scan_fwd_h0 with seqlen 1 and h0 = last_state
 * = state.  dims->seqlen must be 1: u, z, out are (batch, dim), delta is
 * (batch, nheads), B and C are (batch, ngroups, dstate), in the io dtype; A, D,
 * delta_bias and the fp32 state (batch, dim, dstate) are as for the scan.  No
 * plan and no workspace: the call allocates nothing and launches one kernel on
 * `stream`.  state must be 16-byte aligned, B and C 8-byte (bf16) or 16-byte
 * (fp32) aligned, and A 16-byte aligned in the per-channel layout; otherwise
 * SSM_ERR_UNSUPPORTED.  SSM_ERR_INVALID_ARG for a NULL required pointer (state,
 * u, delta, A, B, C, out), seqlen != 1 or a bad shape.
 */
int ssm_selective_state_update(const ssm_dims_t* dims, float* state, const void* u, const void* delta,
                               const float* A, const void* B, const void* C, const float* D, const void* z,
                               const float* delta_bias, int softplus, void* out, ssm_stream_t stream);

/*
 * The causal depthwise convolution in front of the scan (Mamba
 * "architecture-details" page, "Model Configuration": d_conv, the convolution
 * width, and conv_bias; "Parameter Impact": the local context window before the
 * SSM).  For every (b, d, t), with x taken as zero before t = 0:
 *
 *     v = bias[d] + sum_{k < width} w[d,k] * x[b,d,t - width + 1 + k]
 *     out[b,d,t] = silu ? v / (1 + exp(-v)) : v
 *
 * x and out are (batch, dim, seqlen) in io_dtype (ssm_dtype_t), w is (dim,
 * width) fp32, bias is (dim) fp32 or NULL (zero).  The pages name the
 * convolution but not what follows it, so the SiLU is a flag.  width is 1 to 4
 * (4 is the pages' standard), else SSM_ERR_UNSUPPORTED.  No plan, no workspace:
 * one kernel on `stream`.  out must not alias x.  SSM_ERR_INVALID_ARG for a bad
 * shape or dtype or a NULL x, w or out.
 */
int ssm_causal_conv1d_fwd(int64_t batch, int64_t dim, int64_t seqlen, int32_t width, int32_t io_dtype,
                          const void* x, const float* w, const float* bias, int silu, void* out,
                          ssm_stream_t stream);

/*
 * Gradients of the forward scan (ssm_selective_scan_fwd_h0), for training: the
 * backward pass.  The states are not kept by the forward; this call recomputes
 * them ("Agent 229: SSM optimization patterns" page, section 4 "Activation
 * Recomputation": recompute in the backward pass, checkpoint at chunk
 * boundaries; Mamba "architecture-details" page, "Memory Efficiency").  Given
 * dout = dLoss/dout and dlast = dLoss/dlast_state (nullable: zero), with
 * dt, dA = exp(dt*A), h, y as in the forward and g the gradient of the state
 * carried back from step t+1 (dlast at the last step):
 *
 *     dy    = dout * silu(z)                g[n] += dy * C[n]    (= dLoss/dh_t)
 *     dB[n] += g[n] * dt * u                dC[n] += dy * h_t[n]  (summed over channels)
 *     du    = dt * sum_n g[n] B[n] + dy * D
 *     ddt   = u * sum_n g[n] B[n] + sum_n g[n] h_(t-1)[n] A[n] dA[n]
 *     dA[n] += g[n] h_(t-1)[n] dt dA[n]        g[n] *= dA[n]   (carried to t-1)
 *     ddelta = ddt * sigmoid(delta + delta_bias)  (ddt without softplus)
 *     ddelta_bias += ddelta,  dD += dy * u,  dz = dout * y * silu'(z)
 *     dh0 = g after step 0
 *
 * Covered: every layout with dstate in {8, 16, 32, 64, 128}; other dstates return
 * SSM_ERR_UNSUPPORTED.  The S6 layout (nheads == dim) with dstate 16 and dim/ngroups a
 * multiple of 32 runs on the tiled kernel described below.  Every other covered shape
 * (the per-head layout, where A, delta and delta_bias are per head and ddelta, dA and
 * ddelta_bias are summed over each head's channels; the other dstates) runs on a generic
 * kernel: one CTA per group of channels for the whole sequence (no inter-CTA waits),
 * states recomputed from workspace checkpoints every 256 steps; correct, not tuned, and
 * its ddelta for the per-head layout is a sum of atomic adds as well.  Inputs and layouts are the
 * forward's (h0 nullable: zero); dout is (batch, dim, seqlen) in the io dtype,
 * dlast (batch, dim, dstate) fp32.  Outputs (ssm_grads_t, device memory owned
 * by the caller, every one overwritten):
 *     du, dz        (batch, dim, seqlen) io dtype; dz required iff z != NULL
 *     ddelta        (batch, nheads, seqlen) io dtype
 *     dA            like A, fp32
 *     dB, dC        (batch, ngroups, dstate, seqlen) fp32
 *     dD            (dim) fp32, nullable: not computed
 *     ddelta_bias   (nheads) fp32, nullable: not computed
 *     dh0           (batch, dim, dstate) fp32, nullable: not computed
 * The call allocates nothing: `workspace` (device, 256-byte aligned, at least
 * ssm_selective_scan_bwd_workspace_size bytes, which depends on the shape and on
 * the current device's SM count; about batch*dim*seqlen*2 bytes of state
 * checkpoints, one per 32 steps) is the caller's and is scratch after the call;
 * one workspace must not serve two calls at once.  Two kernels on `stream`
 * (after memsets of the workspace's counters and of dB and dC).  dB and dC, sums
 * over the channels of a group, are added up by atomic adds, so their last bits
 * may differ between calls; every other gradient is summed in a fixed order and
 * repeats bit for bit.  The first kernel runs work units
 * (32 channels x a segment of the sequence) on persistent CTAs whose bounded waits
 * record SSM_ERR_TIMEOUT in the workspace; read it with
 * ssm_selective_scan_bwd_device_status.  A, h0, dlast and dh0 must be 8-byte
 * aligned (else SSM_ERR_UNSUPPORTED).  SSM_ERR_INVALID_ARG for a NULL required
 * pointer (u, delta, A, B, C, dout, grads, du, ddelta, dA, dB, dC, workspace),
 * a bad shape or a workspace that is too small.
 */
typedef struct {
    void* du;
    void* ddelta;
    float* dA;
    float* dB;
    float* dC;
    float* dD;
    void* dz;
    float* ddelta_bias;
    float* dh0;
} ssm_grads_t;

int ssm_selective_scan_bwd_workspace_size(const ssm_dims_t* dims, size_t* bytes);

int ssm_selective_scan_bwd(const ssm_dims_t* dims, const void* u, const void* delta, const float* A,
                           const void* B, const void* C, const float* D, const void* z,
                           const float* delta_bias, int softplus, const float* h0, const void* dout,
                           const float* dlast, const ssm_grads_t* grads, void* workspace,
                           size_t workspace_bytes, ssm_stream_t stream);

/*
 * ssm_selective_scan_bwd given the states ssm_selective_scan_fwd_ckpt stored (ckpt, the
 * same layout; device, 8-byte aligned (16-byte aligned: copied in 16-byte pieces), read
 * only) for the same inputs and h0: the kernel then runs no forward recomputation units,
 * writes no checkpoints of its own and rebuilds no window starts: it reads them from ckpt
 * (the workspace size is the same).  ckpt == NULL is exactly
 * ssm_selective_scan_bwd.  The gradients are those of ssm_selective_scan_bwd (the
 * states it would recompute are the ones the forward stored, bit for bit).
 */
int ssm_selective_scan_bwd_ckpt(const ssm_dims_t* dims, const void* u, const void* delta, const float* A,
                                const void* B, const void* C, const float* D, const void* z,
                                const float* delta_bias, int softplus, const float* h0, const void* dout,
                                const float* dlast, const float* ckpt, const ssm_grads_t* grads,
                                void* workspace, size_t workspace_bytes, ssm_stream_t stream);

/* Synchronise `stream` and return the kernel-side status of the last backward call that
 * used `workspace` (SSM_OK or SSM_ERR_TIMEOUT), clearing it. */
int ssm_selective_scan_bwd_device_status(void* workspace, ssm_stream_t stream);

/* Test hooks of the backward, process-wide, for tests only.  stall != 0 makes every
 * wait of a chained work unit wait for a flag value that nothing writes, so the wait
 * runs out, the call records SSM_ERR_TIMEOUT and its outputs are invalid;
 * wait_budget_us > 0 replaces the default limit of a wait (about 1 s), 0 restores it.
 * SSM_ERR_INVALID_ARG for a budget outside [0, 10 s]. */
int ssm_selective_scan_bwd_test_hooks(int stall, int64_t wait_budget_us);

/* Release the plan and its workspace.  NULL is accepted.  Synchronises the device. */
int ssm_scan_destroy(ssm_plan_t plan);

/*
 * Synchronise `stream`, return the kernel-side status recorded since the last
 * call (SSM_OK, SSM_ERR_TIMEOUT, SSM_ERR_BOUNDS) and clear it.
 */
int ssm_scan_device_status(ssm_plan_t plan, ssm_stream_t stream);

/* Static, human-readable text for a status code. */
const char* ssm_status_string(int status);

/*
 * Launch facts of the plan's kernel, for measurement and tests: the grid size,
 * threads per CTA, dynamic shared memory bytes, kernel launches per forward
 * call, and the variant name (static string).  Any output pointer may be NULL.
 */
int ssm_scan_plan_info(ssm_plan_t plan, int* grid, int* block, int* smem_bytes, int* launches_per_call,
                       const char** variant);

/*
 * Measurement helper (not part of the scan): runs `blocks` CTAs of 256 threads,
 * each thread issuing `iters` x 16 independent ex2.approx operations, and
 * writes a checksum per thread to `sink` (blocks*256 floats, device memory).
 * The bench times it to measure the MUFU ex2 rate of the GPU it runs on.
 */
int ssm_probe_ex2(float* sink, int blocks, int iters, ssm_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* SSM_SCAN_H */
