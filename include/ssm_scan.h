/*
 * ssm_scan.h -- C ABI of the B200 (sm_100a) selective state-space scan.
 *
 * The operation (page titles and sections cited):
 *   "Selective Scan trong Mamba toi uu chuoi dai the nao?" (thecsnote.cc)
 *     - "Tai sao Mamba can Selective Scan?": the discrete recurrence
 *       h_t = Abar h_{t-1} + Bbar x_t, y_t = C h_t.
 *     - "Selection pha vo convolution kernel co dinh": B_t, C_t and
 *       Delta_t = softplus(theta + s(x_t)) change per token, so
 *       h_t = Abar_t h_{t-1} + Bbar_t x_t, y_t = C_t h_t.
 *     - "Vi du Python": diagonal A, Abar_t = exp(Delta_t * A).
 *     - "Scan bien recurrence thanh phep toan co the song song hoa ra sao?":
 *       the per-token affine maps compose associatively,
 *       (A2, b2) (x) (A1, b1) = (A2 A1, A2 b1 + b2).
 *     - "Tai sao chi parallel scan van chua du nhanh?" / "Kernel fusion":
 *       the (B, L, D, N) state is never written to HBM.
 *     - "Selective Scan thay doi inference chuoi dai nhu the nao?": decode
 *       keeps one fixed-size state per layer and updates it per token.
 *   "Selective (Data-Dependent) SSM Scan" (cartesia-pytorch, problem 15)
 *     - "Step-by-Step Approach" 2-6 and the reference solution: elementwise
 *       variant h = A_t*h + B_t*x_t, y_t = C_t*h read after the update
 *       (flag SSM_A_DIRECT).
 *
 * Computed per channel (b, d), for t = 0 .. L-1, per state n < N:
 *   Delta   = softplus(delta[b,t,d] + delta_bias[d])   (softplus if flagged)
 *   h[n]    = exp(Delta * A[d,n]) * h[n] + (Delta * B[b,t,n]) * x[b,t,d]
 *             (SSM_ZOH: (exp(Delta*A[d,n]) - 1) / A[d,n] * B[b,t,n] * x[b,t,d])
 *   y[b,t,d]= (sum_n C[b,t,n] * h[n] + D[d] * x[b,t,d]) * silu(z[b,t,d])
 * with h starting at h0 (or 0) and h_last = h after the last token.  The
 * skip and gate terms are present only when flagged; silu(z) = z*sigmoid(z).
 *
 * Layouts (row-major, contiguous, element strides implied by the shape):
 *   x, delta, z, y : (batch, seqlen, dim)         in_dtype / out_dtype
 *   B, C           : (batch, seqlen, dstate)      in_dtype
 *   A              : (dim, dstate) fp32           (SSM_A_DIRECT: (batch, seqlen, dim) in_dtype)
 *   D, delta_bias  : (dim) fp32
 *   h0, h_last     : (batch, dim, dstate) fp32    (SSM_A_DIRECT: (batch, dim))
 *   state (step)   : (batch, dim, dstate) fp32, read and written in place
 *   step inputs    : x, delta, z, y (batch, dim); B, C (batch, dstate)
 *
 * Ownership: the caller owns every tensor; all data pointers are DEVICE
 * pointers on the plan's device.  The plan owns a small workspace allocated
 * by ssm_scan_create; ssm_scan_fwd / ssm_scan_step allocate nothing and are
 * asynchronous on the caller's stream.  Calls on one plan must not overlap
 * in time (issue them on one stream, or order them): they share the
 * workspace.  y must not alias any input; only `state` is updated in place.
 *
 * Errors: argument checks are synchronous and launch nothing.  A failed
 * launch returns SSM_ERR_CUDA.  Device-side waits (a CTA waiting for the
 * carried state of the earlier part of a row that another CTA ran, and for
 * its own TMA loads) are bounded; if it expires the kernel records SSM_ERR_TIMEOUT, finishes without
 * hanging, and y/h_last of that call are unspecified.  ssm_scan_get_status
 * synchronises the device and returns (and clears) that record.
 *
 * Alignment: the fast path needs 16-byte aligned pointers, dim*sizeof(in)
 * and dstate*sizeof(in) multiples of 16 bytes, and dstate in {8, 16} (bf16)
 * or {4, 8, 16} (fp32).  Any other valid shape runs on a slower general
 * kernel of the same library (never on the CPU).
 */
#ifndef SSM_SCAN_H
#define SSM_SCAN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SSM_API __attribute__((visibility("default")))
#else
#define SSM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *ssm_stream_t; /* same object as cudaStream_t */

typedef enum {
  SSM_OK = 0,
  SSM_ERR_INVALID_ARG = 1, /* null/negative/inconsistent argument or flags */
  SSM_ERR_UNSUPPORTED = 2, /* valid but not supported (e.g. dstate > 64) */
  SSM_ERR_MISALIGNED = 3,  /* reserved: misaligned data takes the general kernel */
  SSM_ERR_CUDA = 4,        /* CUDA runtime error (no device, launch failure) */
  SSM_ERR_TIMEOUT = 5,     /* a bounded device-side wait expired */
  SSM_ERR_OOM = 6          /* workspace allocation failed in ssm_scan_create */
} ssm_status;

typedef enum { SSM_F32 = 0, SSM_BF16 = 1 } ssm_dtype;

enum {
  SSM_HAS_Z = 1,            /* multiply y by silu(z) */
  SSM_HAS_D = 2,            /* add D[d] * x */
  SSM_DELTA_SOFTPLUS = 4,   /* Delta = softplus(delta + bias) (else delta + bias) */
  SSM_HAS_DELTA_BIAS = 8,   /* add delta_bias[d] before softplus */
  SSM_HAS_H0 = 16,          /* start from h0 (else from 0) */
  SSM_WANT_HLAST = 32,      /* write h_last */
  SSM_A_DIRECT = 64,        /* elementwise variant: N = 1, A/B/C per (b,t,d), no delta/D/z */
  SSM_ZOH = 128,            /* zero-order-hold input matrix: Bbar = (exp(Delta*A) - 1) / A * B
                               ("Vi du Python" of the first page) instead of Delta * B;
                               Bbar -> Delta * B where A = 0.  Not with SSM_A_DIRECT. */
  SSM_CONV_X = 256          /* the x branch passes through the causal conv front-end first
                               (ssm_scan_fwd_conv); not with SSM_A_DIRECT or SSM_ZOH */
};

typedef struct {
  int64_t batch, seqlen, dim, dstate;
  ssm_dtype in_dtype;  /* x, delta, z, B, C (and A in SSM_A_DIRECT) */
  ssm_dtype out_dtype; /* y; states are always fp32 */
  uint32_t flags;
} ssm_scan_desc;

typedef struct ssm_scan_plan ssm_scan_plan;

/* Plan details chosen by ssm_scan_create (read-only; for tests and tuning). */
typedef struct {
  int path;            /* 0 = fused chunked kernel, 1 = general kernel, 2 = elementwise */
  int lanes_per_chan;  /* lanes sharing one channel's dstate states */
  int warps_per_cta;
  int tile_t;          /* tokens per pipeline stage (one work unit) */
  int stages;          /* stage slots in the TMA ring (fused kernel) */
  int stages_per_row;  /* ceil(seqlen / tile_t) */
  int chans_per_cta;   /* channels per row tile */
  int grid;            /* CTAs launched (each takes work items by ticket) */
  int64_t rows;        /* independent (batch, channel-tile) rows */
  int64_t units;       /* stages in all = rows * stages_per_row */
  int parts_per_row;   /* work items per segment (a segment's parts hand their state on) */
  int stages_per_part;
  size_t smem_bytes;
  size_t workspace_bytes;
  int chans_per_lane;  /* channels a lane owns (1 or 2) */
  int segments;        /* segments per row scanned at the same time (1 = none) */
  int stages_per_segment;
  int carry_grid;      /* CTAs of the carry pass (segments > 1) */
  int launches_per_call; /* kernels one ssm_scan_fwd launches (2 with segments) */
  int scan_loop;       /* 1 + variant options: bit 0 software-pipelined scan loop,
                          bit 1 registers capped for five CTAs per SM, bit 2 B and C
                          widened to fp32 once per CTA (bf16 inputs), bit 3 a quarter of
                          the state exponentials on the FMA pipe, bit 4 (with bit 0) the
                          pipelined loop prepares two tokens ahead */
  int carry_lanes_per_chan; /* lanes per channel of the carry pass (segments > 1) */
  int carry_loop;      /* 1 + the carry pass's variant options (segments > 1) */
  int bwd_warps_per_cta; /* scan warps of the fused backward kernel (0: ssm_scan_bwd
                            uses the general kernel for this problem) */
  int carry_chans_per_lane; /* channels per lane of the carry pass (segments > 1) */
  int bwd_segments;    /* segments per row tile of the fused backward kernel (1 = none) */
} ssm_scan_info;

/* Optional overrides of the launch shape (0 = keep the default). */
typedef struct {
  int lanes_per_chan; /* 1, 2, 4, 8, 16 (<= dstate) */
  int warps_per_cta;  /* scan warps: 2, 4 or 8 (plus one load warp) */
  int grid;           /* CTAs (any number: work items go out by ticket; capped by the items) */
  int tile_t;         /* tokens per pipeline stage: 32 or 64 */
  int chans_per_lane; /* 1 or 2 */
  int segments;       /* segments per row: 1, 2, 4, 8 or 16 (1 = none) */
  int scan_loop;      /* 1 + variant options (0 = free choice): option bit 0 =
                         software-pipelined scan loop (the next token's exponentials and
                         loads issued before this token's update), bit 1 = registers
                         capped so five CTAs fit on an SM, bit 2 = the load warp widens
                         each stage's B and C to fp32 once for the CTA (bf16 inputs),
                         bit 3 = a quarter of the state exponentials on the FMA pipe,
                         bit 4 = (with bit 0) two tokens prepared ahead instead of one;
                         values above 32 are refused */
  int carry_lanes_per_chan; /* carry pass of a segmented scan: lanes per channel (0 = free) */
  int carry_loop;     /* carry pass: 1 + its variant options, as scan_loop (0 = free) */
  int bwd_warps_per_cta; /* fused backward kernel: 2 or 4 scan warps (0 = free) */
  int carry_chans_per_lane; /* carry pass: 1 or 2 channels per lane (0 = free) */
  int bwd_segments;   /* fused backward kernel: segments per row tile, 1, 2, 4, 8 or 16
                         (0 = free); with more than one, a map pass first computes each
                         segment's forward and adjoint maps */
} ssm_scan_config;
/* Only the combinations compiled into the library exist; ssm_scan_set_config
 * returns SSM_ERR_UNSUPPORTED for others (ssm_scan_list_variants lists them). */

/* Create a plan for one problem shape on `device`; allocates the workspace.
 * Returns SSM_ERR_INVALID_ARG / SSM_ERR_UNSUPPORTED for a bad desc (checked
 * before any CUDA call), SSM_ERR_CUDA if the device is unusable,
 * SSM_ERR_OOM if the workspace cannot be allocated. */
SSM_API ssm_status ssm_scan_create(ssm_scan_plan **plan, const ssm_scan_desc *desc, int device);

/* Free the plan and its workspace (synchronises the device first). */
SSM_API ssm_status ssm_scan_destroy(ssm_scan_plan *plan);

/* Full-sequence forward pass (prefill / training forward), the fused
 * discretise + scan + readout + skip + gate of the pages' "Kernel fusion"
 * section.  Optional pointers (delta_bias, D, z, h0, h_last) must be NULL
 * exactly when their flag is clear.  In SSM_A_DIRECT mode pass A, B, C, x,
 * y (and h0/h_last of shape (batch, dim)); delta, delta_bias, D, z must be
 * NULL. */
SSM_API ssm_status ssm_scan_fwd(ssm_scan_plan *plan, const void *x, const void *delta,
                        const float *delta_bias, const void *A, const void *B,
                        const void *C, const float *D, const void *z,
                        const float *h0, void *y, float *h_last, ssm_stream_t stream);

/* Forward pass with every tensor in HOST memory: x, delta, z, B, C, y, h0,
 * h_last and the parameters A, D, delta_bias (shapes, layouts and flags as
 * for ssm_scan_fwd).  For a caller whose data is not on the device: the
 * library streams the sequence through the GPU in chunks of tokens, with the
 * copy-in of chunk c+1, the scan of chunk c (its state carried on from chunk
 * c-1 on the device) and the copy-out of chunk c-1's y overlapping on three
 * streams, so the host<->device transfers rather than the scan set the time.
 * The host buffers should be page-locked (cudaHostAlloc / cudaHostRegister,
 * torch's pin_memory) for the copies to overlap; pageable memory works but
 * serialises.  Stream-ordered: the work starts behind `stream`'s earlier
 * work and `stream` waits for all of it, so synchronising `stream` (or an
 * event recorded on it after the call) covers the copy-out of y and h_last;
 * the host buffers must stay valid and unmodified until then.  Calls on one
 * plan share its staging memory: issue them on one stream (or synchronise
 * between them).
 * `chunk_tokens` is the number of tokens per chunk (0 = the library's
 * choice: about L/12, at least ~8 MB of copies per chunk, rounded up to a
 * multiple of 64).  The first call (and a
 * call with another chunk length) allocates three chunk slots of device
 * staging memory and the plans for the chunk lengths; later calls reuse
 * them.  SSM_A_DIRECT and SSM_CONV_X plans are refused with
 * SSM_ERR_UNSUPPORTED; SSM_ERR_OOM if the staging memory cannot be had. */
SSM_API ssm_status ssm_scan_fwd_host(ssm_scan_plan *plan, const void *x, const void *delta,
                                     const float *delta_bias, const float *A, const void *B,
                                     const void *C, const float *D, const void *z,
                                     const float *h0, void *y, float *h_last,
                                     int64_t chunk_tokens, ssm_stream_t stream);

/* One decode step (as ssm_scan_step) with the token's inputs x, delta, z, B,
 * C and the output y in HOST memory, while the state and the parameters A,
 * D, delta_bias stay on the device (a server whose tokens arrive on the host
 * and whose state is resident).  The batch is streamed through the device in
 * chunks of `chunk_rows` rows (0 = the library's choice: two chunks, at
 * least ~2 MB of copies each): the copy-in of chunk c+1, the step of chunk
 * c and the copy-out of chunk c-1's y overlap on three streams.  Host buffers
 * should be page-locked for the copies to overlap.  Stream-ordered like
 * ssm_scan_fwd_host (the work starts behind `stream`'s earlier work and
 * `stream` waits for all of it; calls on one plan share its staging, so
 * issue them on one stream).  The first call (and one with another chunk
 * size) allocates three chunk slots of staging memory (SSM_ERR_OOM if it
 * cannot).  SSM_A_DIRECT plans get SSM_ERR_INVALID_ARG, SSM_CONV_X plans
 * SSM_ERR_UNSUPPORTED, as for ssm_scan_step. */
SSM_API ssm_status ssm_scan_step_host(ssm_scan_plan *plan, const void *x, const void *delta,
                                      const float *delta_bias, const float *A, const void *B,
                                      const void *C, const float *D, const void *z,
                                      float *state, void *y, int64_t chunk_rows,
                                      ssm_stream_t stream);

/* Forward pass fed by the causal conv front-end of the x branch, fused into
 * the scan kernel so the conv output never goes through HBM unless asked
 * for.  "Tong quan ..." (vietitpro.vn), section 5.3 "Toi uu hoa Kernel
 * Fusion cho Mamba SSM", names causal_conv1d with selective_scan_fn as the
 * fused pair; the operation is the depthwise causal convolution over L with
 * 4 taps per channel, then silu:
 *   x[b,t,d] = silu(conv_b[d] + sum_{k=0..3} conv_w[d,k] * x_in[b, t-3+k, d])
 * with x_in = 0 before t = 0 (conv_w[d,3] weighs the current token).  That x
 * is the scan's x everywhere (the Delta*x input term and the D skip).  The
 * plan must have SSM_CONV_X.  x_in: (batch, seqlen, dim) in_dtype;
 * conv_w: (dim, 4) fp32; conv_b: (dim) fp32 or NULL (0); x_conv: NULL, or
 * (batch, seqlen, dim) out_dtype to receive x.  The other arguments,
 * ownership and errors are those of ssm_scan_fwd, which refuses SSM_CONV_X
 * plans (SSM_ERR_INVALID_ARG).  ssm_scan_step and ssm_scan_bwd return
 * SSM_ERR_UNSUPPORTED for such plans. */
SSM_API ssm_status ssm_scan_fwd_conv(ssm_scan_plan *plan, const void *x_in, const float *conv_w,
                                     const float *conv_b, const void *delta,
                                     const float *delta_bias, const float *A, const void *B,
                                     const void *C, const float *D, const void *z,
                                     const float *h0, void *y, float *h_last, void *x_conv,
                                     ssm_stream_t stream);

/* Map of the plan's whole sequence, for a scan whose L is split over several
 * devices or calls.  The tokens act on each channel's state as one affine
 * map h -> P h + e per state ("Scan bien recurrence thanh phep toan co the
 * song song hoa ra sao?": per-token maps compose associatively,
 * (A2,b2) (x) (A1,b1) = (A2 A1, A2 b1 + b2)), where P = exp(A * sum_t Delta_t)
 * and e is the state the sequence reaches from h = 0.  Writes
 * map_h (batch, dim, dstate) fp32 = e and map_s (batch, dim) fp32 =
 * sum_t Delta_t.  Inputs as for ssm_scan_fwd (x, delta, delta_bias, A, B;
 * C, D, z are not needed).  The first call on a plan allocates a workspace
 * (about 4*(dstate+1) bytes per channel and sub-chunk) and may return
 * SSM_ERR_OOM.  Plans with SSM_A_DIRECT or SSM_CONV_X: SSM_ERR_UNSUPPORTED. */
SSM_API ssm_status ssm_scan_seq_map(ssm_scan_plan *plan, const void *x, const void *delta,
                                    const float *delta_bias, const float *A, const void *B,
                                    float *map_h, float *map_s, ssm_stream_t stream);

/* Composition of `count` sequence maps, in order, onto a starting state:
 * h = h0 (NULL = 0); for j = 0 .. count-1: h = exp(A * s_j) * h + e_j; writes
 * h_out (batch, dim, dstate) fp32.  maps_h: (count, batch, dim, dstate),
 * maps_s: (count, batch, dim), fp32, as ssm_scan_seq_map writes them (one
 * map per earlier piece of the sequence).  The result is the exact state at
 * the start of the next piece, to pass as h0 to ssm_scan_fwd. */
SSM_API ssm_status ssm_scan_fold_maps(ssm_scan_plan *plan, int count, const float *maps_h,
                                      const float *maps_s, const float *A, const float *h0,
                                      float *h_out, ssm_stream_t stream);

/* Backward pass of ssm_scan_fwd (Delta*B input coefficient; plans with
 * SSM_ZOH or SSM_A_DIRECT get SSM_ERR_UNSUPPORTED): gradients of a loss
 * with dL/dy = dy ((batch, seqlen, dim), out_dtype) and dL/dh_last = dh_last
 * ((batch, dim, dstate) fp32, NULL for 0).  The inputs are the forward
 * call's (same pointers, same flags).  Every gradient is fp32 with its
 * input's shape: dx, ddelta, dz (batch, seqlen, dim); dB, dC
 * (batch, seqlen, dstate); dA (dim, dstate); dD, ddelta_bias (dim); dh0
 * (batch, dim, dstate).  dz, dD, ddelta_bias must be non-NULL exactly when
 * SSM_HAS_Z, SSM_HAS_D, SSM_HAS_DELTA_BIAS are set; dh0 may be NULL.  The
 * accumulated gradients (dB, dC, dA, dD, ddelta_bias) are overwritten, not
 * added to.  States are recomputed from per-stage checkpoints rather than
 * stored ("Tai sao chi parallel scan van chua du nhanh?").  The first call on
 * a plan allocates the workspace — for the fused kernel (dstate 8 or 16,
 * TMA-aligned shapes) the stage-start states (about batch*dim*seqlen*dstate/8
 * floats), per-row-tile dB/dC sums (about batch*seqlen*2*dstate floats per 32
 * channels) and, for a segmented plan, the segments' maps; for the general
 * kernel batch*dim*ceil(seqlen/16)*dstate floats — and may return
 * SSM_ERR_OOM; later calls reuse it.  dB and dC are added in a fixed order
 * (reproducible bit for bit) on the fused path; dA, dD and ddelta_bias (and
 * dB, dC on the general path) follow atomics, reproducible to rounding only.
 * ssm_scan_set_config's bwd_warps_per_cta and bwd_segments choose the fused
 * kernel's shape; ssm_scan_get_info reports it. */
SSM_API ssm_status ssm_scan_bwd(ssm_scan_plan *plan, const void *x, const void *delta,
                        const float *delta_bias, const float *A, const void *B,
                        const void *C, const float *D, const void *z, const float *h0,
                        const void *dy, const float *dh_last, float *dx, float *ddelta,
                        float *ddelta_bias, float *dA, float *dB, float *dC, float *dD,
                        float *dz, float *dh0, ssm_stream_t stream);

/* One decode step per the pages' inference section: reads `state`
 * (batch, dim, dstate), applies one token, writes it back and writes y
 * (batch, dim).  desc.seqlen is ignored; SSM_HAS_H0 / SSM_WANT_HLAST /
 * SSM_A_DIRECT are not used. */
SSM_API ssm_status ssm_scan_step(ssm_scan_plan *plan, const void *x, const void *delta,
                         const float *delta_bias, const float *A, const void *B,
                         const void *C, const float *D, const void *z, float *state,
                         void *y, ssm_stream_t stream);

/* Allocation-free forward pass.  The pages have no counterpart: this entry
 * exists for callers that cannot allocate device memory (no cudaMalloc):
 * code running under an allocator that owns all device memory up front,
 * plugins that must not bypass their host's allocator, paths that must not
 * risk the device synchronisation an allocation can cause.  Same operation,
 * layouts and flags as ssm_scan_fwd (SSM_A_DIRECT excluded), on the CALLER'S
 * CURRENT DEVICE, without a plan: the kernel's scratch (carried states,
 * per-chunk flags, work counter) lives in a fixed 4 MiB device array inside
 * the library, which every device that loads the library holds until the
 * process exits.  Limits: the fast-path shape rules above (otherwise
 * SSM_ERR_UNSUPPORTED; misaligned pointers give SSM_ERR_MISALIGNED), and
 * about 4*dstate bytes of scratch per channel of batch*dim (rounded up to the
 * kernel's channel tile): a problem whose scratch exceeds 4 MiB is rejected
 * with SSM_ERR_UNSUPPORTED before anything is launched.  All calls share the
 * scratch, so calls that overlap on the GPU (other streams or threads) race
 * and give wrong results.  The first call on a device looks the scratch
 * address up (cudaGetSymbolAddress); a new CUDA context on the device (e.g.
 * after cudaDeviceReset) makes the next call look it up again.  A device-side wait that runs out
 * is recorded in the scratch (outputs of that call are then unspecified) and
 * reported by ssm_scan_noalloc_status.  Nothing is allocated; inputs and
 * outputs are the caller's device buffers. */
SSM_API ssm_status ssm_scan_fwd_noalloc(const ssm_scan_desc *desc, const void *x,
                                        const void *delta, const float *delta_bias,
                                        const float *A, const void *B, const void *C,
                                        const float *D, const void *z, const float *h0,
                                        void *y, float *h_last, ssm_stream_t stream);

/* Status of the allocation-free entry point on the caller's current device
 * (no counterpart on the pages; it belongs to ssm_scan_fwd_noalloc):
 * synchronises the device, returns the device-side status recorded by the
 * calls since the last query (SSM_OK or SSM_ERR_TIMEOUT) and resets it.
 * Allocates nothing. */
SSM_API ssm_status ssm_scan_noalloc_status(void);

/* Test hook of the allocation-free entry point, process-wide: the bound of
 * its device-side waits (nanoseconds, 0 = default of 2 s) and the work unit
 * whose hand-over of its carried state is skipped (-1 = none), as
 * ssm_scan_set_debug does for a plan. */
SSM_API ssm_status ssm_scan_noalloc_set_debug(uint64_t wait_timeout_ns, int64_t drop_unit);

/* Synchronise the plan's device, return the device-side status recorded by
 * the last calls (SSM_OK or SSM_ERR_TIMEOUT) and reset it to SSM_OK. */
SSM_API ssm_status ssm_scan_get_status(ssm_scan_plan *plan);

/* Fill *info with the plan's launch shape. */
SSM_API ssm_status ssm_scan_get_info(const ssm_scan_plan *plan, ssm_scan_info *info);

/* Override the launch shape (tuning); takes effect on the next call.  May
 * reallocate the workspace, so call it between calls, not during one. */
SSM_API ssm_status ssm_scan_set_config(ssm_scan_plan *plan, const ssm_scan_config *cfg);

/* Test hook: set the bound of device-side waits (nanoseconds, 0 = default
 * of 2 s) and make the run of work units that ends at unit `drop_unit`
 * (-1 = none) skip handing on its carried state, so the CTA that continues
 * that row waits until the bound expires.  Used to test the timeout path
 * without hanging the device. */
SSM_API ssm_status ssm_scan_set_debug(ssm_scan_plan *plan, uint64_t wait_timeout_ns, int64_t drop_unit);

/* Throughput probe for the roofline denominators (a measurement helper; the
 * pages have no counterpart): launches `blocks` CTAs of 256 threads on
 * `stream`, each thread running independent chains of kind 0 = ex2.approx
 * (the special-function unit that computes the exponential of every state
 * update) or kind 1 = fp32 FMA, `iters` x 64 operations per thread.  *ops
 * receives the number of operations launched (results per thread x threads);
 * the caller times the launch (e.g. with CUDA events) and divides.  `sink` is
 * a device buffer of at least `blocks` floats that the probe may write.
 * Returns SSM_ERR_INVALID_ARG for a bad argument, SSM_ERR_CUDA if the launch
 * fails. */
SSM_API ssm_status ssm_probe_peak(int kind, int64_t iters, int blocks, float *sink,
                                  int64_t *ops, ssm_stream_t stream);

/* The kernels' two implementations of 2^x on n device floats x (a check of
 * the FMA-pipe one, no counterpart in the pages): y_fma receives the
 * range-reduced polynomial that kernel option bit 3 uses for a quarter of the
 * state exponentials, y_sfu the special-function unit's ex2.approx.  All three
 * are device pointers of n floats; enqueued on `stream`.  Returns
 * SSM_ERR_INVALID_ARG for a negative n or a null pointer with n > 0. */
SSM_API ssm_status ssm_probe_exp2(const float *x, float *y_fma, float *y_sfu, int64_t n,
                                  ssm_stream_t stream);

/* One compiled variant of the fused kernel. */
typedef struct {
  int dstate, lanes_per_chan, chans_per_lane, warps_per_cta, tile_t;
  int zoh;   /* zero-order-hold input coefficient */
  int carry; /* the carry pass of a segmented launch (not a full scan) */
  int conv;  /* with the causal conv front-end of the x branch */
  int opt;   /* options: bit 0 software-pipelined scan loop, bit 1 five CTAs per SM */
} ssm_scan_variant;

/* The compiled variants of the fused kernel for a dtype pair (a tuning and
 * test aid; the pages have no counterpart): fills up to `max` entries of
 * `out` (which may be NULL) and returns how many exist. */
SSM_API int ssm_scan_list_variants(ssm_dtype in_dtype, ssm_dtype out_dtype,
                                   ssm_scan_variant *out, int max);

/* Static description of a status code. */
SSM_API const char *ssm_status_string(ssm_status s);

/* Library version as 10000*major + 100*minor + patch. */
SSM_API int ssm_scan_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SSM_SCAN_H */
