/*
 * ss_scan.h -- C ABI of libssscan.so: the Mamba-1 selective scan (S6) forward pass
 * and its single-token decode state update on NVIDIA B200 (sm_100a).
 *
 * What is computed (nnterp documentation, "selective_scan" component: the
 * SelectiveScan class description and the two kernel calls it names,
 * mamba_selective_scan on a prompt and mamba_selective_state_update on a decode
 * step; TransformerLens "ssm_mixer" module, compute_ssm_state):
 *
 *   dt_t   = softplus(dt_raw[b,c,t] + dt_bias[c])     (flag SS_DT_SOFTPLUS; else the sum)
 *   h_t[n] = exp(dt_t * A[c,n]) * h_{t-1}[n] + dt_t * B[b,n,t] * x[b,c,t]
 *   y_t    = sum_n C[b,n,t] * h_t[n] + D[c] * x[b,c,t]
 *   out_t  = y_t * silu(z[b,c,t])                       (only when z is not NULL)
 *
 * Enforced boundary reset ("s6_reset" blog draft, Enforced Boundary Resetting):
 * where reset[b,t] != 0 the state is zeroed before token t's update, so
 * h_t = dt_t * B[b,:,t] * x[b,c,t] there; the mask is shared by all channels.
 *
 * Conventions shared by every entry point:
 *  - All tensor pointers are DEVICE pointers to contiguous, row-major arrays in the
 *    channel-first layouts below.  The caller owns all memory; the library never
 *    allocates, frees or keeps a pointer after the call returns.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *    stream).  They return after the launch is enqueued, without synchronising.
 *  - Host-side validation runs first; on any error nothing is launched and the
 *    status below is returned.  A launch failure reported by the CUDA runtime
 *    returns SS_ERR_CUDA.
 *  - Inputs are never modified.  Outputs must not overlap any input, except that
 *    h_last may be the very same buffer as h0 (chaining in place).
 *  - A, D, dt_bias, h0, h_last and the decode state are float32.  x, dt, z, B, C and
 *    y share the element type `dtype` (float32 or bfloat16); y is rounded to it
 *    round-to-nearest-even.  State and accumulation are float32.
 *  - Pointers must be aligned to their element size (SS_ERR_ALIGN otherwise);
 *    16-byte alignment and seq a multiple of 8 enable the vectorised path, any
 *    other size or alignment takes a predicated scalar path.
 */
#ifndef SS_SCAN_H
#define SS_SCAN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SS_API __attribute__((visibility("default")))
#else
#define SS_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st *ss_stream_t;

/* Element type of x, dt, z, B, C and y. */
typedef enum { SS_F32 = 0, SS_BF16 = 1 } ss_dtype_t;

/* Status codes. */
enum {
    SS_OK = 0,
    SS_ERR_NULL = 1,        /* a required pointer is NULL                          */
    SS_ERR_SHAPE = 2,       /* a size is <= 0 or too large for the launch grid     */
    SS_ERR_DTYPE = 3,       /* dtype is not SS_F32 or SS_BF16                       */
    SS_ERR_ALIGN = 4,       /* a pointer is not aligned to its element size        */
    SS_ERR_UNSUPPORTED = 5, /* state_dim not in {4, 8, 16}, or an unknown flag bit */
    SS_ERR_CUDA = 6,        /* the CUDA runtime reported an error                  */
    SS_ERR_TIMEOUT = 7,     /* a bounded device-side wait gave up                  */
    SS_ERR_ALIAS = 8,       /* an output (or the workspace) overlaps an input      */
    SS_ERR_WORKSPACE = 9,   /* workspace smaller than ss_scan_workspace_bytes()    */
    SS_ERR_SCRATCH_LIMIT = 10 /* the shape needs more than SS_STATIC_SCRATCH_BYTES   */
};

/* flags bit 0: apply softplus to dt_raw + dt_bias (mamba's delta_softplus). */
enum { SS_DT_SOFTPLUS = 1u };

/*
 * Prompt scan: the recurrence above over all `seq` tokens of every (b, c) row.
 *
 *   x, dt_raw, z : [batch, channels, seq]  dtype      (z nullable: no gate)
 *   A            : [channels, state_dim]   float32    (negative rates)
 *   B, C         : [batch, state_dim, seq] dtype      (shared by every channel)
 *   D, dt_bias   : [channels]              float32    (nullable: 0)
 *   reset        : [batch, seq]            uint8      (nullable: no resets)
 *   h0           : [batch, channels, state_dim] float32 (nullable: zeros)
 *   y            : [batch, channels, seq]  dtype      (output)
 *   h_last       : [batch, channels, state_dim] float32 (nullable output: the state
 *                  after the last token, what the next decode step starts from)
 *   workspace    : nullable device buffer of at least ss_scan_workspace_bytes()
 *                  bytes, 16-byte aligned, zero-filled by the caller before its FIRST
 *                  use (cudaMemset); every call that completes leaves it ready for the
 *                  next one.  With a workspace the sequence is split into segments
 *                  processed by persistent CTAs that pass the scan carry between
 *                  them, which balances the GPU for any shape.  Without one, each CTA
 *                  scans one group of channels over the whole sequence.  Calls that
 *                  share a workspace must be ordered (same stream, or synchronised).
 *                  For state_dim 16 with few channel groups and a long sequence (the
 *                  single-pass schedule would leave most of the GPU idle), the size
 *                  includes room for a two-level schedule ("s6_reset" blog draft,
 *                  Associative Boundary Resetting): every segment of the sequence is
 *                  scanned at once from zero for its end state, the segments'
 *                  (decay, end state) composites are joined into each one's entering
 *                  state, and every segment is scanned again from it.  It runs when
 *                  the workspace has that size; it does the exponentials twice, in
 *                  exchange for filling the GPU.
 *                  A call whose device-side waits gave up (SS_ERR_TIMEOUT, see
 *                  ss_scan_status) also leaves the workspace ready for the next call:
 *                  its outputs are invalid, but the workspace needs no re-zeroing.
 *
 * state_dim must be 4, 8 or 16.  Returns SS_OK or an error status.
 */
SS_API int ss_scan_fwd(int64_t batch, int64_t channels, int64_t state_dim, int64_t seq,
                       ss_dtype_t dtype, const void *x, const void *dt_raw, const float *A,
                       const void *B, const void *C, const float *D, const void *z,
                       const float *dt_bias, const uint8_t *reset, const float *h0,
                       uint32_t flags, void *y, float *h_last, void *workspace,
                       size_t workspace_bytes, ss_stream_t stream);

/*
 * ss_scan_fwd that also returns, per token, what the interpretability readers ask for
 * (nnterp selective_scan: the state after each token, the step size per token and
 * channel, and the log decay dt * A; TransformerLens ssm_mixer: the unrolled state S_t
 * at every position):
 *
 *   h_all : [batch, channels, seq, state_dim] float32 output (nullable);
 *           h_all[b,c,t,:] = h_t of row (b, c), resets and h0 included.
 *   betas : [batch, channels, seq] float32 output (nullable): the step size of every
 *           token, dt[b,c,t] = softplus(dt_raw[b,c,t] + dt_bias[c]) (without the
 *           softplus when SS_DT_SOFTPLUS is clear), the value the scan itself uses.
 *           The per-token log decay of state n is betas[b,c,t] * A[c,n].
 * At least one of the two must be given (SS_ERR_NULL otherwise).
 *
 * Everything else is as for ss_scan_fwd (same outputs, bit-identical y and h_last).
 * h_all and betas must not overlap any other buffer or each other (SS_ERR_ALIAS).  The
 * extra traffic is 4 * state_dim bytes per (b, t, c) for h_all and 4 for betas, each
 * written once, so with h_all this form is bound by HBM bandwidth rather than by the
 * exponentials.
 */
SS_API int ss_scan_fwd_states(int64_t batch, int64_t channels, int64_t state_dim, int64_t seq,
                              ss_dtype_t dtype, const void *x, const void *dt_raw, const float *A,
                              const void *B, const void *C, const float *D, const void *z,
                              const float *dt_bias, const uint8_t *reset, const float *h0,
                              uint32_t flags, void *y, float *h_last, float *h_all, float *betas,
                              void *workspace, size_t workspace_bytes, ss_stream_t stream);

/*
 * ss_scan_fwd with the causal depthwise convolution and SiLU that produce its input
 * fused in front (TransformerLens ssm_mixer: the scan's x is SiLU of the conv1d
 * output; a decode step carries the conv's recent inputs as its state):
 *
 *   x[b,c,t] = silu( conv_b[c] + sum_{k<conv_k} conv_w[c,k] * u[b,c,t-conv_k+1+k] )
 *
 * with u before t = 0 read from conv_state, and then the scan of ss_scan_fwd on x.
 *
 *   u              : [batch, channels, seq] dtype (the conv input; takes x's place)
 *   conv_w         : [channels, conv_k] float32, conv_k in 1..4
 *   conv_b         : [channels] float32 (nullable: 0)
 *   conv_state     : [batch, channels, conv_k-1] float32 (nullable: zeros), the inputs
 *                    that preceded u, oldest first
 *   conv_state_out : [batch, channels, conv_k-1] float32 (nullable output), the last
 *                    conv_k-1 inputs of conv_state ++ u, for the next call
 *   x_out          : [batch, channels, seq] dtype (nullable output), x itself
 *
 * The other arguments are those of ss_scan_fwd.  SiLU of x is evaluated like the
 * output gate (exact for float32 storage; the MUFU tanh form for bfloat16, within the
 * bfloat16 tolerance).  No output may overlap an input or another output
 * (SS_ERR_ALIAS).
 */
SS_API int ss_scan_fwd_conv(int64_t batch, int64_t channels, int64_t state_dim, int64_t seq,
                            ss_dtype_t dtype, const void *u, const float *conv_w,
                            const float *conv_b, int64_t conv_k, const float *conv_state,
                            float *conv_state_out, void *x_out, const void *dt_raw,
                            const float *A, const void *B, const void *C, const float *D,
                            const void *z, const float *dt_bias, const uint8_t *reset,
                            const float *h0, uint32_t flags, void *y, float *h_last,
                            void *workspace, size_t workspace_bytes, ss_stream_t stream);

/*
 * Launch plan of ss_scan_fwd for a shape, on the current device: what the call would
 * launch for 16-byte aligned tensors (the tile-load path) with or without resets and
 * a workspace.  For tuning and for reporting alongside measurements; launches nothing.
 */
typedef struct {
    int64_t grid;        /* CTAs launched                                        */
    int64_t ctas_per_sm; /* resident CTAs per SM of that kernel (occupancy)      */
    int64_t sms;         /* SMs of the current device                            */
    int64_t groups;      /* channel groups: batch * ceil(channels / per CTA)     */
    int64_t segments;    /* sequence segments per group (1 without a workspace)  */
    int64_t seg_len;     /* tokens per segment                                   */
    int64_t states_per_lane; /* state rows each scan lane owns (2 or 4)          */
    int64_t two_level;   /* 1: the two-level schedule (see ss_scan_fwd), 0: single pass */
} ss_scan_plan_t;
SS_API int ss_scan_plan(int64_t batch, int64_t channels, int64_t state_dim, int64_t seq,
                        ss_dtype_t dtype, int has_reset, int with_workspace,
                        ss_scan_plan_t *plan);

/* Workspace bytes ss_scan_fwd needs for this shape (0 for an invalid shape). */
SS_API int64_t ss_scan_workspace_bytes(int64_t batch, int64_t channels, int64_t state_dim,
                                       int64_t seq);

/*
 * Device-side status of earlier scans: synchronises `stream`, then reads and clears
 * the status word of `workspace` (or, for NULL, the word shared by calls made without
 * a workspace on the current device).  *status becomes SS_OK, or SS_ERR_TIMEOUT if a
 * bounded wait inside a kernel gave up (its outputs are then invalid).  Returns
 * SS_OK, or an error status if the query itself failed.
 */
SS_API int ss_scan_status(const void *workspace, ss_stream_t stream, int *status);

/*
 * The device status word of calls made without a workspace (ss_scan_fwd with a NULL
 * workspace, and every decode call) on the current device: ss_scan_status(NULL,
 * stream, ...) as one return value.  Synchronises `stream`, reads and clears the word,
 * and returns SS_OK, SS_ERR_TIMEOUT (a bounded device-side wait gave up; those calls'
 * outputs are invalid) or the error status of the query itself.
 */
SS_API int ss_debug_status(ss_stream_t stream);

/*
 * ss_scan_fwd without a caller-supplied workspace and without any allocation.
 *
 * The selective-scan method itself has no counterpart to this call: it is a
 * convenience of this library for callers that cannot allocate or own device memory
 * at the moment they scan -- a serving loop whose memory plan is fixed at start-up,
 * or a host program that only receives device pointers from another framework and
 * has no allocator of its own.  It runs the same segmented, balanced schedule as
 * ss_scan_fwd with a workspace, using instead a fixed scratch of
 * SS_STATIC_SCRATCH_BYTES (1 MiB) that the library holds in a static device array,
 * one per device.  Neither this call nor anything it calls allocates memory.
 *
 * Arguments, layouts and results are those of ss_scan_fwd, except:
 *   flags   : SS_DT_SOFTPLUS as for ss_scan_fwd, plus SS_SCRATCH_ZERO to clear the
 *             scratch (an asynchronous memset on `stream`) before this scan.
 *   scratch : nullable; receives the device address of this device's scratch, which
 *             ss_scan_status(scratch, stream, &st) takes to read the device-side
 *             status of these calls.
 *
 * Limit: the shape must need at most SS_STATIC_SCRATCH_BYTES of workspace
 * (ss_scan_workspace_bytes); larger shapes are refused with SS_ERR_SCRATCH_LIMIT
 * before anything is launched.  At state_dim 16 that is up to 992 channel groups of
 * 16, i.e. batch * ceil(channels / 16) <= 992 (batch 1 at 5120 channels, or batch 8
 * at 1536, fit).
 *
 * Zero state: the scratch is zero when the library is loaded, and every scan leaves
 * it ready for the next one, a scan whose waits gave up (SS_ERR_TIMEOUT) included.
 * SS_SCRATCH_ZERO clears all SS_STATIC_SCRATCH_BYTES of it, for a caller that wants
 * a known starting point (after a fault elsewhere in the process, say).
 *
 * Set-up: the first call on each device, with that device current, looks up the
 * scratch's address (which may load the library's device code) and configures the
 * kernel; make that first call before any stream capture begins.
 *
 * Concurrency: all calls on one device share the one scratch.  Two calls whose
 * executions overlap (different streams, not ordered by events) race on it and give
 * wrong results; order them, or use ss_scan_fwd with a workspace per stream.
 */
#define SS_STATIC_SCRATCH_BYTES (1u << 20)
enum { SS_SCRATCH_ZERO = 2u };
SS_API int ss_scan_fwd_static_scratch(int64_t batch, int64_t channels, int64_t state_dim,
                                      int64_t seq, ss_dtype_t dtype, const void *x,
                                      const void *dt_raw, const float *A, const void *B,
                                      const void *C, const float *D, const void *z,
                                      const float *dt_bias, const uint8_t *reset,
                                      const float *h0, uint32_t flags, void *y, float *h_last,
                                      const void **scratch, ss_stream_t stream);

/*
 * Decode step: one token of the same recurrence for every (b, c), updating `state`
 * in place (nnterp selective_scan: the updated state is what the cache receives).
 *
 *   state        : [batch, channels, state_dim] float32 (in/out)
 *   x, dt_raw, z : [batch, channels]        dtype        (z nullable)
 *   A            : [channels, state_dim]    float32
 *   B, C         : [batch, state_dim]       dtype
 *   D, dt_bias   : [channels]               float32      (nullable)
 *   y            : [batch, channels]        dtype        (output)
 *
 * No reset on this path.  Returns SS_OK or an error status.
 */
SS_API int ss_state_update(int64_t batch, int64_t channels, int64_t state_dim, ss_dtype_t dtype,
                    float *state, const void *x, const void *dt_raw, const float *A,
                    const void *B, const void *C, const float *D, const void *z,
                    const float *dt_bias, uint32_t flags, void *y, ss_stream_t stream);

/*
 * Decode step of the fused conv form: the new token's scan input x comes from the
 * causal conv over the row's conv state and the new input u, and the conv state
 * advances by one input (TransformerLens ssm_mixer: SiLU of the conv1d output; a decode
 * step carries the conv's recent inputs as its state):
 *
 *   x[b,c]          = silu( conv_b[c] + sum_{k<conv_k-1} conv_w[c,k] * conv_state[b,c,k]
 *                           + conv_w[c,conv_k-1] * u[b,c] )
 *   conv_state[b,c] = (conv_state[b,c,1:], u[b,c])          (in place)
 *
 * then the update of ss_state_update with x.  conv_state: [batch, channels, conv_k-1]
 * float32, required when conv_k > 1, overlapping no other buffer; conv_w [channels,
 * conv_k], conv_b [channels] (nullable) float32; conv_k in 1..4.  The state must be
 * 16-byte aligned (SS_ERR_ALIGN otherwise).  SiLU of x is the exact form here.
 */
SS_API int ss_state_update_conv(int64_t batch, int64_t channels, int64_t state_dim,
                                ss_dtype_t dtype, float *state, float *conv_state,
                                const float *conv_w, const float *conv_b, int64_t conv_k,
                                const void *u, const void *dt_raw, const float *A, const void *B,
                                const void *C, const float *D, const void *z,
                                const float *dt_bias, uint32_t flags, void *y, ss_stream_t stream);

/*
 * Testing aid: cap every device-side wait of later calls on the current device at
 * `microseconds` (0 restores the default of 2 s).  Used to make a wait that can never
 * be satisfied end quickly with SS_ERR_TIMEOUT; waits for copies already in flight
 * keep the default limit.  Synchronous; returns SS_OK or SS_ERR_CUDA.
 */
SS_API int ss_debug_set_wait_limit(uint32_t microseconds);

/*
 * Testing aid: make later state_dim-16 scans in this process use the layout with
 * `states_per_lane` (2 or 4) state rows per scan lane, whatever the shape; 0 restores
 * the default (two per lane, the faster layout as measured).  Results of the two
 * layouts agree within rounding; they differ only in speed.  Other state sizes always
 * use two.  Returns SS_OK, or
 * SS_ERR_UNSUPPORTED for any other value.  Not thread-safe with respect to scans
 * being issued concurrently from other host threads.
 */
SS_API int ss_debug_set_scan_layout(int states_per_lane);

/*
 * Testing aid: the schedule of later state_dim-16 scans with a workspace.  mode 0
 * (default): the two-level schedule where the shape calls for it; 1: never (always
 * the single-pass schedule); 2: whenever the sequence has at least two segments of
 * sixteen 32-token chunks.  ss_scan_workspace_bytes follows the same setting.  Returns
 * SS_OK, or SS_ERR_UNSUPPORTED for any other mode.  Not thread-safe with respect to
 * scans issued concurrently from other host threads.
 */
SS_API int ss_debug_set_scan_two_level(int mode);

/*
 * Testing aid: the kernel of later ss_gated_scan calls.  mode 0 (default): the
 * chunked tensor-core form where it applies (see ss_gated_scan), 1: always the
 * token-by-token recurrence, 2: as 0, 3: as 0, and in the tensor-core form the compute
 * warps withhold their first "L o S written" arrival, so the issuing warp's wait for it
 * can never be satisfied: the call ends on the wait time limit (shorten it with
 * ss_debug_set_wait_limit) with SS_ERR_TIMEOUT in the status word and no output
 * written (a failure-path test aid: nothing faults, every wait is bounded).  Returns
 * SS_OK, or SS_ERR_UNSUPPORTED for any other mode.
 */
SS_API int ss_debug_set_gated_path(int mode);

/*
 * Gated state scan (the "Mamba 2 Gated State Scan" exercise page): per batch item b,
 *
 *   S_t = gamma[b,t] * S_{t-1} + k[b,t,:] v[b,t,:]^T      (Dk x Dv state, fp32)
 *   outputs[b,t,:] = q[b,t,:]^T S_t                        (the updated state is read)
 *
 * with S_{-1} = h0[b] (zeros when h0 is NULL) and final_state[b] = S_{seq-1}.
 *
 *   q, k        : [batch, seq, dk]  dtype (SS_F32 or SS_BF16)
 *   v           : [batch, seq, dv]  dtype
 *   gamma       : [batch, seq]      float32, any real value (the page's gates are in [0, 1])
 *   h0          : [batch, dk, dv]   float32, nullable
 *   outputs     : [batch, seq, dv]  dtype (output)
 *   final_state : [batch, dk, dv]   dtype (output)
 *
 * Results are rounded to the dtype of q, as the page asks.  dk must be at most 128
 * (SS_ERR_UNSUPPORTED otherwise); dv is unrestricted.  Two kernels:
 *  - bf16 with dk = 128, dv a multiple of 64 and 16-byte aligned tensors: the chunked
 *    form on the tensor cores -- per 128-token chunk, Q K^T, the decay-masked scores
 *    times V, Q times the entering state, and K^T times the decay-weighted V as
 *    tcgen05 matrix products (bf16 operands, fp32 accumulation), the state itself in
 *    fp32;
 *  - every other case: the recurrence token by token, all arithmetic in fp32.
 * Inputs are not modified; outputs must not overlap inputs or each other
 * (SS_ERR_ALIAS).  Asynchronous on `stream`; returns SS_OK or an error status.
 */
SS_API int ss_gated_scan(int64_t batch, int64_t seq, int64_t dk, int64_t dv, ss_dtype_t dtype,
                         const void *q, const void *k, const void *v, const float *gamma,
                         const float *h0, void *outputs, void *final_state, ss_stream_t stream);

/*
 * Sequence cut into segments (one per GPU, say) -- the two joining steps.
 *
 * The scan's recurrence composes associatively ("s6_reset" blog draft, Associative
 * Boundary Resetting: that is what lets a long sequence be scanned in parallel).  A
 * segment acts on the state that enters it as the map h -> decay * h + state, with
 *
 *   decay[b,c,n] = prod over the segment of exp(dt_t * A[c,n])
 *                = exp(A[c,n] * sum_t dt_t), and exactly 0 when reset[b,t] != 0 for
 *                  some t of the segment (the entering state is then discarded);
 *   state[b,c,n] = the segment's end state when it is entered from zero, i.e. the
 *                  h_last of ss_scan_fwd on the segment with h0 = NULL.
 *
 * Joining: segment 0 is scanned from the real h0 and is final.  Every other segment
 * s is scanned once from zero to get its composite; the composites of all segments
 * are gathered (in segment order) on every GPU; ss_join_segments folds those before
 * s into the state entering s; and ss_scan_fwd on segment s with that state as h0
 * gives its final outputs.
 *
 * ss_segment_decay -- the decay of one segment.
 *   dt_raw      : [batch, channels, seq] dtype
 *   A           : [channels, state_dim] float32
 *   dt_bias     : [channels] float32, nullable
 *   reset       : [batch, seq] uint8, nullable (the segment's slice of the mask)
 *   flags       : SS_DT_SOFTPLUS as for ss_scan_fwd (other bits: SS_ERR_UNSUPPORTED)
 *   decay       : [batch, channels, state_dim] float32 (output)
 * The step sizes are summed in float32; decay uses the same flush-to-zero exp2 as
 * the scan.  state_dim must be 4, 8 or 16.  decay must not overlap an input
 * (SS_ERR_ALIAS).  Asynchronous on `stream`; reads dt_raw once.
 */
SS_API int ss_segment_decay(int64_t batch, int64_t channels, int64_t state_dim, int64_t seq, ss_dtype_t dtype,
                            const void *dt_raw, const float *A, const float *dt_bias, const uint8_t *reset,
                            uint32_t flags, float *decay, ss_stream_t stream);

/*
 * ss_join_segments -- fold gathered composites in segment order.
 *   composites  : [segments][2][count] float32: for segment s, decay at
 *                 composites[(2s) * count ...] and end state at
 *                 composites[(2s + 1) * count ...] (count = batch*channels*state_dim).
 *                 Segment 0's entry holds its end state from the real h0; its decay
 *                 is never read.
 *   rank        : the segment whose entering state `carry` receives; 1 <= rank <
 *                 segments when carry is not NULL (SS_ERR_SHAPE otherwise).
 *   carry       : [count] float32, nullable: the state entering segment `rank`.
 *   final_state : [count] float32, nullable: the state after the last segment.
 * At least one of carry, final_state must be given (SS_ERR_NULL).  Outputs must not
 * overlap composites or each other (SS_ERR_ALIAS).  float32 arithmetic, one fused
 * multiply-add per segment and element.  Asynchronous on `stream`.
 */
SS_API int ss_join_segments(int64_t segments, int64_t count, const float *composites, int64_t rank,
                            float *carry, float *final_state, ss_stream_t stream);

/*
 * Measurement aid: the throughput of the special-function unit that bounds the prompt
 * scan (its exponentials).  Launches `blocks` CTAs of 512 threads (one per SM when
 * blocks is the SM count) that each run 8 independent chains of `iters` operations:
 * op 0 = ex2.approx.ftz.f32 (the decays), op 1 = tanh.approx.f32 (the bf16 output
 * gate).  cycles (device, [blocks] int64) receives each CTA's SM clock cycles for its
 * loop; sink (device, [512] float) is written only to keep the work live; the host
 * gets *ops_per_block, so ops / cycles is the unit's results per clock per SM.
 * Asynchronous on `stream`; returns SS_OK or an error status.
 */
SS_API int ss_debug_mufu_probe(int op, int64_t iters, int64_t blocks, long long *cycles, float *sink,
                               int64_t *ops_per_block, ss_stream_t stream);

/*
 * Debug build with index checks (libssscan_bounds.so, compiled with SS_BOUNDS_CHECK):
 * every runtime-computed global and shared-memory index of the scan and decode kernels
 * is checked before its access; a failed check skips the access and records the
 * number of its site (the first one wins) in a device word, without a trap.  This call
 * synchronises `stream`, stores that site in *site (0: no failed check) and clears it.
 * In the normal build it stores -1 and returns SS_ERR_UNSUPPORTED.
 */
SS_API int ss_debug_bounds_status(ss_stream_t stream, int *site);

/* Human-readable name of a status code (static string, never NULL). */
SS_API const char *ss_status_string(int status);

/* ABI version of this library: (major << 16) | minor. */
SS_API int ss_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SS_SCAN_H */
