/*
 * ssm_scan.h -- C ABI of the B200 selective-scan (S6) library, libssmscan.so.
 *
 * The operation (all entry points below compute parts of it):
 *
 *   Delta_t = softplus(delta_t + delta_bias)        (or delta_t + delta_bias)
 *   Abar_t  = exp(Delta_t * A)                     diagonal A, per channel
 *   h_t     = Abar_t (.) h_{t-1} + Delta_t * B_t * u_t
 *   y_t     = (C_t . h_t + D * u_t) * SiLU(z_t)
 *
 * Sources: "Mamba: Linear-Time Sequence Modeling with Selective State Spaces"
 * (xyznot.com reading guide), section "Metodo" (zero-order hold,
 * Abar = exp(Delta A), recurrence h_t = Abar h_{t-1} + Bbar x_t) and section
 * "O Mecanismo de Selecao (S6)" (B_t, C_t input dependent, Delta_t =
 * softplus(Parameter + s_Delta(x_t))); "O que e um modelo Mamba?" (ibm.com),
 * output equation y = C h + D x and the Mamba block walk-through (the SSM
 * output is multiplied by the activated z branch); "Как работает Mamba
 * (State Space Model)..." (aivaro.ru), section 3, the selective_scan(u,
 * delta, A, B, C, D) example, whose Euler input term B_bar = delta * B this
 * library uses.  The expanded (batch, seqlen, dim, dstate) state is never
 * written to memory (reading guide, "Expansao de Estado Ciente de Hardware").
 *
 * Layouts (row-major, last index contiguous; "dim" is d_inner, "dstate" N):
 *   u, delta, z, y, dout, du, ddelta, dz   [batch][dim][seqlen]   io dtype
 *   B, C, dB, dC                           [batch][seqlen][dstate] io dtype
 *   A, dA                                  [dim][dstate]          fp32
 *   D, delta_bias, dD, ddelta_bias         [dim]                  fp32
 *   initial_state, last_state, dinitial_state [batch][dim][dstate] fp32
 * io dtype is fp32 or bf16 (ssm_shape.io_dtype).  State and all arithmetic
 * are fp32.  bf16 results are rounded to nearest-even.
 *
 * Ownership and threading: the caller owns every buffer, device pointers
 * throughout.  The library allocates no memory; scratch comes from the
 * caller's workspace (sizes from the *_workspace_bytes queries).  Every call
 * only enqueues work on `stream` and returns; nothing synchronises except
 * ssm_scan_check().  Calls are thread-safe; two calls that share a workspace
 * must be ordered on the GPU (same stream, or events).
 *
 * Errors: argument checks happen before any launch and return a status with
 * nothing enqueued.  Launch failures return SSM_ERR_CUDA.  Kernels never trap:
 * a bounded device-side wait that gives up records SSM_ERR_DEVICE_TIMEOUT in
 * the workspace header, which ssm_scan_check() reports.
 */
#ifndef SSM_SCAN_H_
#define SSM_SCAN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st *ssm_stream_t;

typedef enum {
  SSM_OK = 0,
  SSM_ERR_INVALID_ARG = -1,    /* null required pointer, bad size, misaligned */
  SSM_ERR_UNSUPPORTED = -2,    /* dstate > 64, unknown dtype or path */
  SSM_ERR_WORKSPACE = -3,      /* workspace missing or smaller than required */
  SSM_ERR_CUDA = -4,           /* a CUDA runtime call or launch failed */
  SSM_ERR_DEVICE_TIMEOUT = -5  /* a bounded device wait gave up */
} ssm_status;

typedef enum { SSM_F32 = 0, SSM_BF16 = 1 } ssm_dtype;

/* Forward schedule.  A warp holds 32/lanes channels, each walked by `lanes`
 * lanes over dstate/lanes states.  AUTO picks from the shape and the device:
 *  LOOKBACK  one persistent launch; every warp gets an equal share of
 *            (channel group x 32-step chunk) items; a group split between
 *            two warps passes its state through the workspace with a
 *            bounded wait (taken only after the writer's first item);
 *  SPLIT_L   two passes over time segments (segment end states from zero,
 *            a sequential carry over segments, then the output pass);
 *            for long sequences with few channels;
 *  PER_GROUP one warp per channel group over the whole sequence;
 *  LOOKBACK_WS  the look-back schedule (16-step chunks) with warp
 *            specialisation: producer warps load inputs and compute softplus,
 *            the gate and the output epilogue on the FMA pipe, consumer warps
 *            run only the recurrence.  2 lanes per channel (16-channel groups;
 *            the default when lanes = 0) or 4 (8-channel groups, dstate 5..16,
 *            channel-major, no saved states; SSM_ERR_UNSUPPORTED otherwise).
 *            AUTO picks it with 2 lanes once batch * ceil(dim/16) reaches 3/4
 *            of the device's SM sub-partitions (4 per SM), with 4 lanes when
 *            batch * ceil(dim/8) reaches them, and falls back to LOOKBACK
 *            where its shared memory does not fit (fp32, dstate > 32). */
typedef enum {
  SSM_PATH_AUTO = 0,
  SSM_PATH_LOOKBACK = 1,
  SSM_PATH_SPLIT_L = 2,
  SSM_PATH_PER_GROUP = 3,
  SSM_PATH_LOOKBACK_WS = 4
} ssm_path;

typedef struct {
  int64_t batch;    /* >= 0 */
  int64_t dim;      /* d_inner, >= 0 */
  int64_t seqlen;   /* L, >= 0; any value (ragged chunks are handled) */
  int64_t dstate;   /* N, 1..64 */
  int32_t io_dtype; /* ssm_dtype */
  int32_t path;     /* ssm_path (forward only; ignored by the backward) */
  int32_t lanes;    /* lanes per channel in the forward: 0 = auto, 2 or 4 (see LOOKBACK_WS) */
  int32_t flags;    /* ssm_flags bits; others must be 0 */
} ssm_shape;

/* Discretisation of the input term (ssm_shape.flags).
 *  default             Euler: Bbar = Delta * B, as in the aivaro.ru
 *                      selective_scan example (section 3).
 *  SSM_FLAG_ZOH_EXACT  exact zero-order hold for diagonal A, the reading
 *                      guide's "Metodo" formula Bbar = (Delta A)^-1
 *                      (exp(Delta A) - I) Delta B, i.e. per state
 *                      Bbar_n = (exp(Delta A_n) - 1) / A_n * B_n (Delta * B_n
 *                      where A_n = 0).  Forward on paths LOOKBACK and
 *                      LOOKBACK_WS (AUTO picks one of them; SPLIT_L and
 *                      PER_GROUP return SSM_ERR_UNSUPPORTED), ssm_scan_step,
 *                      and ssm_scan_bwd (channel-major activations). */
typedef enum {
  SSM_FLAG_ZOH_EXACT = 1,
  SSM_FLAG_SAVE_STATES = 2,
  SSM_FLAG_TOKEN_MAJOR = 4
} ssm_flags;

/* SSM_FLAG_TOKEN_MAJOR: u, delta, z and y (and, in ssm_scan_bwd, dout, du,
 * ddelta and dz) are laid out [batch][seqlen][dim] (dim contiguous), as a
 * projection produces them, instead of [batch][dim][seqlen]; B and C keep
 * their layout.  bf16 only, dim % 8 == 0, those activations 16-byte aligned,
 * the Euler term (SSM_ERR_UNSUPPORTED otherwise, SSM_ERR_INVALID_ARG for
 * misaligned pointers).  Forward on path AUTO or LOOKBACK_WS; backward for
 * dstate 9..16 (the d_state-16 kernel).  ssm_scan_step ignores it (one token
 * has no time axis). */

/* SSM_FLAG_SAVE_STATES (forward): besides y, the forward writes into its
 * workspace the state entering every 8-step chunk of every channel (fp32,
 * 4 * batch * G * ceil(seqlen/8) * 16 * NP bytes with G = 4 * ceil(dim/64)
 * groups of 16 channels and NP = dstate rounded up to a power of two >= 4;
 * ssm_scan_fwd_workspace_bytes counts them).  Passing that workspace as
 * fwd_workspace to ssm_scan_bwd, with the same shape and flags, lets the
 * backward skip its own forward pass over the chunks.  It runs on path
 * LOOKBACK_WS (AUTO picks it; other explicit paths, lanes = 4, and fp32 with
 * dstate > 32, whose tiles do not fit that kernel's shared memory, return
 * SSM_ERR_UNSUPPORTED). */

/* Bytes of workspace ssm_scan_fwd needs for `shape` on the current device
 * (at least 256: the header holding the device error word).  Returns 0 for
 * an invalid shape. */
size_t ssm_scan_fwd_workspace_bytes(const ssm_shape *shape);

/* Bytes of workspace ssm_scan_bwd needs (header, state checkpoints of the
 * forward recomputation, fp32 per-block partial sums of dB/dC, dA, dD and
 * ddelta_bias).  0 for an invalid shape. */
size_t ssm_scan_bwd_workspace_bytes(const ssm_shape *shape);

/* Forward selective scan (the operation above).
 *  u, delta, B, C, A, y          required
 *  D, z, delta_bias              nullable (term omitted / no gate / no bias)
 *  initial_state                 nullable: h_{-1} = 0 (aivaro.ru example)
 *  last_state                    nullable: h_{L-1} is written when given
 *  delta_softplus                nonzero: Delta = softplus(delta + bias)
 *  workspace/ws_bytes            device scratch, >= ssm_scan_fwd_workspace_bytes
 * Pointers must be aligned to their element size; 16-byte aligned rows take
 * the vector path.  y may not alias an input. */
ssm_status ssm_scan_fwd(const ssm_shape *shape, const void *u, const void *delta,
                        const float *A, const void *B, const void *C,
                        const float *D, const void *z, const float *delta_bias,
                        int delta_softplus, const float *initial_state,
                        void *y, float *last_state,
                        void *workspace, size_t ws_bytes, ssm_stream_t stream);

/* Backward of ssm_scan_fwd by recomputation: the states inside each chunk
 * are recomputed from the inputs, reading guide, "Expansao de Estado Ciente
 * de Hardware"; only the state entering each 8-step chunk may come from the
 * forward (fwd_workspace, nullable: a workspace that ssm_scan_fwd filled with
 * SSM_FLAG_SAVE_STATES for the same shape, flags, inputs and initial state;
 * the shape passed here must carry that flag too).  Without it the backward
 * first recomputes those chunk states itself.  Gradients of sum(dout * y):
 *  du, ddelta, dz          [batch][dim][seqlen] io dtype (ddelta is with
 *                          respect to the raw delta argument)
 *  dB, dC                  [batch][seqlen][dstate] io dtype, summed over dim
 *  dA                      [dim][dstate] fp32, summed over batch and seqlen
 *  dD, ddelta_bias         [dim] fp32, summed over batch and seqlen
 *  dinitial_state          [batch][dim][dstate] fp32 (nullable)
 * dz must be given exactly when z is, dD exactly when D is, ddelta_bias when
 * delta_bias is (else NULL).  Outputs are overwritten, not accumulated.
 * Every sum over channels, steps or the batch is formed per block and the
 * blocks are added in a fixed order (no atomics): a call repeated on the
 * same inputs gives bitwise-equal gradients.  The workspace holds those
 * per-block partial sums (ssm_scan_bwd_workspace_bytes). */
ssm_status ssm_scan_bwd(const ssm_shape *shape, const void *u, const void *delta,
                        const float *A, const void *B, const void *C,
                        const float *D, const void *z, const float *delta_bias,
                        int delta_softplus, const float *initial_state,
                        const void *dout, const void *fwd_workspace,
                        void *du, void *ddelta, float *dA, void *dB, void *dC,
                        float *dD, void *dz, float *ddelta_bias,
                        float *dinitial_state,
                        void *workspace, size_t ws_bytes, ssm_stream_t stream);

/* Forward scan for callers that cannot allocate device memory: inference
 * engine or framework plugins whose host owns every allocation and forbids
 * one on the execute path, or real-time loops that allocate nothing after
 * start-up.  The pages have no counterpart of this: it is a deployment
 * convenience.  Same arguments and results as ssm_scan_fwd, without the
 * workspace: the scratch lives in one 16 MiB device array inside the library
 * (held on every GPU that loads it until the process exits).
 *  - path AUTO keeps ssm_scan_fwd's own choice when that is LOOKBACK,
 *    LOOKBACK_WS (the default for Mamba layer shapes, token-major included)
 *    or PER_GROUP, whose scratch is bounded by the resident warps or is
 *    just the error word; where AUTO would pick SPLIT_L, whose scratch grows
 *    with the problem, it takes LOOKBACK instead.
 *  - SSM_FLAG_SAVE_STATES returns SSM_ERR_UNSUPPORTED: the saved states
 *    would sit in the shared array, out of the backward's reach.  The other
 *    flags behave as in ssm_scan_fwd.
 *  - Shapes needing more scratch than the array return SSM_ERR_UNSUPPORTED
 *    before any launch.
 *  - All calls share the array: calls whose kernels overlap on the GPU
 *    race, so order them on one stream.
 *  - Every call looks up the array's address for the current device and
 *    context (a host-side query; nothing is allocated or cached), so a
 *    device reset between calls is harmless and a failed lookup fails only
 *    that call (SSM_ERR_CUDA).
 *  - The device error word sits in the array too, so a bounded look-back
 *    wait that gives up is not reported to the caller of this entry point. */
ssm_status ssm_scan_fwd_noalloc(const ssm_shape *shape, const void *u, const void *delta,
                                const float *A, const void *B, const void *C,
                                const float *D, const void *z, const float *delta_bias,
                                int delta_softplus, const float *initial_state,
                                void *y, float *last_state, ssm_stream_t stream);

/* Single-step (recurrent) update: one new token for every (batch, channel),
 * the constant-time-per-token inference mode in which only the fixed-size
 * state is kept between tokens ("Mamba: Linear-Time Sequence Modeling with
 * Selective State Spaces", xyznot.com reading guide, the question on KV
 * caches; "O que e um modelo Mamba?", ibm.com, constant inference memory;
 * "Как работает Mamba", aivaro.ru, O(1) per step).  Computes, with the same
 * arithmetic as one step of ssm_scan_fwd:
 *   Delta = softplus(delta + delta_bias)   (or delta + delta_bias)
 *   state <- exp(Delta * A) (.) state + Delta * B * u      (in place)
 *   y      = (C . state + D * u) * SiLU(z)
 * shape->seqlen must be 1 (SSM_ERR_INVALID_ARG otherwise); path and lanes
 * are ignored.  Layouts: u, delta, z, y [batch][dim] io dtype; B, C
 * [batch][dstate] io dtype; A [dim][dstate], D and delta_bias [dim] fp32;
 * state [batch][dim][dstate] fp32, read and overwritten.  D, z and
 * delta_bias are nullable.  No workspace; nothing is allocated.  y may not
 * alias an input; state must not alias any other argument.  Calling it
 * seqlen times, feeding each token, gives the same y and final state as
 * ssm_scan_fwd over the seqlen tokens with initial_state = state (up to
 * rounding).  dstate % 4 == 0 with 16-byte aligned state and A (and B/C
 * rows aligned to 4 elements) takes 16-byte accesses; with dstate % 8 == 0 a
 * lane's 8 states of a row move as one 32-byte access where the state is
 * 32-byte aligned. */
ssm_status ssm_scan_step(const ssm_shape *shape, const void *u, const void *delta,
                         const float *A, const void *B, const void *C,
                         const float *D, const void *z, const float *delta_bias,
                         int delta_softplus, float *state, void *y, ssm_stream_t stream);

/* Causal depthwise 1-D convolution along seqlen, then SiLU if `silu`: the
 * convolution layer the Mamba block applies to x_proj before the SSM, whose
 * output goes through SiLU to become the SSM input ("O que e um modelo
 * Mamba?", ibm.com, the Mamba block walk-through).  Per channel d:
 *   out_t = act(bias[d] + sum_{k < width} weight[d][k] * x_{t - width + 1 + k})
 * so weight[d][width-1] multiplies the current token.  Inputs before t = 0
 * come from initial_state (zeros when NULL); final_state receives the last
 * width-1 inputs, so that a sequence can be convolved in pieces.
 *  x, out                     [batch][dim][seqlen]  io dtype (io_dtype)
 *  weight                     [dim][width] fp32, required
 *  bias                       [dim] fp32, nullable
 *  initial_state, final_state [batch][dim][width-1] fp32, nullable
 *                             (oldest input first; unused when width == 1)
 * width is 1..8 (SSM_ERR_UNSUPPORTED above).  out may not alias x.  Rows
 * whose bytes are a multiple of 32 on 32-byte aligned buffers move 32 bytes
 * per access, multiples of 16 on 16-byte aligned buffers 16 bytes; other rows
 * take element accesses. */
ssm_status ssm_causal_conv1d(int64_t batch, int64_t dim, int64_t seqlen, int32_t width,
                             int32_t io_dtype, const void *x, const float *weight,
                             const float *bias, const float *initial_state, int silu,
                             void *out, float *final_state, ssm_stream_t stream);

/* Backward of ssm_causal_conv1d: gradients of sum(dout * out) with respect
 * to x, weight, bias and the initial state, for the same arguments as the
 * forward call.  With a_t = bias + sum_k weight_k x_{t-width+1+k} and
 * out_t = act(a_t): da_t = dout_t act'(a_t); dx_s = sum_k weight_k
 * da_{s+width-1-k}; dweight_k = sum over batch and t of da_t x_{t-width+1+k};
 * dbias = sum of da_t.  The activations are recomputed, never stored.
 *  dout, dx                  [batch][dim][seqlen] io dtype (dx overwritten)
 *  dweight                   [dim][width] fp32, overwritten (required)
 *  dbias                     [dim] fp32, exactly when bias is given
 *  dinitial_state            [batch][dim][width-1] fp32, nullable
 * Argument checks as in the forward.  dx may not alias x or dout.  dx and
 * dinitial_state are bitwise repeatable; dweight and dbias are fp32 partial
 * sums (one per warp and row) added with atomics, so their last bits may
 * differ between runs. */
ssm_status ssm_causal_conv1d_bwd(int64_t batch, int64_t dim, int64_t seqlen, int32_t width,
                                 int32_t io_dtype, const void *x, const float *weight,
                                 const float *bias, const float *initial_state, int silu,
                                 const void *dout, void *dx, float *dweight, float *dbias,
                                 float *dinitial_state, ssm_stream_t stream);

/* Synchronises `stream`, reads and clears the device error word of
 * `workspace`.  SSM_OK, SSM_ERR_DEVICE_TIMEOUT or SSM_ERR_CUDA. */
ssm_status ssm_scan_check(void *workspace, ssm_stream_t stream);

/* Runs only the bounded inter-warp wait used by SSM_PATH_LOOKBACK on a flag
 * that nothing sets, with a limit of `timeout_us` microseconds (1..10^6), so
 * that the give-up path can be tested without faulting or hanging the GPU.
 * Afterwards ssm_scan_check(workspace) must report SSM_ERR_DEVICE_TIMEOUT.
 * workspace: >= 256 bytes. */
ssm_status ssm_scan_test_wait_timeout(void *workspace, size_t ws_bytes,
                                      int64_t timeout_us, ssm_stream_t stream);

/* Test hook for callers' error paths: the next `count` calls of
 * ssm_scan_fwd, ssm_scan_bwd, ssm_scan_step, ssm_causal_conv1d and
 * ssm_causal_conv1d_bwd (ssm_scan_fwd_noalloc included) that pass their
 * argument and workspace checks return SSM_ERR_CUDA as if their first launch
 * had failed with cudaErrorLaunchFailure; they launch nothing and leave every
 * buffer untouched.  count <= 0 disarms it.  Process-wide, thread-safe;
 * failures are consumed in call order. */
void ssm_scan_test_fail_next(int32_t count);

/* Test hook for ssm_scan_fwd_noalloc across a device reset: runs it on a
 * small seeded fp32 problem (batch 2, dim 32, seqlen 200, dstate 16) on
 * buffers it allocates, calls cudaDeviceReset, allocates afresh and runs it
 * again.  Returns 0 when both calls give equal bits, 1 when they differ, a
 * negative ssm_status when a call fails (SSM_ERR_CUDA for a failed
 * allocation, copy or reset).  The reset ends the process's primary context
 * on the current device: every earlier device allocation of the process is
 * gone, so call it only from a process that holds none it still needs. */
int32_t ssm_scan_test_noalloc_reset_cycle(void);

/* Path AUTO would choose for `shape` on the current device (for tests and
 * the benchmark); SSM_PATH_AUTO itself for an invalid shape. */
int32_t ssm_scan_fwd_path(const ssm_shape *shape);

const char *ssm_status_string(ssm_status status);

/* Library version, major*10000 + minor*100 + patch. */
int32_t ssm_scan_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SSM_SCAN_H_ */
