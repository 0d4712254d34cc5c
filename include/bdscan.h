/*
 * bdscan.h -- C ABI of libbdscan, the cache-aligned bidirectional Mamba-2 scan
 * of a block-diffusion (BDLM Mamba-H style) denoiser, for NVIDIA B200 (sm_100a).
 *
 * The operation (per batch row b and head h, with group g = h / (H / G)):
 *
 *   a_t = exp(dt_t * A_h)
 *   h_t = a_t * h_{t-1} + dt_t * x_t B_t^T               state h_t is P x N, fp32
 *   y_t = (h_t C_t + D_h * x_t) [* silu(z_t) if z is given]
 *
 * ("Training Hybrid Block Diffusion Language Models with Partial
 * Bidirectionality", eq. (1), Mamba-2 form with a scalar decay per head.)
 * The sequence is cut into blocks of T = block_len tokens.  The forward
 * direction runs over the whole sequence and leaves one boundary state per
 * block (eq. (10)); the reverse direction runs right to left inside each block
 * only, from a zero state, with its own parameters (eq. (12)); the two outputs
 * are summed (eq. (13); "Breaking the Bottleneck with DiffuApriel",
 * section 3.2, eq. (6)).
 *
 * Layouts: every tensor is dense row-major, innermost dimension last.
 *   x, z, y    [B][L][H][P]     in_dtype (x, z) / out_dtype (y)
 *   dt         [B][L][H]        in_dtype; already positive (softplus applied)
 *   B, C       [B][L][G][N]     in_dtype
 *   A, D       [H]              fp32
 *   state      [B][H][P][N]     fp32 (h0, state_in, state_out, final_state)
 *   block_states [B][K][H][P][N] fp32, K = L / T; block_states[b][k] is the
 *              forward state after token (k+1)*T - 1 (end of block k).
 *
 * Ownership: the caller owns every buffer, including the workspace; the
 * library allocates no device memory.  Its only global mutable state is the
 * process-wide options (bdscan_set_option) and, for
 * bdscan_block_step_noalloc alone, that entry point's built-in device scratch
 * buffer; every other entry point works only on the caller's buffers, so
 * calls with distinct buffers are reentrant.  All device pointers must be
 * device-accessible memory of the current device.  Every call is asynchronous
 * on `cuda_stream` (a cudaStream_t; NULL = the legacy default stream).
 *
 * Errors: every entry point validates its arguments synchronously, before any
 * launch, and returns a BDSCAN_* status; nothing aborts the process.  A launch
 * failure returns BDSCAN_ERR_CUDA.  Numeric problems (NaN/Inf inputs) are not
 * trapped; they propagate to the outputs of the same (b, h) only.
 */
#ifndef BDSCAN_H
#define BDSCAN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* element types (bdscan_shape_t.in_dtype / out_dtype) */
#define BDSCAN_BF16 0
#define BDSCAN_FP32 1

/* status codes */
#define BDSCAN_OK 0
#define BDSCAN_ERR_INVALID_ARG (-1)       /* null pointer, bad enum, negative size, aliasing */
#define BDSCAN_ERR_UNSUPPORTED_SHAPE (-2) /* shape outside the supported set (see below) */
#define BDSCAN_ERR_MISALIGNED (-3)        /* a pointer is not 16-byte aligned */
#define BDSCAN_ERR_WORKSPACE (-4)         /* ws NULL or ws_bytes < bdscan_workspace_size() */
#define BDSCAN_ERR_CUDA (-5)              /* a kernel launch or CUDA runtime call failed */
#define BDSCAN_ERR_TIMEOUT (-6)           /* a bounded device-side wait ran out (check_status) */
#define BDSCAN_ERR_SCRATCH_LIMIT (-7)     /* shape needs more than the built-in no-alloc scratch */

/* operations (bdscan_workspace_size) */
#define BDSCAN_OP_PREFIX 0
#define BDSCAN_OP_BLOCK_STEP 1
#define BDSCAN_OP_ALLBLOCK 2
#define BDSCAN_OP_ALLBLOCK_BACKWARD 3
#define BDSCAN_OP_CONV_PREFIX 4   /* no workspace (bdscan_workspace_size returns 0) */
#define BDSCAN_OP_CONV_ALLBLOCK 5 /* no workspace */
#define BDSCAN_OP_GATED_RMSNORM 6 /* no workspace */
#define BDSCAN_OP_CONV_BLOCK_STEP 7

/* Problem shape.  Supported: batch >= 0, seqlen >= 0, seqlen % block_len == 0,
 * 1 <= block_len <= 32 or block_len % 32 == 0 (<= 256), chunk_len % block_len
 * == 0 (chunk_len is the tile of tokens a kernel stages at once; it changes
 * no result beyond rounding order), nheads % ngroups == 0, headdim in
 * {16, 32, 64, 128}, 1 <= dstate <= 256. */
typedef struct {
    int64_t batch, seqlen, nheads, headdim, dstate, ngroups, block_len, chunk_len;
    int32_t in_dtype;  /* BDSCAN_BF16 | BDSCAN_FP32: x, dt, B, C, z */
    int32_t out_dtype; /* BDSCAN_FP32 | BDSCAN_BF16: y */
} bdscan_shape_t;

/* One scan direction's inputs (device pointers).  z may be NULL (no gate).
 * A direction may alias another (tied weights). */
typedef struct {
    const void *x, *dt, *B, *C, *z;
    const float *A, *D;
} bdscan_dir_t;

/* bdscan_prefix -- clean-prefix scan, for prefill and for committing blocks.
 * Source: eq. (10) (boundary states) and the commit described after eq. (6)
 * ("after the block is finalized, a clean forward pass ... appends") of the
 * first page; eq. (12)-(13) for the optional block-local reverse.
 *   fwd          forward direction (required)
 *   rev          reverse direction, applied inside every block; NULL = none
 *   h0           [B][H][P][N] initial state; NULL = zeros
 *   y            [B][L][H][P] output (out_dtype), y = y_fwd + y_rev
 *   block_states [B][K][H][P][N] or NULL: forward state at the end of each block
 *   final_state  [B][H][P][N] or NULL: forward state after token L-1
 *                (== h0, or zeros, when L == 0)
 *   ws, ws_bytes workspace of at least bdscan_workspace_size(shape, PREFIX)
 *                bytes (16-byte aligned); its contents need no initialisation
 * y must not overlap any input; block_states / final_state must not overlap
 * h0 or any input. */
int bdscan_prefix(const bdscan_shape_t *shape, const bdscan_dir_t *fwd, const bdscan_dir_t *rev,
                  const float *h0, void *y, float *block_states, float *final_state, void *ws,
                  size_t ws_bytes, void *cuda_stream);

/* bdscan_block_step -- one denoising step of the active block from the cached
 * forward state: forward continuation (eq. (11)), block-local reverse
 * (eq. (12)), sum (eq. (13)).  shape->seqlen must equal shape->block_len.
 *   state_in   [B][H][P][N] cached state (read only; never modified unless it
 *              is also passed as state_out)
 *   y          [B][T][H][P] output
 *   state_out  [B][H][P][N] or NULL: forward state after the block (commit);
 *              may be equal to state_in (in-place commit), must not partially
 *              overlap it. */
int bdscan_block_step(const bdscan_shape_t *shape, const bdscan_dir_t *fwd,
                      const bdscan_dir_t *rev, const float *state_in, void *y, float *state_out,
                      void *ws, size_t ws_bytes, void *cuda_stream);

/* bdscan_allblock -- all-block training pass (eq. (14) and the all-block
 * objective after eq. (5)): the clean stream is scanned as by bdscan_prefix
 * (with clean_rev inside each block) and emits every boundary state; every
 * noisy block k is scanned forward from the clean boundary state before it
 * (h0 for k = 0) plus its own block-local reverse.
 *   y_clean      [B][L][H][P] or NULL
 *   y_noisy      [B][L][H][P] (required)
 *   block_states [B][K][H][P][N] (required) */
int bdscan_allblock(const bdscan_shape_t *shape, const bdscan_dir_t *clean_fwd,
                    const bdscan_dir_t *clean_rev, const bdscan_dir_t *noisy_fwd,
                    const bdscan_dir_t *noisy_rev, const float *h0, void *y_clean, void *y_noisy,
                    float *block_states, void *ws, size_t ws_bytes, void *cuda_stream);

/* Gradients of one direction (fp32, overwritten): dx [B][L][H][P],
 * ddt [B][L][H], dB and dC [B][L][G][N] (summed over the heads of a group),
 * dA and dD [H] (summed over batch rows and tokens). */
typedef struct {
    float *dx, *ddt, *dB, *dC, *dA, *dD;
} bdscan_grad_t;

/* bdscan_allblock_backward -- reverse-mode derivative of bdscan_allblock for
 * training: given dL/dy_clean, dL/dy_noisy and dL/dstates of a loss
 * L(y_clean, y_noisy, block_states), the gradients of every input.  The
 * all-block objective makes the noisy blocks' losses reach the clean prefix
 * scan through the boundary states ("Training Hybrid Block Diffusion Language
 * Models with Partial Bidirectionality", all-block paragraph after eq. (5),
 * eq. (14)); the derivative itself is that of eq. (1) over eqs. (10)-(13).
 *   directions    as for bdscan_allblock (ungated only: a direction with z
 *                 gives BDSCAN_ERR_UNSUPPORTED_SHAPE)
 *   h0            [B][H][P][N] or NULL (zeros), as in the forward call
 *   block_states  [B][K][H][P][N]: the forward call's output (required)
 *   dy_clean      [B][L][H][P] of out_dtype, or NULL (no loss on y_clean)
 *   dy_noisy      [B][L][H][P] of out_dtype (required)
 *   dstates       [B][K][H][P][N] fp32 or NULL (no loss on the states)
 *   g_*           gradient outputs per direction (required for the present
 *                 directions; pointers of the absent ones are ignored)
 *   dh0           [B][H][P][N] or NULL
 *   ws, ws_bytes  at least bdscan_workspace_size(shape, ALLBLOCK_BACKWARD)
 *                 bytes (per-head / per-row partial sums, reduced in a fixed
 *                 order: the result is deterministic)
 * Shapes: as for the forward; additionally block_len and dstate must be
 * multiples of 4 and the per-block shared-memory plan (P, N, block_len) must
 * fit one CTA (P = 64, N = 128, block_len = 32 does).
 * Gradients must not overlap any input or each other. */
int bdscan_allblock_backward(const bdscan_shape_t *shape, const bdscan_dir_t *clean_fwd,
                             const bdscan_dir_t *clean_rev, const bdscan_dir_t *noisy_fwd,
                             const bdscan_dir_t *noisy_rev, const float *h0, const float *block_states,
                             const void *dy_clean, const void *dy_noisy, const float *dstates,
                             const bdscan_grad_t *g_clean_fwd, const bdscan_grad_t *g_clean_rev,
                             const bdscan_grad_t *g_noisy_fwd, const bdscan_grad_t *g_noisy_rev,
                             float *dh0, void *ws, size_t ws_bytes, void *cuda_stream);

/* ---- Short convolution in front of the scan ---------------------------------
 *
 * In a Mamba-2 layer the scan's x, B and C are not the input projection's
 * outputs themselves: each of their channels first goes through a short
 * depthwise convolution over time and a SiLU.  The layer's cache for the
 * block-diffusion decoder therefore keeps, beside the scan state, the
 * convolution's state: the last width-1 pre-convolution rows of the forward
 * stream ("Training Hybrid Block Diffusion Language Models with Partial
 * Bidirectionality", the paragraph after eq. (14) on the cache object of a
 * Mamba layer).  The forward direction's convolution is causal; the reverse
 * direction's is anti-causal ("Breaking the Bottleneck with DiffuApriel",
 * section 3.2, after eq. (5)) and, like its scan, confined to the block.
 *
 * Per channel c of one direction, with u the pre-convolution input, v the
 * output, W = width, w[c][0..W-1] the taps and s(v) = v / (1 + exp(-v)):
 *   forward:  v_t = s(bias[c] + sum_j w[c][j] * u_{t-(W-1)+j})
 *             where u_{t'} for t' < 0 is row W-1+t' of the conv state (zeros
 *             when no state is given); tokens earlier than the state are 0.
 *   reverse:  v_t = s(bias[c] + sum_j w[c][j] * u_{t+(W-1)-j})
 *             where u_{t'} = 0 for t' past the end of t's block: the forward
 *             rule applied to the block read right to left, from zeros.
 * (s is skipped when `silu` is 0.)
 *
 * Channels: the x channels (h, p) in order, then B's (g, n), then C's (g, n):
 * Cx = H*P + 2*G*N channels.  dt and z are not convolved.
 * Layouts: inputs and outputs have the layouts of bdscan_dir_t's x, B, C and
 * the element type in_dtype; weight [Cx][W] fp32; bias [Cx] fp32 or NULL;
 * conv state [B][W-1][Cx] in_dtype (rows oldest first; row W-2 is the token
 * just before the sequence).
 * Supported: 1 <= width <= 4 (else BDSCAN_ERR_UNSUPPORTED_SHAPE), G*N a
 * multiple of 4, every pointer 16-byte aligned.  Each output is computed in
 * fp32 (taps applied oldest row first, bias first) from the rounded inputs and
 * rounded once to in_dtype.  The calls take no workspace; one kernel launch. */
typedef struct {
    const void *x, *B, *C;  /* pre-convolution inputs */
    const float *weight;    /* [Cx][width] */
    const float *bias;      /* [Cx] or NULL (zeros) */
    void *x_out, *B_out, *C_out;
} bdscan_conv_t;

/* bdscan_conv_prefix -- the convolution of one sequence (prefill, commit, or
 * one denoising step of the active block with shape->seqlen == block_len).
 *   fwd             forward direction (required)
 *   rev             reverse direction (anti-causal inside each block) or NULL
 *   conv_state_in   [B][W-1][Cx] or NULL (zeros): rows before token 0
 *   conv_state_out  [B][W-1][Cx] or NULL: the last W-1 rows of the forward
 *                   stream (conv_state_in followed by fwd's inputs); may
 *                   equal conv_state_in only when seqlen <= 32
 * Outputs must not overlap any input or each other (except the in-place
 * state above). */
int bdscan_conv_prefix(const bdscan_shape_t *shape, int width, int silu, const bdscan_conv_t *fwd,
                       const bdscan_conv_t *rev, const void *conv_state_in, void *conv_state_out,
                       void *cuda_stream);

/* bdscan_conv_allblock -- the convolution of the all-block training pass: the
 * clean stream as by bdscan_conv_prefix; each noisy block k's forward
 * convolution continues from the clean stream's rows before the block (the
 * conv state at the end of block k-1; conv_state_in for k = 0), the noisy
 * reverse stays inside the block.  clean_rev / noisy_rev may be NULL. */
int bdscan_conv_allblock(const bdscan_shape_t *shape, int width, int silu,
                         const bdscan_conv_t *clean_fwd, const bdscan_conv_t *clean_rev,
                         const bdscan_conv_t *noisy_fwd, const bdscan_conv_t *noisy_rev,
                         const void *conv_state_in, void *cuda_stream);

/* bdscan_conv_block_step -- one denoising step of a Mamba layer's
 * selective-scan core from its cache, without commit: the short convolution
 * (+SiLU) of both directions' x, B and C over the active block, the forward
 * direction continuing from the conv state (exactly bdscan_conv_prefix with
 * seqlen == block_len), then the scan step on the convolved inputs from the
 * cached scan state (exactly bdscan_block_step with state_out NULL).  The two
 * halves are the same operations as those calls ("Training Hybrid Block
 * Diffusion Language Models with Partial Bidirectionality", the paragraph after
 * eq. (14): a Mamba layer's cache holds its conv state beside its scan state).
 *   conv_fwd, conv_rev  pre-convolution inputs, weights and bias of the two
 *                       directions (both required); x_out, B_out and C_out
 *                       are ignored: the convolved inputs are not returned
 *   conv_state_in       [B][W-1][Cx] or NULL (zeros), as bdscan_conv_prefix
 *   fwd, rev            the scan directions' dt, A, D and z (both required);
 *                       their x, B and C are ignored (the convolution's
 *                       outputs take their place)
 *   state_in            [B][H][P][N] cached scan state (read only)
 *   y                   [B][T][H][P] output (shape->out_dtype)
 *   ws, ws_bytes        at least bdscan_workspace_size(shape, CONV_BLOCK_STEP)
 * shape->seqlen must equal shape->block_len.  The convolution kernel writes
 * the convolved inputs into the workspace and the step's kernels follow as
 * programmatic dependents (two launches for a small batch on the tensor-core
 * path: bdscan_kernel_launches).  y must not overlap any input. */
int bdscan_conv_block_step(const bdscan_shape_t *shape, int width, int silu, const bdscan_conv_t *conv_fwd,
                           const bdscan_conv_t *conv_rev, const void *conv_state_in, const bdscan_dir_t *fwd,
                           const bdscan_dir_t *rev, const float *state_in, void *y, void *ws, size_t ws_bytes,
                           void *cuda_stream);

/* bdscan_gated_rmsnorm -- the normalisation of the summed output before the
 * layer's projection ("Breaking the Bottleneck with DiffuApriel", section 3.2
 * after eq. (6)), read as the Mamba-2 layer's gated RMSNorm with the gate
 * before the norm, written in bf16.  Per token row (b, t), with C = H*P
 * channels cut into `groups` groups of gs = C / groups consecutive channels:
 *   v_c   = y_c * silu(z_c)            (v = y when z is NULL)
 *   out_c = v_c * weight_c / sqrt(mean_{c' in group(c)} v_c'^2 + eps)
 *   y       [B][L][H][P] of shape->out_dtype (a scan call's output)
 *   z       [B][L][H][P] of shape->in_dtype, or NULL
 *   weight  [H*P] fp32
 *   groups  >= 1, C % groups == 0, gs % 4 == 0 (else UNSUPPORTED_SHAPE); the
 *           row (4*C + C + 4*groups bytes) must fit one CTA's shared memory
 *   eps     >= 0 and finite
 *   out     [B][L][H][P] bf16; may be y itself when y is bf16 (in place),
 *           must not overlap y otherwise, nor z or weight
 * Computed in fp32 (sums of squares in a fixed order: deterministic), rounded
 * once to bf16.  One kernel launch; no workspace. */
int bdscan_gated_rmsnorm(const bdscan_shape_t *shape, const void *y, const void *z, const float *weight,
                         int64_t groups, float eps, void *out, void *cuda_stream);

/* Workspace bytes an operation needs for this shape (>= 256: the first 256
 * bytes hold the device status word).  Returns 0 for an invalid shape/op. */
size_t bdscan_workspace_size(const bdscan_shape_t *shape, int op);

/* Number of kernels one call of `op` launches for this shape (0 for an empty
 * problem, -1 for an invalid shape/op).  Lets a caller size CUDA graphs and
 * count launches; it does not launch anything.  BDSCAN_OP_BLOCK_STEP counts a
 * step without state_out; a committing step launches the C B^T pre-pass too
 * (2 on the tensor-core path).  Options in force at the call are assumed
 * (BDSCAN_OPT_CB_PREPASS, BDSCAN_OPT_FORCE_GENERIC). */
int bdscan_kernel_launches(const bdscan_shape_t *shape, int op);

/* Reads the device status word in ws after the work queued on cuda_stream
 * completes (synchronises that stream), clears it, and returns it
 * (BDSCAN_OK or BDSCAN_ERR_TIMEOUT).  Returns BDSCAN_ERR_CUDA if the copy fails. */
int bdscan_check_status(const void *ws, void *cuda_stream);

/* Static description of a status code. */
const char *bdscan_status_string(int status);

/* bdscan_block_step_noalloc -- the denoising step of bdscan_block_step for
 * callers that cannot allocate device memory: code that runs under a fixed
 * memory plan that has already handed out all device memory (an inference
 * server or graph executor with a static arena), or code that runs while a
 * stream is being captured, where cudaMalloc is not allowed.  The pages have
 * no counterpart; this is a deployment convenience.
 *
 * Same arguments, results and errors as bdscan_block_step, minus the
 * workspace: the scratch it needs (the status word and the tensor-core path's
 * C B^T tiles) lives in a static device buffer of BDSCAN_NOALLOC_SCRATCH_BYTES
 * inside the library, which every GPU that loads the library holds until the
 * process exits.  It calls no cudaMalloc or cudaFree.
 *   - Shapes whose workspace (bdscan_workspace_size(shape, BLOCK_STEP)) exceeds
 *     BDSCAN_NOALLOC_SCRATCH_BYTES are rejected with BDSCAN_ERR_SCRATCH_LIMIT
 *     (for the tensor-core shapes: batch * ngroups <= 1024).
 *   - The first call on a device looks up the buffer's device address on that
 *     device (the device current at the call); make that first call before any
 *     stream capture begins.
 *   - All calls share the one buffer: calls that may overlap on the GPU (other
 *     streams, other host threads) race on it; serialise them on one stream.
 *   - bdscan_check_status() reads its status word through
 *     bdscan_noalloc_scratch(), which returns the buffer's device address on
 *     the current device (NULL if the lookup fails). */
#define BDSCAN_NOALLOC_SCRATCH_BYTES ((size_t)(4u << 20) + 1024u)
int bdscan_block_step_noalloc(const bdscan_shape_t *shape, const bdscan_dir_t *fwd,
                              const bdscan_dir_t *rev, const float *state_in, void *y,
                              float *state_out, void *cuda_stream);
void *bdscan_noalloc_scratch(void);

/* Library version (major * 10000 + minor * 100 + patch). */
int bdscan_version(void);

/* Process-wide options.  Their initial values come from the environment,
 * read once at the first call that uses them (not per call):
 *   BDSCAN_OPT_WAIT_TIMEOUT_NS  limit of every bounded device-side wait of
 *                               the tensor-core kernels, in ns (default 2e9;
 *                               env BDSCAN_WAIT_TIMEOUT_NS).  A wait that runs
 *                               out sets BDSCAN_ERR_TIMEOUT in the status word.
 *   BDSCAN_OPT_FORCE_GENERIC    1: every scan runs on the CUDA-core kernel
 *                               (default 0; env BDSCAN_FORCE_GENERIC=1)
 *   BDSCAN_OPT_VERBOSE          1: launch failures are printed to stderr
 *                               (default 0; env BDSCAN_VERBOSE=1)
 *   BDSCAN_OPT_CB_PREPASS       1: small-batch block steps (no state out, at
 *                               most one (sequence, head) per SM) also take the
 *                               separate C B^T pre-pass instead of computing
 *                               C B^T inside the scan kernel (default 0; env
 *                               BDSCAN_CB_PREPASS=1).  Same results up to the
 *                               bf16 rounding of the C B^T tiles.
 * bdscan_set_option returns the previous value, or BDSCAN_ERR_INVALID_ARG for
 * an unknown option or a value out of range; a change applies to calls made
 * after it returns.  bdscan_get_option returns the current value (or
 * BDSCAN_ERR_INVALID_ARG). */
#define BDSCAN_OPT_WAIT_TIMEOUT_NS 0
#define BDSCAN_OPT_FORCE_GENERIC 1
#define BDSCAN_OPT_VERBOSE 2
#define BDSCAN_OPT_CB_PREPASS 3
long long bdscan_set_option(int option, long long value);
long long bdscan_get_option(int option);

#ifdef __cplusplus
}
#endif
#endif /* BDSCAN_H */
