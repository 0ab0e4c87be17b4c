/*
 * ssm_scan.h -- C ABI of libssmscan.so, a selective-scan (S6) library for
 * NVIDIA B200 (sm_100a).
 *
 * What the library computes (forward), per batch row b and channel d, for
 * t = 0 .. seqlen-1, with n = 0 .. dstate-1:
 *
 *   Δ_t     = softplus(delta[b,d,t] + delta_bias[d])   (no softplus if the
 *             flag is 0; bias treated as 0 if NULL)
 *   Ā_t[n]  = exp(Δ_t A[d,n])
 *   h_t[n]  = Ā_t[n] h_{t-1}[n] + Δ_t B[b,n,t] u[b,d,t],   h_{-1} = 0
 *   y_t     = Σ_n C[b,n,t] h_t[n] + D[d] u[b,d,t]          (D term if D given)
 *   out_t   = y_t · z_t · sigmoid(z_t)                      (if z given)
 *
 * Sources: booiljung.github.io, "3.2 선택적 스캔(Selective Scan) 알고리즘과
 * 정보의 압축 및 선별" -- §1.1 (the recurrence and readout), §1.2 (selection:
 * Δ_t = Softplus(Parameter + Linear_1(x_t)), B_t and C_t per token), §2.1
 * (Ā_t = exp(Δ_t A) with diagonal A), §3.2 (fused kernel: only y reaches
 * HBM), §3.3 (backward recomputes the states); 정보관리기술사 학습 노트,
 * "상태공간 모델(SSM)과 Mamba 아키텍처", §3 (SiLU gate branch multiplied into
 * the SSM output).  The input matrix is discretised as B̄_t = Δ_t B_t and the
 * D skip term is added before the gate.
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library
 *    never allocates or frees device memory.  Layouts are dense row-major:
 *      u, delta, z, out, dout       [batch][dim][seqlen]   io dtype
 *      B, C                         [batch][dstate][seqlen] io dtype
 *      A                            [dim][dstate]          float32
 *      D, delta_bias                [dim]                  float32
 *      last_state                   [batch][dim][dstate]   float32
 *      ckpt                         [batch][dim][nchunk][dstate] float32,
 *                                   nchunk = ceil(seqlen / SSM_CKPT_CHUNK)
 *      du, ddelta, dz               [batch][dim][seqlen]   float32
 *      dB, dC                       [batch][dstate][seqlen] float32
 *      dA                           [dim][dstate]          float32
 *      dD, ddelta_bias              [dim]                  float32
 *    Pointers must be aligned to their element size.  The fast path (16-byte
 *    vector loads and stores) is taken when every io tensor is 16-byte
 *    aligned and seqlen * element size is a multiple of 16; otherwise the
 *    same kernels use element-wise accesses.
 *  - Pointers are checked with cudaPointerGetAttributes: host memory, or
 *    memory of a device other than the current one, is refused with
 *    SSM_ERR_INVALID_ARG before anything is launched.
 *  - Calls are asynchronous on `stream` (a cudaStream_t passed as void*;
 *    NULL is the legacy default stream).  The return value reports argument
 *    and launch errors only; use the stream's own synchronisation to wait.
 *  - On any error nothing is launched, and ssm_last_error_string() (per
 *    calling thread) describes it.
 *  - Supported: dstate in {1, 2, 4, 8, 16, 32}; io dtype float32 or bfloat16;
 *    1 <= seqlen, batch, dim; batch * dim * seqlen < 2^31.
 */
#ifndef SSM_SCAN_H
#define SSM_SCAN_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SSM_OK = 0,
    SSM_ERR_INVALID_ARG = 1, /* null required pointer, bad size, misalignment */
    SSM_ERR_UNSUPPORTED = 2, /* valid but not implemented (e.g. dstate = 3) */
    SSM_ERR_CUDA = 3,        /* a CUDA runtime call or kernel launch failed */
    SSM_ERR_TIMEOUT = 4      /* a bounded device-side wait gave up */
} ssm_status_t;

typedef enum { SSM_F32 = 0, SSM_BF16 = 1 } ssm_dtype_t;

typedef struct {
    int batch;            /* number of independent sequences */
    int dim;              /* channels D (each has its own A row, D, bias) */
    int seqlen;           /* L, time steps */
    int dstate;           /* N, state size per channel */
    ssm_dtype_t io_dtype; /* dtype of u, delta, z, B, C, out, dout */
} ssm_shape_t;

/* Discretisation of the input matrix (booiljung.github.io, "3.2 선택적
 * 스캔(Selective Scan) 알고리즘", §2.1 prints the zero-order hold
 * B̄ = (ΔA)^-1 (exp(ΔA) - I) ΔB; with diagonal A it is elementwise). */
typedef enum {
    SSM_DISC_DELTA_B = 0, /* B̄ = Δ B: what every entry point without _ex uses */
    SSM_DISC_ZOH = 1      /* B̄ = (exp(Δ A) - 1) / A · B, Δ B where A = 0 (its limit) */
} ssm_discretization_t;

/* Options of the _ex entry points. */
typedef struct {
    int delta_softplus;                  /* nonzero: Δ = softplus(delta + delta_bias) */
    ssm_discretization_t discretization;
} ssm_options_t;

/* Steps between two saved states in the forward's checkpoint buffer.  The
 * backward recomputes each such window of steps once from its saved state. */
#define SSM_CKPT_CHUNK 8

/* Library version, major * 10000 + minor * 100 + patch. */
int ssm_version(void);

/* Message for the last error returned on this thread ("" if none). */
const char *ssm_last_error_string(void);

/*
 * Diagnostic (the pages have no counterpart): which kernels the last forward
 * or backward call on this thread launched: "fwd:tma", "fwd:general",
 * "fwd:chunked" (the two-level scan of ssm_selective_scan_fwd_ws), "bwd:tma"
 * or "bwd:general" ("" before any call).  A static string; the library owns
 * it.
 */
const char *ssm_last_kernel_path(void);

/*
 * Bytes of the optional checkpoint buffer `ckpt` of ssm_selective_scan_fwd:
 * batch * dim * ceil(seqlen / SSM_CKPT_CHUNK) * dstate * 4.
 */
ssm_status_t ssm_selective_scan_ckpt_bytes(const ssm_shape_t *shape, size_t *bytes);

/*
 * The same size under the name of the boundary's original plan: the bytes
 * of the checkpoint buffer (the backward's workspace when the caller keeps
 * the forward's checkpoints).  Identical to ssm_selective_scan_ckpt_bytes.
 */
ssm_status_t ssm_selective_scan_workspace_size(const ssm_shape_t *shape, size_t *ckpt_bytes);

/*
 * Forward selective scan (see the header comment for the arithmetic).
 *
 *  u, delta, A, B, C : required inputs.
 *  D, z, delta_bias  : optional (NULL = term absent).
 *  delta_softplus    : nonzero applies softplus to delta + delta_bias.
 *  out               : required output, io dtype (may not alias an input).
 *  last_state        : optional output, h_{seqlen-1}.
 *  ckpt              : optional output; ckpt[b][d][k][:] = h at the last step
 *                      of chunk k (step min(seqlen, (k+1)*SSM_CKPT_CHUNK) - 1).
 *                      Pass it to ssm_selective_scan_bwd to skip the
 *                      backward's state-recompute pre-pass.
 * Errors: SSM_ERR_INVALID_ARG, SSM_ERR_UNSUPPORTED, SSM_ERR_CUDA.
 */
ssm_status_t ssm_selective_scan_fwd(const ssm_shape_t *shape,
                                    const void *u, const void *delta,
                                    const float *A, const void *B, const void *C,
                                    const float *D, const void *z,
                                    const float *delta_bias, int delta_softplus,
                                    void *out, float *last_state, float *ckpt,
                                    void *stream);

/*
 * ssm_selective_scan_fwd with options: opts->delta_softplus replaces
 * delta_softplus and opts->discretization selects B̄ (the backward serves
 * SSM_DISC_ZOH with its general kernel; the forward with its fast kernel at
 * dstate 16).  Checkpoints written with SSM_DISC_ZOH must be passed to a
 * backward with SSM_DISC_ZOH.
 * Errors: as ssm_selective_scan_fwd, plus SSM_ERR_INVALID_ARG for a NULL
 * opts or an unknown discretization.
 */
ssm_status_t ssm_selective_scan_fwd_ex(const ssm_shape_t *shape, const ssm_options_t *opts,
                                       const void *u, const void *delta,
                                       const float *A, const void *B, const void *C,
                                       const float *D, const void *z,
                                       const float *delta_bias,
                                       void *out, float *last_state, float *ckpt,
                                       void *stream);

/*
 * Workspace for the two-level scan along the sequence (booiljung.github.io,
 * "3.2 선택적 스캔(Selective Scan) 알고리즘" §2.2: chunk summaries (Ā product,
 * local state) composed with the associative operator (a_j, b_j)•(a_i, b_i) =
 * (a_j a_i, a_j b_i + b_j)).  When a shape has long sequences over few
 * channel rows (fewer than 64 rows per SM), ssm_selective_scan_fwd_ws cuts
 * the sequence into K chunks of whole 128-step blocks and runs three launches
 * on `stream`: the summaries of chunks 0..K-2 (end state from a zero state,
 * and Σ_t Δ_t), the exclusive combine of the summaries (the state entering
 * each chunk), and every chunk from its entering state.
 *
 * ssm_selective_scan_fwd_workspace_bytes: the bytes of workspace that
 *   ssm_selective_scan_fwd_ws uses for this shape on the current device (0:
 *   the one-pass forward is used, and the workspace may be NULL).  The plan
 *   assumes 16-byte aligned rows; with unaligned pointers the one-pass path
 *   runs and the workspace is not touched.
 * ssm_selective_scan_fwd_ws: ssm_selective_scan_fwd_ex with a caller-owned
 *   device workspace (16-byte aligned, `workspace_bytes` long; its contents
 *   on entry are ignored and on return undefined).  Results match the
 *   one-pass forward to within fp32 rounding (the chunks' states are joined
 *   in fp32).  Calls that share a workspace must not overlap on the GPU.
 * Errors: as ssm_selective_scan_fwd_ex, plus SSM_ERR_INVALID_ARG when the
 * workspace is smaller than the plan needs.
 */
ssm_status_t ssm_selective_scan_fwd_workspace_bytes(const ssm_shape_t *shape,
                                                    const ssm_options_t *opts, size_t *bytes);

ssm_status_t ssm_selective_scan_fwd_ws(const ssm_shape_t *shape, const ssm_options_t *opts,
                                       const void *u, const void *delta,
                                       const float *A, const void *B, const void *C,
                                       const float *D, const void *z,
                                       const float *delta_bias,
                                       void *out, float *last_state, float *ckpt,
                                       void *workspace, size_t workspace_bytes,
                                       void *stream);

/*
 * Bytes of device scratch that ssm_selective_scan_bwd needs: 0 when the
 * caller passes the forward's checkpoints (have_ckpt != 0), otherwise the
 * size of a checkpoint buffer, which the backward fills itself first.
 */
ssm_status_t ssm_selective_scan_bwd_scratch_bytes(const ssm_shape_t *shape,
                                                  int have_ckpt, size_t *bytes);

/*
 * Backward selective scan: given dout = dLoss/dout, writes the gradients of
 * Loss with respect to every input of the forward.  The states are recomputed
 * from the checkpoints (booiljung.github.io "3.2 Selective Scan" §3.3);
 * nothing of size batch*dim*seqlen*dstate is ever stored.
 *
 *  u .. delta_softplus : the forward's inputs, unchanged.
 *  dout                : required, io dtype.
 *  ckpt                : the forward's checkpoint buffer, or NULL.
 *  du, ddelta, dA, dB, dC : required outputs (float32, overwritten).
 *  dD, dz, ddelta_bias : required iff D, z, delta_bias (resp.) are non-NULL,
 *                        and must be NULL otherwise.
 *  scratch, scratch_bytes : device scratch of at least
 *                        ssm_selective_scan_bwd_scratch_bytes(shape, ckpt != NULL)
 *                        bytes (may be NULL when that is 0).
 * The gradient outputs must not alias each other or any input.
 * Errors: SSM_ERR_INVALID_ARG, SSM_ERR_UNSUPPORTED, SSM_ERR_CUDA.
 */
ssm_status_t ssm_selective_scan_bwd(const ssm_shape_t *shape,
                                    const void *u, const void *delta,
                                    const float *A, const void *B, const void *C,
                                    const float *D, const void *z,
                                    const float *delta_bias, int delta_softplus,
                                    const void *dout, const float *ckpt,
                                    float *du, float *ddelta, float *dA,
                                    float *dB, float *dC, float *dD, float *dz,
                                    float *ddelta_bias,
                                    void *scratch, size_t scratch_bytes,
                                    void *stream);

/*
 * Backward selective scan that allocates nothing (the pages have no
 * counterpart: they describe no memory management interface).
 *
 * For callers that cannot provide device scratch: ones with no device
 * allocator at hand, or that must not call one (cudaMalloc and cudaFree can
 * synchronise the whole device, and some runtimes forbid allocation after
 * start-up), and that do not keep the forward's checkpoints.  Same arguments
 * and results as ssm_selective_scan_bwd with ckpt = NULL, except that the
 * checkpoint scratch comes from a static device array of
 * SSM_NOALLOC_SCRATCH_BYTES inside the library, which every GPU that loads
 * the library holds until the process exits.
 *
 *  - Shapes whose scratch (ssm_selective_scan_bwd_scratch_bytes(shape, 0))
 *    exceeds SSM_NOALLOC_SCRATCH_BYTES are rejected with
 *    SSM_ERR_UNSUPPORTED before anything is launched.
 *  - Every call looks up the array's device address on the current device
 *    (a runtime query, no allocation); make the first call on a device
 *    before any stream capture, since that first query also loads the
 *    library's module on the device.
 *  - Every call on a device shares the one array and overwrites it: calls
 *    that overlap on the GPU (e.g. on two streams) race, so serialise them.
 *    Nothing of a previous call's contents is relied upon.
 *  - Calls no cudaMalloc, cudaFree or other allocating routine.
 */
#define SSM_NOALLOC_SCRATCH_BYTES (32u << 20)

ssm_status_t ssm_selective_scan_bwd_noalloc(const ssm_shape_t *shape,
                                            const void *u, const void *delta,
                                            const float *A, const void *B, const void *C,
                                            const float *D, const void *z,
                                            const float *delta_bias, int delta_softplus,
                                            const void *dout,
                                            float *du, float *ddelta, float *dA,
                                            float *dB, float *dC, float *dD, float *dz,
                                            float *ddelta_bias, void *stream);

/*
 * One step of the recurrence for decoding (the recurrent form of the
 * selective SSM: 정보관리기술사 학습 노트, "상태공간 모델(SSM)과 Mamba 아키텍처"
 * §2, with the selective Δ, B, C of booiljung.github.io §1.1).  For each
 * (b, d), in place:
 *   Δ = softplus(delta[b][d] + delta_bias[d])   (raw sum if delta_softplus == 0)
 *   state[b][d][n] = exp(Δ A[d][n]) state[b][d][n] + Δ B[b][n] u[b][d]
 *   y = Σ_n C[b][n] state[b][d][n] + D[d] u[b][d];  out[b][d] = y z σ(z)
 * This equals ssm_selective_scan_fwd over one step started from `state`.
 *
 *  shape        : seqlen must be 1; u, delta, z, out are [batch][dim] and
 *                 B, C are [batch][dstate], all in the io dtype.
 *  state        : [batch][dim][dstate] fp32, read and overwritten (caller
 *                 owned); 16-byte alignment of state, A, B and C enables
 *                 vector access but is not required.
 *  A, D, delta_bias, z : as in ssm_selective_scan_fwd (D, z, delta_bias
 *                 optional).
 *  out          : required, io dtype; may not alias the state or an input.
 * Asynchronous on `stream`; no device allocation.
 * Errors: SSM_ERR_INVALID_ARG (seqlen != 1, NULL or misaligned pointers,
 * host pointers, aliasing), SSM_ERR_UNSUPPORTED (dstate, batch > 65535),
 * SSM_ERR_CUDA.
 */
ssm_status_t ssm_selective_state_update(const ssm_shape_t *shape, float *state,
                                        const void *u, const void *delta,
                                        const float *A, const void *B, const void *C,
                                        const float *D, const void *z,
                                        const float *delta_bias, int delta_softplus,
                                        void *out, void *stream);

/*
 * ssm_selective_scan_bwd with options (see ssm_selective_scan_fwd_ex): the
 * adjoint of the forward with the same options.  With SSM_DISC_ZOH, du and
 * dB use the ZOH factor (Ā - 1)/A in place of Δ, the B term of dΔ carries
 * dB̄/dΔ = Ā B, and dA gains the derivative of (Ā - 1)/A with respect to A.
 */
ssm_status_t ssm_selective_scan_bwd_ex(const ssm_shape_t *shape, const ssm_options_t *opts,
                                       const void *u, const void *delta,
                                       const float *A, const void *B, const void *C,
                                       const float *D, const void *z,
                                       const float *delta_bias, const void *dout,
                                       const float *ckpt,
                                       float *du, float *ddelta, float *dA,
                                       float *dB, float *dC, float *dD, float *dz,
                                       float *ddelta_bias,
                                       void *scratch, size_t scratch_bytes, void *stream);

/* ssm_selective_state_update with options (see ssm_selective_scan_fwd_ex). */
ssm_status_t ssm_selective_state_update_ex(const ssm_shape_t *shape, const ssm_options_t *opts,
                                           float *state, const void *u, const void *delta,
                                           const float *A, const void *B, const void *C,
                                           const float *D, const void *z,
                                           const float *delta_bias, void *out, void *stream);

/*
 * Synchronises `stream`, then reports (and clears) the device-side error word
 * that kernels set when one of their bounded waits gives up: SSM_OK if none
 * did since the previous call, SSM_ERR_TIMEOUT otherwise.  Kernel waits are
 * on shared-memory barriers that complete asynchronous copies, each limited
 * to about 2 s of clock cycles, so a fault in the copy engine surfaces here
 * instead of hanging the stream.
 */
ssm_status_t ssm_device_error_status(void *stream);

/* The same check under the name of the boundary's original plan; identical
 * to ssm_device_error_status. */
ssm_status_t ssm_check_device_errors(void *stream);

/*
 * Diagnostic: launches on `stream` a one-warp kernel whose bounded wait (on a
 * shared-memory barrier that nothing completes) gives up after about 1 ms of
 * SM clock and sets the device error word, exactly as a stalled copy would.
 * The next ssm_device_error_status then returns SSM_ERR_TIMEOUT (and clears
 * the word).  Nothing faults or hangs; the stream stays usable.  The pages
 * have no counterpart: this exists to test the library's failure reporting.
 */
ssm_status_t ssm_selftest_wait_timeout(void *stream);

/*
 * Forward over one SEGMENT of a longer sequence (sequence sharding).
 *
 * The same forward as ssm_selective_scan_fwd_ex, over seqlen steps of a
 * segment, started from the state h0 ([batch][dim][dstate] float32, the state
 * after the previous segment's last step; NULL means zeros, as at the start of
 * a sequence).  last_state receives the state after the segment's last step.
 * delta_sum (nullable, [batch][dim] float32) receives Σ_t Δ_t over the
 * segment, with Δ exactly as the scan forms it (softplus of delta + bias when
 * enabled).
 *
 * A sequence cut into segments 0..S-1 is reassembled with the associative
 * operator of the two-level scan (booiljung.github.io, "3.2 선택적 스캔
 * (Selective Scan) 알고리즘과 정보의 압축 및 선별", §2.2):
 *   1. run every segment from h0 = NULL, keeping last_state (e_s) and
 *      delta_sum (Σ_s);
 *   2. ssm_scan_combine_carries turns (Σ_s, e_s) into the state entering each
 *      segment;
 *   3. run segments 1..S-1 again from those states; their out and last_state
 *      then equal the forward over the whole sequence.
 * Segment 0's first run is already final.  The checkpoints written from
 * h0 != NULL are the states of that run; the backward entry points assume a
 * zero initial state and must not be given them.
 * Errors: as ssm_selective_scan_fwd_ex; h0 may not alias last_state or ckpt.
 */
ssm_status_t ssm_selective_scan_fwd_segment(const ssm_shape_t *shape, const ssm_options_t *opts,
                                            const void *u, const void *delta, const float *A,
                                            const void *B, const void *C, const float *D,
                                            const void *z, const float *delta_bias, const float *h0,
                                            void *out, float *last_state, float *ckpt,
                                            float *delta_sum, void *stream);

/*
 * Exclusive scan of segment summaries, in sequence order, for S = nseg
 * segments of one sequence batch ([batch][dim] channel rows, dstate states):
 *   h_in[0] = h0 (zeros if NULL)
 *   h_in[s+1][r][n] = exp(A[r % dim][n] · delta_sums[s][r]) · h_in[s][r][n]
 *                     + h_ends[s][r][n]
 * exp(A Σ_t Δ_t) is the product of the segment's per-step factors exp(Δ_t A).
 * Layouts (float32, device): A [dim][dstate], delta_sums [nseg][batch][dim],
 * h_ends and h_in [nseg][batch][dim][dstate], h0 [batch][dim][dstate].
 * One thread per (row, state); asynchronous on `stream`.
 * Errors: SSM_ERR_INVALID_ARG (sizes < 1, NULL/host/misaligned pointers,
 * h_in aliasing an input), SSM_ERR_CUDA.
 */
ssm_status_t ssm_scan_combine_carries(int nseg, int batch, int dim, int dstate, const float *A,
                                      const float *delta_sums, const float *h_ends,
                                      const float *h0, float *h_in, void *stream);

/*
 * Selection projections: the per-token Linear layers that make the scan's
 * step size, B and C functions of its input x (= u of the scan).
 * booiljung.github.io, "3.2 선택적 스캔(Selective Scan) 알고리즘과 정보의 압축
 * 및 선별", §1.2: B_t = Linear_N(x_t), C_t = Linear_N(x_t),
 * Δ_t = Softplus(Parameter + Linear_1(x_t)); honbul.tistory.com, "Mamba" §2
 * (s_B, s_C, s_Δ).  The step-size projection is taken as the rank-R
 * factorisation Linear_D(Linear_R(x)); the pages' broadcast Linear_1 is
 * R = 1 with an all-ones up-projection, which this call expresses with
 * dt_rank = 8 and zero weights in the seven extra rows and columns.  The
 * Parameter (delta_bias) and the softplus are applied by the scan.
 *
 * For every batch row b and step t, with M1 = dt_rank + 2 * dstate:
 *   xdbl_t  = W_x · x[b, :, t]                 (M1 values, fp32 accumulation)
 *   dt_low[b, r, t] = xdbl_t[r]                r < dt_rank
 *   B[b, n, t]      = xdbl_t[dt_rank + n]
 *   C[b, n, t]      = xdbl_t[dt_rank + dstate + n]
 *   delta[b, d, t]  = Σ_r W_dt[d, r] dt_low[b, r, t]   (on the bf16-stored dt_low)
 * Every output is rounded to bfloat16 (nearest even) from fp32.
 *
 * Layouts (row-major, all bfloat16, all device memory owned by the caller):
 *   x       [batch][dim][seqlen]          W_x   [M1][dim]
 *   W_dt    [dim][dt_rank]                dt_low [batch][dt_rank][seqlen]
 *   delta   [batch][dim][seqlen]          B, C  [batch][dstate][seqlen]
 * B, C and delta are exactly the scan's inputs of the same names; dt_low is
 * an intermediate the caller provides the memory for.  Outputs must not
 * overlap the inputs or each other.
 *
 * Requirements: every pointer 16-byte aligned; seqlen, dim and dt_rank
 * multiples of 8; 1 <= dstate <= 64; batch <= 65535; io_dtype SSM_BF16
 * (shape->dstate and shape->io_dtype are read from `shape`, `dt_rank` is
 * separate).  Runs on the tensor cores (tcgen05, fp32 accumulators in tensor
 * memory) as two launches on `stream`.
 * Errors: SSM_ERR_INVALID_ARG (NULL, misaligned, host or overlapping
 * pointers, sizes not multiples of 8), SSM_ERR_UNSUPPORTED (io dtype, dstate,
 * batch, no tensor-map support in the driver), SSM_ERR_CUDA.
 */
ssm_status_t ssm_selection_projections(const ssm_shape_t *shape, int dt_rank,
                                       const void *x, const void *W_x, const void *W_dt,
                                       void *dt_low, void *delta, void *B, void *C,
                                       void *stream);

#ifdef __cplusplus
}
#endif

#endif /* SSM_SCAN_H */
