/*
 * sp_region.h -- C ABI of the B200 (sm_100a) sequence-parallel boundary.
 *
 * The boundary sits where a tensor-parallel (TP) region hands its output to a
 * sequence-parallel (SP) region and back:
 *
 *   t partial sums of a row-parallel linear
 *     -> reduce-scatter along the sequence (each rank keeps s/t tokens)
 *     -> + bias -> dropout -> + residual -> LayerNorm / RMSNorm
 *     -> all-gather back to the full [s, b, h] input of the next
 *        column-parallel linear
 *
 * and its backward, in which the all-gather and the reduce-scatter swap
 * places.  Sources (web pages on Megatron sequence parallelism):
 *   "Sequence Parallelism math" (aicassindra.com transformer-math), sections
 *     "The move", "The collective substitution", "Why the byte count is
 *     identical" and equations A_layer, A_TP, A_TP+SP;
 *   "SP: Partition Activations Alongside TP" (llm-systems-engineering),
 *     sections "Normalize and add residuals by token", "Change layouts
 *     between SP and TP", "Connect SP and TP across a layer";
 *   "TP and SP explained with pictures" (medium), section "Add Sequence
 *     parallelism".
 *
 * On one GPU the t ranks are emulated: rank k's partial sum is its own
 * buffer in the same HBM, and rank r's token shard is rows
 * [r*N/t, (r+1)*N/t) of the [s, b, h] tensors (N = s*b).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Layout      [s, b, h] with h fastest, stored as N = s*b token rows of h
 *             elements; token row n = s_idx*b + b_idx.  Rank r owns rows
 *             [r*N/t, (r+1)*N/t), which is contiguous because the shard is
 *             along s, the outermost dimension.
 * Dtypes      cfg->dtype applies to partial sums, residual, gamma, beta,
 *             bias and every [s,b,h] output, except that with cfg->res_f32
 *             the residual stream's tensors (residual, residual_out, the
 *             entry's x, dR_next, dresidual_in) are fp32; mean, rstd and the parameter
 *             gradients are always fp32.  Arithmetic is fp32.
 * Memory      every pointer argument named "device" is a CUDA device
 *             pointer on the current device; arrays of pointers
 *             (partials, gathered, dn_partials, shards, outs) are HOST arrays
 *             of device pointers.  The caller owns every buffer; the library
 *             allocates nothing.
 * Execution   device work is enqueued on `stream` (a cudaStream_t passed as
 *             void*; NULL is the legacy default stream) and is asynchronous.
 *             No call synchronises.  The return value reports argument
 *             validation and launch only.
 * Errors      a call that returns anything but SP_OK enqueued nothing.
 *             Arguments are validated before any launch: NULL required
 *             pointers, s % t != 0, t outside [1, SP_MAX_T], h < 1,
 *             p_drop outside [0, 1), eps <= 0 or not finite, unknown dtype
 *             or norm codes, and s*b or h beyond the 32-bit Philox counter
 *             give SP_ERR_INVALID_ARG.  A failed launch gives SP_ERR_CUDA.
 *             Device-side waits are bounded in time; a wait that runs out
 *             records a code that sp_device_error() reports, and the kernel
 *             returns instead of hanging.
 * Alignment   the fast kernels need 16-byte aligned [s,b,h] pointers and
 *             h*elem_bytes a multiple of 16; other shapes take a slower
 *             general kernel with the same results.  Nothing is rejected for
 *             alignment except pointers not aligned to their element size.
 */
#ifndef SP_REGION_H
#define SP_REGION_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SP_MAX_T 64

typedef enum {
    SP_OK = 0,
    SP_ERR_INVALID_ARG = 1,
    SP_ERR_UNSUPPORTED = 2,
    SP_ERR_CUDA = 3,
    SP_ERR_DEVICE_TIMEOUT = 4
} sp_status;

typedef enum { SP_F32 = 0, SP_BF16 = 1 } sp_dtype;
typedef enum { SP_LAYERNORM = 0, SP_RMSNORM = 1 } sp_norm;

/* Problem description.
 *   s, b, h  sequence length, micro-batch, hidden size
 *   t        tensor/sequence-parallel degree (number of emulated ranks)
 *   dtype    sp_dtype of the I/O tensors
 *   norm     sp_norm
 *   eps      added to the variance (LayerNorm) or the mean square (RMSNorm)
 *            inside the square root
 *   p_drop   dropout probability in [0, 1)
 *   seed, offset   Philox4x32-10 key and counter offset of the dropout mask
 *   fwd_plan, bwd_plan   kernel configuration hints, no counterpart on the
 *            pages: 0 lets the library choose; k > 0 asks for fast-kernel
 *            plan k-1 of the forward / backward plan tables (vectors per
 *            thread, consumer groups per CTA, block size) when that plan
 *            fits the shape, else the library chooses.  Results do not
 *            depend on the plan except through the fp32 summation order of
 *            the backward's parameter gradients.  Out-of-range values are
 *            treated as 0.
 *   row_begin, row_end   the global token rows [row_begin, row_end) this
 *            call processes; 0, 0 means all N rows.  With t GPUs as t real
 *            ranks, rank r passes its own shard [r*N/t, (r+1)*N/t) (its
 *            residual, stored outputs, mask and statistics hold only those
 *            rows, indexed from 0) while partials, gathered outputs and dY
 *            are full [s,b,h] tensors indexed by global row -- on a real
 *            system, peers' buffers reached through peer pointers.  The
 *            dropout counter uses the global row, so a split into ranges
 *            gives exactly the rows of the whole call.  Parameter gradients
 *            of a range cover its rows only; summing them over the ranges
 *            (the all-reduce of replicated parameters) gives the total.
 *   res_f32  0: the residual stream has the I/O dtype.  1 (with dtype
 *            SP_BF16): the residual stream is fp32 -- residual, residual_out
 *            and the entry's x, and in the backward residual_out (x),
 *            dR_next and dresidual_in -- while partials, bias, gamma, beta,
 *            gathered outputs and dY stay bf16.  The pages fix no precision
 *            for the residual ("SP: Partition Activations Alongside TP",
 *            section "Normalize and add residuals by token"); a
 *            mixed-precision layer keeps it in fp32.  The residual sum is
 *            then stored exactly as computed in fp32 and the norm reads it.
 *            Ignored for SP_F32.  Other values: SP_ERR_INVALID_ARG. */
typedef struct {
    int64_t s, b, h;
    int32_t t;
    int32_t dtype;
    int32_t norm;
    float eps;
    float p_drop;
    uint64_t seed, offset;
    int32_t fwd_plan, bwd_plan;
    int64_t row_begin, row_end;
    int32_t res_f32;
} sp_cfg;

/* Number of fast-kernel plans of the forward and the backward (valid hint
 * values are 1 .. count). */
int sp_plan_count(int32_t* fwd_plans, int32_t* bwd_plans);

/*
 * Forward of the boundary: reduce-scatter + bias + dropout + residual add +
 * norm, with the all-gather fused into the output write.
 *
 * Defined by: "Sequence Parallelism math", section "The collective
 * substitution" (leaving a TP region the all-reduce becomes a reduce-scatter
 * that sums the partials and scatters sequence shards; entering the next, an
 * all-gather); section "The move" (LayerNorm per token, dropout elementwise);
 * "SP: Partition Activations Alongside TP", sections "Normalize and add
 * residuals by token" and "Connect SP and TP across a layer" (residual add in
 * the token layout, its result is what the norm consumes).
 *
 * For every token row n (rank r = n / (N/t) owns it):
 *   y       = sum_{k=0..t-1} partials[k][n, :]      fp32, k ascending
 *   y      += bias                                   (once, if bias != NULL)
 *   z       = keep(n, j) ? y / (1 - p_drop) : 0      inverted dropout
 *   r_out   = round(residual[n, :] + z)              stored in the residual
 *                                                    stream's dtype (res_f32)
 *   LN:  o  = (r_out - mean) * rstd * gamma + beta,
 *        mean, var = mean and biased variance of r_out over h,
 *        rstd = 1 / sqrt(var + eps)
 *   RMS: o  = r_out * rstd * gamma, rstd = 1 / sqrt(mean(r_out^2) + eps)
 *   gathered[q][n, :] = round(o) for every q < n_gathered   (all-gather)
 * keep(n, j): Philox4x32-10 with key (seed lo, seed hi) and counter
 * (j >> 2, n, offset lo, offset hi); word j & 3 is compared with
 * floor(p_drop * 2^32) and the element is dropped iff it is smaller.  n is
 * the global row, so results do not depend on t.
 *
 * Arguments (device unless stated):
 *   partials     HOST array of t device pointers, each [s,b,h]
 *   bias         [h] or NULL
 *   residual     [s,b,h] (fp32 with cfg->res_f32)
 *   gamma        [h]
 *   beta         [h] or NULL (LayerNorm without shift; ignored for RMSNorm)
 *   residual_out [s,b,h] (fp32 with cfg->res_f32), may alias residual (in-place update)
 *   gathered     HOST array of n_gathered device pointers, each [s,b,h]; on
 *                one GPU the shard-major norm output is already the gathered
 *                tensor, so n_gathered = 1 is the plain case and n_gathered
 *                = t writes per-rank replicas.  Must not alias the inputs.
 *   n_gathered   1 .. SP_MAX_T
 *   mask_bits    [N][ceil(h/32)] uint32 or NULL: bit j&31 of word
 *                n*ceil(h/32) + (j>>5) is 1 iff element j was kept; padding
 *                bits are 0.  With p_drop = 0 every valid bit is 1.
 *   mean, rstd   [N] fp32 or NULL (mean is not written for RMSNorm)
 *   stream       cudaStream_t
 */
int sp_rs_bias_dropout_add_norm_fwd(const sp_cfg* cfg,
                                    const void* const* partials,
                                    const void* bias, const void* residual,
                                    const void* gamma, const void* beta,
                                    void* residual_out,
                                    void* const* gathered, int32_t n_gathered,
                                    uint32_t* mask_bits, float* mean,
                                    float* rstd, void* stream);

/*
 * Entry into a tensor-parallel region: per-token norm of the caller's shard,
 * then the all-gather into the full [s,b,h] input of the column-parallel
 * linear.
 *
 * Defined by: "SP: Partition Activations Alongside TP", section "Connect SP
 * and TP across a layer" (in a pre-norm layer each GPU first normalizes its
 * own tokens, then the all-gather combines the inputs of the QKV / first FFN
 * projection); "TP and SP explained with pictures", section "Add Sequence
 * parallelism" (apply LayerNorm locally, then all-gather).
 *
 * For every token row n of the call (cfg->row_begin/row_end, default all):
 *   LN:  o = (x - mean) * rstd * gamma + beta   RMS: o = x * rstd * gamma
 *   gathered[q][n, :] = round(o) for every q < n_gathered
 * cfg->p_drop is ignored (no dropout here); nothing is reduced.
 *
 * Arguments (device unless stated):
 *   x          [s,b,h] (the caller's shard when a row range is given;
 *              fp32 with cfg->res_f32)
 *   gamma      [h];  beta [h] or NULL (ignored for RMSNorm)
 *   gathered   HOST array of n_gathered device pointers, each [s,b,h],
 *              indexed by global row
 *   mean, rstd [rows of the call] fp32 or NULL (mean not written for RMS)
 * Its backward is sp_rs_norm_dropout_bwd with p_drop = 0, mask_bits = NULL,
 * dY = NULL and dbias = NULL: the reduce-scatter of the upstream gradient
 * partials, then the norm backward (plus dR_next) into dresidual_in.
 */
int sp_norm_all_gather_fwd(const sp_cfg* cfg, const void* x, const void* gamma,
                           const void* beta, void* const* gathered,
                           int32_t n_gathered, float* mean, float* rstd,
                           void* stream);

/*
 * All-gather of t sequence shards into n_out full [s,b,h] tensors.
 *
 * Defined by: "SP: Partition Activations Alongside TP", section "Change
 * layouts between SP and TP" (the token shards of the SP region combine into
 * the same input X on every GPU); "Sequence Parallelism math", section "The
 * collective substitution".
 *
 *   shards  HOST array of t device pointers; shard r is [N/t, h] rows of
 *           rank r (they may be consecutive slices of one buffer)
 *   outs    HOST array of n_out device pointers, each [s,b,h]; out[q] rows
 *           [r*N/t, (r+1)*N/t) receive shard r.  Must not overlap shards.
 *   n_out   1 .. SP_MAX_T
 */
int sp_all_gather(const sp_cfg* cfg, const void* const* shards,
                  void* const* outs, int32_t n_out, void* stream);

/*
 * Backward of the boundary: reduce-scatter of the upstream gradient partials
 * + norm backward + residual-stream gradient + dropout backward, with the
 * all-gather of the gradient w.r.t. the partial sums fused into its write.
 *
 * Defined by: "Sequence Parallelism math", section "The collective
 * substitution" (the backward swaps all-gather and reduce-scatter, their
 * conjugates); the norm and dropout derivatives are the textbook ones.
 *
 * For every token row n:
 *   dn   = sum_k dn_partials[k][n, :]            (all-gather's backward)
 *   xhat = (x - mean) * rstd (LN) or x * rstd (RMS), x = residual_out
 *   g    = dn * gamma
 *   LN:  dx = rstd * (g - mean_j(g) - xhat * mean_j(g * xhat))
 *   RMS: dx = rstd * (g - xhat * mean_j(g * xhat))
 *   dr   = dx + dR_next (if given)
 *   dresidual_in[n, :] = round(dr)
 *   dz   = keep ? dr / (1 - p_drop) : 0,  keep read from mask_bits
 *   dY[n, :] = round(dz)                         (reduce-scatter's backward)
 *   dgamma += dn * xhat, dbeta += dn, dbias += dz   summed over all N rows
 *
 * Arguments (device unless stated):
 *   dn_partials  HOST array of t device pointers, each [s,b,h]
 *   dR_next      [s,b,h] or NULL (fp32 with cfg->res_f32)
 *   residual_out, mask_bits, mean, rstd   the forward's outputs (mask_bits
 *                may be NULL only when p_drop == 0; mean unused for RMS)
 *   gamma        [h]
 *   dresidual_in [s,b,h] (fp32 with cfg->res_f32, like residual_out);
 *                dY [s,b,h] or NULL (not written; the backward of
 *                the entry into a TP region has no dropout input)
 *   dgamma [h] fp32; dbeta [h] fp32 or NULL; dbias [h] fp32 or NULL
 *   workspace    device scratch of at least sp_bwd_workspace_bytes() bytes,
 *                16-byte aligned; no initial contents needed.  Calls that
 *                overlap on the GPU must not share a workspace.
 * The parameter gradients are deterministic: per-CTA partial sums in a
 * fixed order, then one fixed-order sum over CTAs.
 */
int sp_rs_norm_dropout_bwd(const sp_cfg* cfg, const void* const* dn_partials,
                           const void* dR_next, const void* residual_out,
                           const void* gamma, const uint32_t* mask_bits,
                           const float* mean, const float* rstd,
                           void* dresidual_in, void* dY, float* dgamma,
                           float* dbeta, float* dbias, void* workspace,
                           size_t workspace_bytes, void* stream);

/*
 * Row-parallel linear with the reduce-scatter fused into its epilogue.
 *
 * Defined by: "TP and SP explained with pictures", sections "Tensor
 * parallelism, take two: split the inner dimension" (each rank computes a
 * full-shape partial sum from its slice of the inner dimension; the partials
 * are summed across ranks) and "Add Sequence parallelism" (with SP that sum
 * is a reduce-scatter back to token shards, followed by the SP region);
 * "Chapter 6: TP and SP", section 3 (Row Parallel Linear: Y_i = X_i A_i).
 *
 * x [rows][f] bf16 holds, for this call's token rows, the row-parallel
 * input; rank k's slice is columns [k*f/t, (k+1)*f/t).  w [h][f] bf16 is the
 * weight in output-by-input layout; rank k's rows of the weight are its
 * columns [k*f/t, (k+1)*f/t).  For every row n of the call:
 *   y[n, j] = sum_{k=0..t-1} sum_{i in slice k} x[n, i] * w[j, i]
 *           (the t partials are summed in one fp32 accumulator in tensor
 *            memory, slice by slice; no partial is ever stored)
 *   then bias, inverted dropout (the forward's Philox mask) and the residual
 *   add exactly as sp_rs_bias_dropout_add_norm_fwd: residual_out = round(
 *   residual + dropout(y + bias)), mask_bits as there.
 * The norm and the all-gather follow in sp_linear_rs_bias_dropout_add_norm_fwd.
 *
 * Requirements: cfg->dtype SP_BF16 and res_f32 = 0 (else SP_ERR_UNSUPPORTED);
 * f % t == 0 (else SP_ERR_INVALID_ARG); f and h multiples of 8 (else
 * SP_ERR_UNSUPPORTED); x, w, bias, residual, residual_out 16-byte aligned.
 * The row range of cfg selects the call's rows: x, residual, residual_out
 * and mask_bits are indexed by local row, the dropout counter by global row.
 */
int sp_rowpar_linear_rs_fwd(const sp_cfg* cfg, int64_t f, const void* x, const void* w,
                            const void* bias, const void* residual, void* residual_out,
                            uint32_t* mask_bits, void* stream);

/*
 * The forward boundary with its reduce-scatter inside the row-parallel GEMM:
 * sp_rowpar_linear_rs_fwd, then the per-token norm of residual_out and the
 * all-gather of the result into `gathered` (the same kernel as
 * sp_norm_all_gather_fwd).  Outputs and their layouts are those of
 * sp_rs_bias_dropout_add_norm_fwd; the t partials of that call are replaced
 * by x and w.  Two launches on `stream`.
 */
int sp_linear_rs_bias_dropout_add_norm_fwd(const sp_cfg* cfg, int64_t f, const void* x,
                                           const void* w, const void* bias,
                                           const void* residual, const void* gamma,
                                           const void* beta, void* residual_out,
                                           void* const* gathered, int32_t n_gathered,
                                           uint32_t* mask_bits, float* mean, float* rstd,
                                           void* stream);

/*
 * Column-parallel linear with the all-gather fused into its prologue.
 *
 * Defined by: "TP and SP explained with pictures", sections "Tensor
 * parallelism, take one: split the output dimension" (every rank multiplies
 * the full input by its slice of the weight's output columns) and "Add
 * Sequence parallelism" (with SP the full input is all-gathered from the
 * sequence shards first); "Chapter 6: TP and SP", section 2.
 *
 *   out[n, o] = round( sum_i X[n, i] * w[o, i] ),  X = concat_r shards[r]
 * shards: HOST array of t device pointers, shard r = rows [r*N/t, (r+1)*N/t)
 * of the SP region's output, [N/t][h] bf16 each; the GEMM reads its A tiles
 * straight from the shards, so no gathered copy is made.  w [f_out][h] bf16
 * (output-by-input); out [N][f_out] bf16.  fp32 accumulation in tensor
 * memory, one rounding.
 *
 * Requirements: SP_BF16; t <= 16 and (t == 1 or (N/t) % 128 == 0); h and
 * f_out multiples of 8 (else SP_ERR_UNSUPPORTED); no row range (else
 * SP_ERR_INVALID_ARG); 16-byte aligned pointers.
 */
int sp_ag_colpar_linear_fwd(const sp_cfg* cfg, int64_t f_out, const void* const* shards,
                            const void* w, void* out, void* stream);

/*
 * The backward with dY written to n_dY full buffers: each row of the
 * dropout gradient goes to every buffer, as the forward writes its
 * normalised rows to every gathered buffer.  With t real ranks, rank r runs
 * its row range (cfg->row_begin/row_end) and passes the t ranks' dY buffers
 * (peers' through peer pointers): the all-gather of dY, the reduce-scatter's
 * backward ("Sequence Parallelism math", section "The collective
 * substitution"), is then done by the kernels' own stores, and every rank's
 * copy is complete once every rank's call has finished.  Arguments are
 * those of sp_rs_norm_dropout_bwd with dY replaced by a HOST array of n_dY
 * (1 .. SP_MAX_T) device pointers, each [s,b,h] indexed by global row.
 */
int sp_rs_norm_dropout_bwd_ag(const sp_cfg* cfg, const void* const* dn_partials,
                              const void* dR_next, const void* residual_out,
                              const void* gamma, const uint32_t* mask_bits,
                              const float* mean, const float* rstd, void* dresidual_in,
                              void* const* dY, int32_t n_dY, float* dgamma, float* dbeta,
                              float* dbias, void* workspace, size_t workspace_bytes,
                              void* stream);

/*
 * Ring attention (context parallelism) over t ranks, forward.
 *
 * Defined by: "Sequence Parallelism math", sections "Where SP stops: the
 * attention core and long sequences" and "Context parallelism and ring
 * attention": Q, K and V are sharded along the sequence, rank r holding the
 * contiguous block r of s/t tokens; at step i rank r attends its queries
 * against K/V block (r - i) mod t and folds the scores into an online
 * softmax (running maximum m, sum l of exp(score - m), weighted values o),
 * so after t steps every query has seen every key.
 *
 * For every batch b, head, and query n (its rank r = n / (s/t)):
 *   score(n, j) = scale * sum_c q[n, c] * k[j, c]   over all s keys j,
 *   visited block by block in ring order (block r first), 128 keys a tile
 *   out[n, :] = round( sum_j exp(score(n, j) - m) v[j, :] / l )
 *   lse[n]    = m + log(l)  (natural log; NULL: not written)
 * Attention is full (every query sees every key), as on the page.
 *
 * cfg: s = sequence length, b = batch, t = ranks of the ring, dtype SP_BF16,
 * h = heads * 128 (head dimension 128), no row range.  q, k, v, out:
 * [b][heads][s][128] bf16, 16-byte aligned; lse [b][heads][s] fp32 or NULL.
 * Requirements: s % 128 == 0 and (s / t) % 128 == 0, b * heads * s < 2^31
 * (else SP_ERR_UNSUPPORTED); scale > 0 (else SP_ERR_INVALID_ARG).  The
 * probabilities enter the second product as bf16; both products accumulate
 * in fp32 in tensor memory.
 */
int sp_ring_attention_fwd(const sp_cfg* cfg, int32_t heads, float scale, const void* q,
                          const void* k, const void* v, void* out, float* lse,
                          void* stream);

/*
 * The same ring attention, with scratch for balancing the last round of work.
 *
 * Same definition, arguments and requirements as sp_ring_attention_fwd, plus
 * a workspace.  One CTA takes a unit (one or two 128-query tiles of one
 * head) through every ring step, and the GPU runs one CTA per SM.  When the
 * units do not fill the last round of SMs, the call cuts each unit of that
 * round into up to 8 contiguous ranges of ring steps (at least 4 key tiles
 * each). Each range keeps its own online-softmax state (m_i, l_i, o_i), as a
 * rank does between ring steps. A second kernel then combines the ranges
 * of every such query in range order:
 *   m = max m_i,  l = sum exp(m_i - m) l_i,  out = sum exp(m_i - m) o_i / l
 * which is the online-softmax update of the page applied once per range.
 * The order of the additions differs from the unsplit call, so results agree
 * with it to rounding, not bit for bit; repeated calls with the same shape on
 * the same GPU give the same bits.
 *
 *   workspace        device scratch of at least
 *                    sp_ring_attention_workspace_bytes() bytes, 16-byte
 *                    aligned, no initial contents; may be NULL when that
 *                    size is 0.  Calls that overlap on the GPU must not
 *                    share a workspace.
 * SP_ERR_INVALID_ARG when the workspace is missing or too small.
 */
int sp_ring_attention_fwd_ws(const sp_cfg* cfg, int32_t heads, float scale, const void* q,
                             const void* k, const void* v, void* out, float* lse,
                             void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of device scratch sp_ring_attention_fwd_ws needs for cfg and heads
 * on CUDA device `device` (its SM count sets the split): 0 when the units
 * fill whole rounds.  Host-only.  The errors of sp_ring_attention_fwd's
 * shape checks; SP_ERR_INVALID_ARG for bytes == NULL. */
int sp_ring_attention_workspace_bytes(const sp_cfg* cfg, int32_t heads, int32_t device,
                                      size_t* bytes);

/* Bytes of device scratch sp_rs_norm_dropout_bwd needs for cfg on CUDA
 * device `device`: the slices of 3*h fp32 parameter-gradient partial sums
 * that the kernel the call picks writes, for 16-byte aligned pointers or for
 * misaligned ones (the general kernel), whichever is more.  With the
 * library's own plan choice that is one slice per CTA, min(s*b, SMs) slices
 * (one per SM at most); a plan hint (cfg->bwd_plan) may pick a plan with
 * one slice per consumer group (up to 4 per CTA).  Host-only; it reads the
 * device's SM count and shared-memory limit.  SP_ERR_UNSUPPORTED when no
 * backward kernel takes the shape.  Departs from a plain size_t return so
 * that it can report errors like every other call. */
int sp_bwd_workspace_bytes(const sp_cfg* cfg, int32_t device, size_t* bytes);

/*
 * Activation memory of one transformer layer per device, host-only.
 *
 * Defined by: "Sequence Parallelism math", equation A_layer (section "The
 * problem: activation memory") and equations A_TP and A_TP+SP (section "The
 * activation-memory saving"); "TP and SP explained with pictures" and the
 * anthology record summarise the same accounting.
 *   mode 0: A_layer  = s*b*h * (34 + 5*a*s/h)
 *   mode 1: A_TP     = s*b*h * (10 + 24/t + 5*a*s/(h*t))
 *   mode 2: A_TP+SP  = (s*b*h / t) * (34 + 5*a*s/h)
 * *out = coefficient * s*b*h * bytes_per_elem (the page's worked example
 * multiplies by 2 bytes for fp16).  SP_ERR_INVALID_ARG for non-positive
 * sizes, an unknown mode or out == NULL.
 */
int sp_activation_bytes(int64_t s, int64_t b, int64_t h, int64_t a,
                        int32_t t, int32_t mode, double bytes_per_elem,
                        double* out);

/* Static text for a status code. */
const char* sp_status_string(int status);

/* Reads the device-side error word of CUDA device `device` (0: none; else
 * the code of the first bounded wait that ran out: 1 a consumer waiting for a
 * staged row, 2 the producer waiting for a free stage, 3 an aborted CTA
 * draining its copies, 9 the diagnostic below) and clears it when
 * clear != 0.  Synchronises the device.  No counterpart on the pages: this
 * is the library's failure detection. */
int sp_device_error(int32_t device, int32_t* code, int32_t clear);

/* Failure-detection diagnostic, no counterpart on the pages: launches one
 * CTA that waits on an mbarrier nothing will complete, through the same
 * bounded wait the streaming kernels use, with a limit of limit_ns
 * (0 .. 10^10).  The wait must run out: the kernel writes *status = 1 (a
 * device int32) and records code 9, and the context stays usable.  *status
 * = 0 would mean the wait completed. */
int sp_debug_wait_timeout(int64_t limit_ns, int32_t* status, void* stream);

/*
 * Backward without caller-provided scratch: sp_rs_norm_dropout_bwd with the
 * workspace taken from a fixed array inside the library.  The pages have no
 * counterpart; this exists for callers that cannot allocate device memory
 * where they run the backward (a memory-capped arena that owns every byte, an
 * allocator that must not be re-entered from here, or a loop that may not
 * synchronise, since cudaMalloc and cudaFree can).
 *
 * Arguments, layout and results are those of sp_rs_norm_dropout_bwd without
 * `workspace` / `workspace_bytes`.  The call allocates nothing: the scratch
 * is a 64 MiB array of this library's device image, reserved on every GPU
 * that loads the library and held until the process exits.
 *
 * Limit   the call picks its kernel for the given pointers exactly as
 *         sp_rs_norm_dropout_bwd does; if the scratch that kernel writes
 *         (its slices times 12*h bytes) exceeds 64 MiB, it returns
 *         SP_ERR_UNSUPPORTED before any launch.  With the library's own plan
 *         choice a call writes min(s*b, SMs) slices, so on a 148-SM B200
 *         every shape with h <= 37786 fits (the fast kernels take h up to
 *         16384 in bf16 and fp32; the general kernel up to about 57000).  A
 *         plan hint that picks one slice per consumer group divides the
 *         limit by the group count.
 * Set-up  every call looks up the array's device address on the current
 *         device (cudaGetSymbolAddress); the first call on a device also
 *         loads the library's device code there, so make it before any
 *         stream capture.
 * Sharing every call on a device uses the same array and leaves its
 *         contents behind; the kernels write every part of it they read, so
 *         nothing needs clearing, but calls that overlap on the GPU (other
 *         streams, other host threads) race on it and must be serialised by
 *         the caller.
 */
int sp_rs_norm_dropout_bwd_noalloc(const sp_cfg* cfg,
                                   const void* const* dn_partials,
                                   const void* dR_next,
                                   const void* residual_out,
                                   const void* gamma,
                                   const uint32_t* mask_bits,
                                   const float* mean, const float* rstd,
                                   void* dresidual_in, void* dY,
                                   float* dgamma, float* dbeta, float* dbias,
                                   void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SP_REGION_H */
