/*
 * CPU oracle for the Megatron sequence-parallel (SP) boundary.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, obviously correct
 * reference that the tests, the smoke check and the benchmark's CPU baseline
 * compare the CUDA path against.  Nothing in the product links it, calls it or
 * shares code with it.
 *
 * Arithmetic is scalar C in double precision.  Inputs arrive as the I/O dtype
 * (fp32 or bf16 bit patterns) and are widened exactly; every output that the
 * product stores in the I/O dtype is rounded here once, to nearest-even, at
 * the same point the method stores it.
 *
 * What it computes, and where each step comes from:
 *
 *   "Sequence Parallelism math" (aicassindra transformer-math page),
 *     section "The collective substitution": leaving a tensor-parallel region
 *     the all-reduce becomes a reduce-scatter that sums the t partial outputs
 *     and hands each rank only its sequence shard; entering the next one an
 *     all-gather assembles the full sequence.  The backward swaps the two.
 *   same page, section "The move": rank i owns tokens [i*s/t, (i+1)*s/t); the
 *     LayerNorm and the residual dropout act on each token independently.
 *   "SP: Partition Activations Alongside TP" (llm-systems-engineering),
 *     sections "Normalize and add residuals by token" and "Change layouts
 *     between SP and TP": whole token vectors stay on one GPU, the residual
 *     uses the same token layout, reduce-scatter completes each rank's tokens
 *     with the other ranks' contributions, all-gather rebuilds the input X of
 *     the column-parallel linear; RMSNorm is the scale-only norm.
 *   same page, section "Connect SP and TP across a layer": the residual add
 *     produces the tensor that the following norm consumes (pre-norm layer).
 *   "Sequence Parallelism math", equations A_layer, A_TP and A_TP+SP:
 *     activation-memory closed forms.
 *
 * Readings where the pages are silent (stated once, used everywhere):
 *   - the bias of the row-parallel linear is added once, after the reduction;
 *   - dropout is inverted dropout: kept values are scaled by 1/(1-p);
 *   - the keep decision uses Philox4x32-10 (Salmon, Moraes, Dror, Shaw,
 *     "Parallel Random Numbers: As Easy as 1, 2, 3", SC'11) with
 *     key = (seed lo, seed hi), counter = (j>>2, n, offset lo, offset hi),
 *     output word j&3; an element is dropped iff that word is below
 *     floor(p * 2^32); n is the global token row so the mask does not depend
 *     on t;
 *   - the mask is bit-packed: bit j&31 of word n*W + (j>>5), W = ceil(h/32);
 *   - LayerNorm uses the biased variance and eps inside the square root;
 *     RMSNorm has no mean and no beta;
 *   - the norm reads the residual sum after it is rounded to the residual
 *     stream's dtype (that rounded tensor is what is stored for the
 *     backward);
 *   - the residual stream (residual in, the stored sum, the gradient arriving
 *     on it and the residual gradient out) has its own dtype, res_dtype: the
 *     I/O dtype, or fp32 beside bf16 partial sums, parameters and norm
 *     outputs (a mixed-precision layer keeps its residual stream in fp32).
 *
 * Parity pins for every function here live in the oracle tests; none of the
 * functions is unpinned.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_F32 0
#define ORC_BF16 1
#define ORC_LAYERNORM 0
#define ORC_RMSNORM 1

typedef struct {
    int64_t s, b, h;
    int32_t t;
    int32_t dtype;   /* ORC_F32 or ORC_BF16 */
    int32_t norm;    /* ORC_LAYERNORM or ORC_RMSNORM */
    float eps;
    float p_drop;
    uint64_t seed, offset;
    int32_t res_dtype;   /* dtype of the residual stream tensors */
} orc_cfg;

/* ------------------------------------------------------------------------- */
/* Philox4x32-10, from the SC'11 paper's definition.                          */
/* One round maps (x0,x1,x2,x3) with round key (k0,k1) to                    */
/*   (hi(M1*x2) ^ x1 ^ k0, lo(M1*x2), hi(M0*x0) ^ x3 ^ k1, lo(M0*x0));       */
/* the key is bumped by the Weyl constants between rounds.                    */
/* ------------------------------------------------------------------------- */
#define PHILOX_M0 0xD2511F53u
#define PHILOX_M1 0xCD9E8D57u
#define PHILOX_W0 0x9E3779B9u
#define PHILOX_W1 0xBB67AE85u

void orc_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2],
                       uint32_t out[4])
{
    uint32_t x0 = ctr_in[0], x1 = ctr_in[1], x2 = ctr_in[2], x3 = ctr_in[3];
    uint32_t k0 = key_in[0], k1 = key_in[1];
    for (int round = 0; round < 10; ++round) {
        if (round > 0) {
            k0 += PHILOX_W0;
            k1 += PHILOX_W1;
        }
        uint64_t p0 = (uint64_t)PHILOX_M0 * (uint64_t)x0;
        uint64_t p1 = (uint64_t)PHILOX_M1 * (uint64_t)x2;
        uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        uint32_t y0 = hi1 ^ x1 ^ k0;
        uint32_t y1 = lo1;
        uint32_t y2 = hi0 ^ x3 ^ k1;
        uint32_t y3 = lo0;
        x0 = y0; x1 = y1; x2 = y2; x3 = y3;
    }
    out[0] = x0; out[1] = x1; out[2] = x2; out[3] = x3;
}

/* ------------------------------------------------------------------------- */
/* Rounding to the I/O dtype, from the definition of a binary floating-point  */
/* format: keep `bits` significant bits, round to nearest with ties to even,  */
/* subnormal spacing below the smallest normal, overflow to infinity.         */
/* fp32: 24 bits, min normal 2^-126, max exponent 127; bf16: 8 bits, same     */
/* exponent range.                                                            */
/* ------------------------------------------------------------------------- */
static double round_format(double x, int bits)
{
    if (x != x || x == 0.0 || isinf(x)) return x;
    int e;
    (void)frexp(x, &e);                 /* x = m * 2^e, 0.5 <= |m| < 1 */
    int q = e - bits;                   /* spacing of the format at x */
    if (q < -126 - (bits - 1)) q = -126 - (bits - 1);   /* subnormal floor */
    double scaled = ldexp(x, -q);       /* exact: a power-of-two scale */
    double r = nearbyint(scaled);       /* default mode: to nearest, ties even */
    double y = ldexp(r, q);
    if (fabs(y) >= ldexp(1.0, 128)) return x > 0 ? INFINITY : -INFINITY;
    return y;
}

double orc_round(double x, int dtype)
{
    return round_format(x, dtype == ORC_BF16 ? 8 : 24);
}

/* exact widening of one stored element */
static double ld(const void* p, int64_t i, int dtype)
{
    if (dtype == ORC_F32) return (double)((const float*)p)[i];
    uint32_t bits = (uint32_t)((const uint16_t*)p)[i] << 16;
    float f;
    memcpy(&f, &bits, 4);
    return (double)f;
}

/* store a value rounded once to the I/O dtype */
static void st(void* p, int64_t i, int dtype, double v)
{
    double r = orc_round(v, dtype);
    float f = (float)r;                 /* exact: r is representable */
    if (dtype == ORC_F32) {
        ((float*)p)[i] = f;
    } else {
        uint32_t bits;
        memcpy(&bits, &f, 4);
        ((uint16_t*)p)[i] = (uint16_t)(bits >> 16);
    }
}

/* ------------------------------------------------------------------------- */
/* Dropout keep decision                                                      */
/* ------------------------------------------------------------------------- */
uint32_t orc_drop_threshold(float p)
{
    return (uint32_t)floor((double)p * 4294967296.0);
}

int orc_keep(uint64_t seed, uint64_t offset, int64_t n, int64_t j, float p)
{
    uint32_t ctr[4] = {(uint32_t)(j >> 2), (uint32_t)n, (uint32_t)offset,
                       (uint32_t)(offset >> 32)};
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t u[4];
    orc_philox4x32_10(ctr, key, u);
    return u[j & 3] >= orc_drop_threshold(p);
}

int64_t orc_mask_words(int64_t h) { return (h + 31) / 32; }

/* ------------------------------------------------------------------------- */
/* Collectives over t emulated ranks                                          */
/* ------------------------------------------------------------------------- */

/* all-reduce: every rank receives sum_k P_k (k ascending) */
void orc_all_reduce(int t, int64_t count, int dtype, const void* const* parts,
                    double* out)
{
    for (int64_t i = 0; i < count; ++i) {
        double acc = 0.0;
        for (int k = 0; k < t; ++k) acc += ld(parts[k], i, dtype);
        out[i] = acc;
    }
}

/* reduce-scatter along the sequence: rank r receives rows [r*R, (r+1)*R) of
 * sum_k P_k, R = rows/t, each row holding h features */
void orc_reduce_scatter(int t, int64_t rows, int64_t h, int dtype,
                        const void* const* parts, int rank, double* shard)
{
    int64_t per = rows / t;
    for (int64_t i = 0; i < per; ++i) {
        int64_t n = (int64_t)rank * per + i;
        for (int64_t j = 0; j < h; ++j) {
            double acc = 0.0;
            for (int k = 0; k < t; ++k) acc += ld(parts[k], n * h + j, dtype);
            shard[i * h + j] = acc;
        }
    }
}

/* all-gather along the sequence: the output is shard 0, then shard 1, ... */
void orc_all_gather(int t, int64_t shard_rows, int64_t h,
                    const double* const* shards, double* out)
{
    for (int r = 0; r < t; ++r)
        for (int64_t i = 0; i < shard_rows * h; ++i)
            out[(int64_t)r * shard_rows * h + i] = shards[r][i];
}

/* ------------------------------------------------------------------------- */
/* The SP region on one token row (forward)                                   */
/* ------------------------------------------------------------------------- */
static void region_row_fwd(const orc_cfg* c, int64_t n, const double* y,
                           const void* bias, const void* resid, int64_t rrow,
                           const void* gamma, const void* beta, void* rout,
                           double* o, uint32_t* mask_row, double* mean_out,
                           double* rstd_out, double* x)
{
    const int64_t h = c->h;
    const double scale = 1.0 / (1.0 - (double)c->p_drop);
    if (mask_row)
        for (int64_t w = 0; w < orc_mask_words(h); ++w) mask_row[w] = 0u;

    for (int64_t j = 0; j < h; ++j) {
        /* bias of the row-parallel linear, once, after the reduction */
        double v = y[j] + (bias ? ld(bias, j, c->dtype) : 0.0);
        /* residual dropout */
        int keep = orc_keep(c->seed, c->offset, n, j, c->p_drop);
        v = keep ? v * scale : 0.0;
        if (mask_row && keep) mask_row[j >> 5] |= 1u << (j & 31);
        /* residual add; the sum is stored in the residual stream's dtype */
        double r = orc_round(ld(resid, rrow * h + j, c->res_dtype) + v, c->res_dtype);
        st(rout, rrow * h + j, c->res_dtype, r);
        x[j] = r;
    }

    /* per-token norm over the h features of the stored residual sum */
    double mean = 0.0, var = 0.0, rstd;
    if (c->norm == ORC_LAYERNORM) {
        for (int64_t j = 0; j < h; ++j) mean += x[j];
        mean /= (double)h;
        for (int64_t j = 0; j < h; ++j) var += (x[j] - mean) * (x[j] - mean);
        var /= (double)h;
        rstd = 1.0 / sqrt(var + (double)c->eps);
        for (int64_t j = 0; j < h; ++j) {
            double b = beta ? ld(beta, j, c->dtype) : 0.0;
            o[j] = orc_round((x[j] - mean) * rstd * ld(gamma, j, c->dtype) + b,
                             c->dtype);
        }
    } else {
        double ms = 0.0;
        for (int64_t j = 0; j < h; ++j) ms += x[j] * x[j];
        ms /= (double)h;
        rstd = 1.0 / sqrt(ms + (double)c->eps);
        for (int64_t j = 0; j < h; ++j)
            o[j] = orc_round(x[j] * rstd * ld(gamma, j, c->dtype), c->dtype);
    }
    if (mean_out) *mean_out = mean;
    if (rstd_out) *rstd_out = rstd;
}

static int cfg_ok(const orc_cfg* c)
{
    if (c->s <= 0 || c->b <= 0 || c->h <= 0 || c->t <= 0) return 0;
    if (c->s % c->t) return 0;
    if (!(c->p_drop >= 0.0f && c->p_drop < 1.0f)) return 0;
    if (!(c->eps > 0.0f)) return 0;
    if (c->res_dtype != ORC_F32 && c->res_dtype != ORC_BF16) return 0;
    return 1;
}

/*
 * Forward of the whole boundary on t emulated ranks.
 *   parts[k]      rank k's partial output of the row-parallel linear, [s,b,h]
 *   residual      [s,b,h], rank r's shard is its rows
 *   residual_out  [s,b,h] (rank r writes its rows), residual stream dtype
 *   gathered      n_out buffers [s,b,h]: the all-gathered norm output
 *   mask          [s*b][W] u32 or NULL;  mean/rstd [s*b] (mean NULL for RMS)
 * Returns 0, or -1 for an invalid configuration.
 */
int orc_fwd(const orc_cfg* c, const void* const* parts, const void* bias,
            const void* residual, const void* gamma, const void* beta,
            void* residual_out, void* const* gathered, int n_out,
            uint32_t* mask, double* mean, double* rstd)
{
    if (!cfg_ok(c)) return -1;
    const int64_t N = c->s * c->b, h = c->h, per = N / c->t;
    const int64_t W = orc_mask_words(h);
    double* y = (double*)malloc(sizeof(double) * (size_t)(per * h));
    double* x = (double*)malloc(sizeof(double) * (size_t)h);
    double** shards = (double**)malloc(sizeof(double*) * (size_t)c->t);
    double* full = (double*)malloc(sizeof(double) * (size_t)(N * h));
    if (!y || !x || !shards || !full) {
        free(y); free(x); free(shards); free(full);
        return -2;
    }
    for (int r = 0; r < c->t; ++r) {
        /* reduce-scatter: rank r's rows, with every rank's contribution */
        orc_reduce_scatter(c->t, N, h, c->dtype, parts, r, y);
        shards[r] = full + (int64_t)r * per * h;   /* rank r's norm output */
        for (int64_t i = 0; i < per; ++i) {
            int64_t n = (int64_t)r * per + i;
            region_row_fwd(c, n, y + i * h, bias, residual, n, gamma, beta,
                           residual_out, shards[r] + i * h,
                           mask ? mask + n * W : NULL, mean ? mean + n : NULL,
                           rstd ? rstd + n : NULL, x);
        }
    }
    /* all-gather: every requested replica receives all shards, in order */
    double* g = (double*)malloc(sizeof(double) * (size_t)(N * h));
    if (!g) {
        free(y); free(x); free(shards); free(full);
        return -2;
    }
    orc_all_gather(c->t, per, h, (const double* const*)shards, g);
    for (int q = 0; q < n_out; ++q)
        for (int64_t i = 0; i < N * h; ++i) st(gathered[q], i, c->dtype, g[i]);
    free(g); free(y); free(x); free(shards); free(full);
    return 0;
}

/*
 * Forward on selected token rows only (the large workloads' sampled check).
 * A reduce-scatter result row is the all-reduced row ("all-reduce, then keep
 * your rows"), so row n needs only the t partial rows of token n.
 *   row_ids[i]    global token row of sample i
 *   parts[k]      [nrows, h] partial rows of rank k, residual [nrows, h]
 *   outputs       [nrows, ...] in the same sample order
 */
int orc_fwd_rows(const orc_cfg* c, int64_t nrows, const int64_t* row_ids,
                 const void* const* parts, const void* bias,
                 const void* residual, const void* gamma, const void* beta,
                 void* residual_out, void* norm_out, uint32_t* mask,
                 double* mean, double* rstd)
{
    if (!cfg_ok(c)) return -1;
    const int64_t h = c->h, W = orc_mask_words(h);
    double* y = (double*)malloc(sizeof(double) * (size_t)h);
    double* x = (double*)malloc(sizeof(double) * (size_t)h);
    double* o = (double*)malloc(sizeof(double) * (size_t)h);
    if (!y || !x || !o) { free(y); free(x); free(o); return -2; }
    for (int64_t i = 0; i < nrows; ++i) {
        for (int64_t j = 0; j < h; ++j) {
            double acc = 0.0;
            for (int k = 0; k < c->t; ++k) acc += ld(parts[k], i * h + j, c->dtype);
            y[j] = acc;
        }
        region_row_fwd(c, row_ids[i], y, bias, residual, i, gamma, beta,
                       residual_out, o, mask ? mask + i * W : NULL,
                       mean ? mean + i : NULL, rstd ? rstd + i : NULL, x);
        for (int64_t j = 0; j < h; ++j) st(norm_out, i * h + j, c->dtype, o[j]);
    }
    free(y); free(x); free(o);
    return 0;
}

/*
 * Entry into a tensor-parallel region ("SP: Partition Activations Alongside
 * TP", section "Connect SP and TP across a layer": each GPU first normalizes
 * its own tokens, then the all-gather combines the inputs of the QKV /
 * first FFN linear).  Rank r normalises its rows of x; every requested
 * replica receives all ranks' shards in order.  No reduction, bias, dropout
 * or residual add: the SP region's sum was formed by the previous exit.
 *   x         [s,b,h] in the residual stream's dtype, rank r's shard is its rows
 *   gathered  n_out buffers [s,b,h];  mean/rstd [s*b] (mean NULL for RMS)
 */
int orc_norm_ag_fwd(const orc_cfg* c, const void* x, const void* gamma,
                    const void* beta, void* const* gathered, int n_out,
                    double* mean, double* rstd)
{
    if (!cfg_ok(c)) return -1;
    const int64_t N = c->s * c->b, h = c->h, per = N / c->t;
    double* full = (double*)malloc(sizeof(double) * (size_t)(N * h));
    double** shards = (double**)malloc(sizeof(double*) * (size_t)c->t);
    double* xr = (double*)malloc(sizeof(double) * (size_t)h);
    if (!full || !shards || !xr) {
        free(full); free(shards); free(xr);
        return -2;
    }
    for (int r = 0; r < c->t; ++r) {
        shards[r] = full + (int64_t)r * per * h;
        for (int64_t i = 0; i < per; ++i) {
            const int64_t n = (int64_t)r * per + i;
            double* o = shards[r] + i * h;
            for (int64_t j = 0; j < h; ++j) xr[j] = ld(x, n * h + j, c->res_dtype);
            double mu = 0.0, var = 0.0, rs;
            if (c->norm == ORC_LAYERNORM) {
                for (int64_t j = 0; j < h; ++j) mu += xr[j];
                mu /= (double)h;
                for (int64_t j = 0; j < h; ++j) var += (xr[j] - mu) * (xr[j] - mu);
                var /= (double)h;
                rs = 1.0 / sqrt(var + (double)c->eps);
                for (int64_t j = 0; j < h; ++j) {
                    double b = beta ? ld(beta, j, c->dtype) : 0.0;
                    o[j] = (xr[j] - mu) * rs * ld(gamma, j, c->dtype) + b;
                }
            } else {
                double ms = 0.0;
                for (int64_t j = 0; j < h; ++j) ms += xr[j] * xr[j];
                ms /= (double)h;
                rs = 1.0 / sqrt(ms + (double)c->eps);
                for (int64_t j = 0; j < h; ++j)
                    o[j] = xr[j] * rs * ld(gamma, j, c->dtype);
            }
            if (mean) mean[n] = mu;
            if (rstd) rstd[n] = rs;
        }
    }
    double* g = (double*)malloc(sizeof(double) * (size_t)(N * h));
    if (!g) {
        free(full); free(shards); free(xr);
        return -2;
    }
    orc_all_gather(c->t, per, h, (const double* const*)shards, g);
    for (int q = 0; q < n_out; ++q)
        for (int64_t i = 0; i < N * h; ++i) st(gathered[q], i, c->dtype, g[i]);
    free(g); free(full); free(shards); free(xr);
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Backward                                                                   */
/* ------------------------------------------------------------------------- */

/* reverse-mode through norm, residual add and dropout for one token row.
 *   dn    gradient w.r.t. the norm output of this row (after the
 *         reduce-scatter that is the all-gather's backward)
 *   x     the stored residual sum of the row (residual stream dtype)
 *   acc   per-rank accumulators: dgamma[h], dbeta[h], dbias[h]
 *   dz    gradient w.r.t. the dropout input (the reduced partial sum) */
static void region_row_bwd(const orc_cfg* c, const double* dn,
                           const void* drnext, int64_t row, const void* x,
                           const void* gamma, const uint32_t* mask_row,
                           double mean, double rstd, void* dres_in, double* dz,
                           double* dgamma, double* dbeta, double* dbias,
                           double* xhat)
{
    const int64_t h = c->h;
    const double scale = 1.0 / (1.0 - (double)c->p_drop);
    double sum_g = 0.0, sum_gx = 0.0;
    for (int64_t j = 0; j < h; ++j) {
        double xv = ld(x, row * h + j, c->res_dtype);
        xhat[j] = (c->norm == ORC_LAYERNORM) ? (xv - mean) * rstd : xv * rstd;
        double g = dn[j] * ld(gamma, j, c->dtype);
        sum_g += g;
        sum_gx += g * xhat[j];
        dgamma[j] += dn[j] * xhat[j];
        if (dbeta) dbeta[j] += dn[j];
    }
    const double mg = sum_g / (double)h, mgx = sum_gx / (double)h;
    for (int64_t j = 0; j < h; ++j) {
        double g = dn[j] * ld(gamma, j, c->dtype);
        double dx = (c->norm == ORC_LAYERNORM)
                        ? rstd * (g - mg - xhat[j] * mgx)
                        : rstd * (g - xhat[j] * mgx);
        /* the residual sum feeds both the norm and the next residual add */
        double dr = dx + (drnext ? ld(drnext, row * h + j, c->res_dtype) : 0.0);
        st(dres_in, row * h + j, c->res_dtype, dr);
        int keep = mask_row ? (int)((mask_row[j >> 5] >> (j & 31)) & 1u) : 1;
        dz[j] = keep ? dr * scale : 0.0;
        if (dbias) dbias[j] += dz[j];
    }
}

/*
 * Backward of the whole boundary on t emulated ranks.
 *   dparts[k]      rank k's partial gradient w.r.t. the gathered norm output
 *   drnext         [s,b,h] gradient arriving on the residual stream, or NULL
 *   x              the forward's residual_out, [s,b,h]
 *   mask           the forward's mask (NULL: nothing dropped)
 *   mean, rstd     the forward's statistics (mean unused for RMS)
 *   dres_in        [s,b,h] gradient w.r.t. the residual input (sharded)
 *   dY             [s,b,h] all-gathered gradient w.r.t. the partial sums
 *   dgamma/dbeta/dbias [h] (dbeta, dbias may be NULL), all-reduced over ranks
 */
int orc_bwd(const orc_cfg* c, const void* const* dparts, const void* drnext,
            const void* x, const void* gamma, const uint32_t* mask,
            const double* mean, const double* rstd, void* dres_in, void* dY,
            double* dgamma, double* dbeta, double* dbias)
{
    if (!cfg_ok(c)) return -1;
    const int64_t N = c->s * c->b, h = c->h, per = N / c->t;
    const int64_t W = orc_mask_words(h);
    double* dn = (double*)malloc(sizeof(double) * (size_t)(per * h));
    double* xhat = (double*)malloc(sizeof(double) * (size_t)h);
    double* dz_all = (double*)malloc(sizeof(double) * (size_t)(N * h));
    double* gather = (double*)malloc(sizeof(double) * (size_t)(N * h));
    double* acc = (double*)calloc((size_t)(3 * h), sizeof(double));
    double** shards = (double**)malloc(sizeof(double*) * (size_t)c->t);
    if (!dn || !xhat || !dz_all || !gather || !acc || !shards) {
        free(dn); free(xhat); free(dz_all); free(gather); free(acc); free(shards);
        return -2;
    }
    for (int64_t j = 0; j < h; ++j) {
        dgamma[j] = 0.0;
        if (dbeta) dbeta[j] = 0.0;
        if (dbias) dbias[j] = 0.0;
    }
    for (int r = 0; r < c->t; ++r) {
        /* the all-gather's backward is a reduce-scatter of the gradients */
        orc_reduce_scatter(c->t, N, h, c->dtype, dparts, r, dn);
        double* ag = acc;            /* rank-local parameter gradients */
        double* ab = acc + h;
        double* ac = acc + 2 * h;
        for (int64_t j = 0; j < 3 * h; ++j) acc[j] = 0.0;
        shards[r] = dz_all + (int64_t)r * per * h;
        for (int64_t i = 0; i < per; ++i) {
            int64_t n = (int64_t)r * per + i;
            region_row_bwd(c, dn + i * h, drnext, n, x, gamma,
                           mask ? mask + n * W : NULL,
                           (c->norm == ORC_LAYERNORM) ? mean[n] : 0.0, rstd[n],
                           dres_in, shards[r] + i * h, ag,
                           dbeta ? ab : NULL, dbias ? ac : NULL, xhat);
        }
        /* gamma, beta and bias are replicated on every rank: their gradients
         * are summed over the ranks (ascending) */
        for (int64_t j = 0; j < h; ++j) {
            dgamma[j] += ag[j];
            if (dbeta) dbeta[j] += ab[j];
            if (dbias) dbias[j] += ac[j];
        }
    }
    /* the reduce-scatter's backward is an all-gather of the gradients */
    orc_all_gather(c->t, per, h, (const double* const*)shards, gather);
    for (int64_t i = 0; i < N * h; ++i) st(dY, i, c->dtype, gather[i]);
    free(dn); free(xhat); free(dz_all); free(gather); free(acc); free(shards);
    return 0;
}

/*
 * Backward on selected rows.  Inputs and outputs are [nrows, ...] in sample
 * order.  dgamma, dbeta, dbias (each [h] or NULL) receive the chunk's share
 * of the parameter gradients, the sums over these rows only in sample order;
 * the parameters are replicated, so the gradient over all tokens is the sum
 * of the chunks' shares (the same all-reduce orc_bwd performs over ranks).
 */
int orc_bwd_rows(const orc_cfg* c, int64_t nrows, const void* const* dparts,
                 const void* drnext, const void* x, const void* gamma,
                 const uint32_t* mask, const double* mean, const double* rstd,
                 void* dres_in, void* dY, double* dgamma, double* dbeta,
                 double* dbias)
{
    if (!cfg_ok(c)) return -1;
    const int64_t h = c->h, W = orc_mask_words(h);
    double* dn = (double*)malloc(sizeof(double) * (size_t)h);
    double* xhat = (double*)malloc(sizeof(double) * (size_t)h);
    double* dz = (double*)malloc(sizeof(double) * (size_t)h);
    double* acc = (double*)calloc((size_t)(3 * h), sizeof(double));
    if (!dn || !xhat || !dz || !acc) {
        free(dn); free(xhat); free(dz); free(acc);
        return -2;
    }
    for (int64_t i = 0; i < nrows; ++i) {
        for (int64_t j = 0; j < h; ++j) {
            double a = 0.0;
            for (int k = 0; k < c->t; ++k) a += ld(dparts[k], i * h + j, c->dtype);
            dn[j] = a;
        }
        region_row_bwd(c, dn, drnext, i, x, gamma, mask ? mask + i * W : NULL,
                       (c->norm == ORC_LAYERNORM) ? mean[i] : 0.0, rstd[i],
                       dres_in, dz, acc, acc + h, acc + 2 * h, xhat);
        for (int64_t j = 0; j < h; ++j) st(dY, i * h + j, c->dtype, dz[j]);
    }
    for (int64_t j = 0; j < h; ++j) {
        if (dgamma) dgamma[j] = acc[j];
        if (dbeta) dbeta[j] = acc[h + j];
        if (dbias) dbias[j] = acc[2 * h + j];
    }
    free(dn); free(xhat); free(dz); free(acc);
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Tensor-parallel linears on t emulated ranks                                 */
/* ------------------------------------------------------------------------- */

/*
 * Row-parallel linear ("TP and SP explained with pictures", section "Tensor
 * parallelism, take two: split the inner dimension"; "Chapter 6: TP and SP",
 * section 3): rank k holds columns [k*f/t, (k+1)*f/t) of the input x and the
 * same slice of the inner dimension of the weight w, and computes the
 * full-shape partial
 *     p_k[n, j] = sum over i in slice k of x[n, i] * w[j, i];
 * the partials are then summed across the ranks, k ascending.
 *   x [rows][f] bf16, w [h][f] bf16 (output-by-input), y [rows][h] double.
 * The partials are kept in double: in the fused path none of them is ever
 * stored, so none is rounded to the I/O dtype.
 */
void orc_rowpar_reduce(int64_t rows, int64_t f, int64_t h, int t, const void* x,
                       const void* w, double* y)
{
    const int64_t per = f / t;
    for (int64_t n = 0; n < rows; ++n)
        for (int64_t j = 0; j < h; ++j) {
            double acc = 0.0;
            for (int k = 0; k < t; ++k) {
                double part = 0.0;
                for (int64_t i = k * per; i < (k + 1) * per; ++i)
                    part += ld(x, n * f + i, ORC_BF16) * ld(w, j * f + i, ORC_BF16);
                acc += part;
            }
            y[n * h + j] = acc;
        }
}

/*
 * The forward boundary with the row-parallel linear in front, on selected
 * token rows: y = the reduced partials of orc_rowpar_reduce, then the SP
 * region exactly as orc_fwd_rows (bias once, dropout, residual add, norm).
 *   row_ids[i]   global token row of sample i (the dropout counter)
 *   x_rows       [nrows][f] bf16; residual_rows [nrows][h]; outputs
 *                [nrows][...] in sample order
 */
int orc_linear_rs_fwd_rows(const orc_cfg* c, int64_t f, int64_t nrows, const int64_t* row_ids,
                           const void* x_rows, const void* w, const void* bias,
                           const void* residual, const void* gamma, const void* beta,
                           void* residual_out, void* norm_out, uint32_t* mask, double* mean,
                           double* rstd)
{
    if (!cfg_ok(c) || f < 1 || f % c->t) return -1;
    const int64_t h = c->h, W = orc_mask_words(h);
    double* y = (double*)malloc(sizeof(double) * (size_t)h);
    double* x = (double*)malloc(sizeof(double) * (size_t)h);
    double* o = (double*)malloc(sizeof(double) * (size_t)h);
    if (!y || !x || !o) { free(y); free(x); free(o); return -2; }
    for (int64_t i = 0; i < nrows; ++i) {
        const uint16_t* xr = (const uint16_t*)x_rows + i * f;
        orc_rowpar_reduce(1, f, h, c->t, xr, w, y);
        region_row_fwd(c, row_ids[i], y, bias, residual, i, gamma, beta, residual_out, o,
                       mask ? mask + i * W : NULL, mean ? mean + i : NULL,
                       rstd ? rstd + i : NULL, x);
        for (int64_t j = 0; j < h; ++j) st(norm_out, i * h + j, c->dtype, o[j]);
    }
    free(y); free(x); free(o);
    return 0;
}

/*
 * Column-parallel linear with the all-gather in front ("TP and SP explained
 * with pictures", sections "Tensor parallelism, take one: split the output
 * dimension" and "Add Sequence parallelism"; "Chapter 6: TP and SP", section
 * 2): the t sequence shards are all-gathered into the full input X (shard 0
 * first), then out[n, o] = sum_i X[n, i] * w[o, i], rounded once to bf16.
 *   shards[r] [shard_rows][h] bf16, w [f_out][h] bf16, out [t*shard_rows][f_out]
 */
int orc_ag_colpar_fwd(int t, int64_t shard_rows, int64_t h, int64_t f_out,
                      const void* const* shards, const void* w, void* out)
{
    if (t < 1 || shard_rows < 1 || h < 1 || f_out < 1) return -1;
    const int64_t N = (int64_t)t * shard_rows;
    double** sh = (double**)malloc(sizeof(double*) * (size_t)t);
    double* full = (double*)malloc(sizeof(double) * (size_t)(N * h));
    double* X = (double*)malloc(sizeof(double) * (size_t)(N * h));
    if (!sh || !full || !X) { free(sh); free(full); free(X); return -2; }
    for (int r = 0; r < t; ++r) {
        sh[r] = full + (int64_t)r * shard_rows * h;
        for (int64_t i = 0; i < shard_rows * h; ++i) sh[r][i] = ld(shards[r], i, ORC_BF16);
    }
    orc_all_gather(t, shard_rows, h, (const double* const*)sh, X);
    for (int64_t n = 0; n < N; ++n)
        for (int64_t o = 0; o < f_out; ++o) {
            double acc = 0.0;
            for (int64_t i = 0; i < h; ++i) acc += X[n * h + i] * ld(w, o * h + i, ORC_BF16);
            st(out, n * f_out + o, ORC_BF16, acc);
        }
    free(sh); free(full); free(X);
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Context parallelism: ring attention                                         */
/* ------------------------------------------------------------------------- */

/*
 * Ring attention ("Sequence Parallelism math", section "Context parallelism
 * and ring attention"): Q, K and V are sharded along the sequence, rank r
 * holding the contiguous block r of s/t tokens.  The ranks form a ring; at
 * step i (0 .. t-1) rank r holds K/V block (r - i) mod t (each step every
 * rank passes its block to the next rank), attends its queries against it
 * and folds the result into an online softmax: for each query the running
 * maximum m of its scores so far, the sum l of exp(score - m) and the
 * exp(score - m)-weighted sum o of the values.  When a block raises the
 * maximum, l and o are rescaled by exp(m_old - m_new).  After the t steps
 * every query has seen every key and the output is o / l.
 *   score(n, j) = scale * sum_c q[n, c] * k[j, c]
 *   q, k, v  [bh][s][d] bf16 (bh = batch * heads, each head its own problem)
 *   out      [bh][s][d] bf16, rounded once
 *   lse      [bh][s] double, m + log(l) (the log-sum-exp of the scores), or NULL
 */
int orc_ring_attention(int64_t bh, int64_t s, int64_t d, int t, double scale, const void* q,
                       const void* k, const void* v, void* out, double* lse)
{
    if (bh < 1 || s < 1 || d < 1 || t < 1 || s % t) return -1;
    const int64_t per = s / t;
    double* sc = (double*)malloc(sizeof(double) * (size_t)per);
    double* o = (double*)malloc(sizeof(double) * (size_t)d);
    if (!sc || !o) { free(sc); free(o); return -2; }
    for (int64_t g = 0; g < bh; ++g) {
        const int64_t base = g * s * d;
        for (int64_t n = 0; n < s; ++n) {
            const int r = (int)(n / per);
            double m = -INFINITY, l = 0.0;
            for (int64_t c = 0; c < d; ++c) o[c] = 0.0;
            for (int i = 0; i < t; ++i) {
                const int64_t blk = ((int64_t)r - i + t) % t;
                /* the block's scores and their maximum */
                double bmax = -INFINITY;
                for (int64_t jj = 0; jj < per; ++jj) {
                    const int64_t j = blk * per + jj;
                    double acc = 0.0;
                    for (int64_t c = 0; c < d; ++c)
                        acc += ld(q, base + n * d + c, ORC_BF16) * ld(k, base + j * d + c, ORC_BF16);
                    sc[jj] = scale * acc;
                    if (sc[jj] > bmax) bmax = sc[jj];
                }
                /* fold the block into the running softmax */
                const double mnew = bmax > m ? bmax : m;
                const double alpha = exp(m - mnew);   /* exp(-inf) = 0 at the first step */
                l *= alpha;
                for (int64_t c = 0; c < d; ++c) o[c] *= alpha;
                for (int64_t jj = 0; jj < per; ++jj) {
                    const int64_t j = blk * per + jj;
                    const double p = exp(sc[jj] - mnew);
                    l += p;
                    for (int64_t c = 0; c < d; ++c) o[c] += p * ld(v, base + j * d + c, ORC_BF16);
                }
                m = mnew;
            }
            for (int64_t c = 0; c < d; ++c) st(out, base + n * d + c, ORC_BF16, o[c] / l);
            if (lse) lse[g * s + n] = m + log(l);
        }
    }
    free(sc); free(o);
    return 0;
}

/* The same on selected query rows of one head g: rows[i] is a token index;
 * out [nrows][d], lse [nrows]. */
int orc_ring_attention_rows(int64_t s, int64_t d, int t, double scale, const void* q_rows,
                            const int64_t* rows, int64_t nrows, const void* k, const void* v,
                            void* out, double* lse)
{
    if (s < 1 || d < 1 || t < 1 || s % t) return -1;
    const int64_t per = s / t;
    double* sc = (double*)malloc(sizeof(double) * (size_t)per);
    double* o = (double*)malloc(sizeof(double) * (size_t)d);
    if (!sc || !o) { free(sc); free(o); return -2; }
    for (int64_t i0 = 0; i0 < nrows; ++i0) {
        const int r = (int)(rows[i0] / per);
        double m = -INFINITY, l = 0.0;
        for (int64_t c = 0; c < d; ++c) o[c] = 0.0;
        for (int i = 0; i < t; ++i) {
            const int64_t blk = ((int64_t)r - i + t) % t;
            double bmax = -INFINITY;
            for (int64_t jj = 0; jj < per; ++jj) {
                const int64_t j = blk * per + jj;
                double acc = 0.0;
                for (int64_t c = 0; c < d; ++c)
                    acc += ld(q_rows, i0 * d + c, ORC_BF16) * ld(k, j * d + c, ORC_BF16);
                sc[jj] = scale * acc;
                if (sc[jj] > bmax) bmax = sc[jj];
            }
            const double mnew = bmax > m ? bmax : m;
            const double alpha = exp(m - mnew);
            l *= alpha;
            for (int64_t c = 0; c < d; ++c) o[c] *= alpha;
            for (int64_t jj = 0; jj < per; ++jj) {
                const int64_t j = blk * per + jj;
                const double p = exp(sc[jj] - mnew);
                l += p;
                for (int64_t c = 0; c < d; ++c) o[c] += p * ld(v, j * d + c, ORC_BF16);
            }
            m = mnew;
        }
        for (int64_t c = 0; c < d; ++c) st(out, i0 * d + c, ORC_BF16, o[c] / l);
        if (lse) lse[i0] = m + log(l);
    }
    free(sc); free(o);
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Activation memory per layer and device ("Sequence Parallelism math",      */
/* equations A_layer, A_TP, A_TP+SP).  mode 0: A_layer = sbh(34 + 5as/h);    */
/* 1: A_TP = sbh(10 + 24/t + 5as/(ht)); 2: A_TP+SP = (sbh/t)(34 + 5as/h).     */
/* The result is coefficient * sbh * bytes_per_elem.                          */
/* ------------------------------------------------------------------------- */
double orc_activation_bytes(int64_t s, int64_t b, int64_t h, int64_t a,
                            int32_t t, int32_t mode, double bytes_per_elem)
{
    const double sbh = (double)s * (double)b * (double)h;
    const double attn = 5.0 * (double)a * (double)s / (double)h;
    double coeff;
    if (mode == 0)
        coeff = 34.0 + attn;
    else if (mode == 1)
        coeff = 10.0 + 24.0 / (double)t + attn / (double)t;
    else
        coeff = (34.0 + attn) / (double)t;
    return coeff * sbh * bytes_per_elem;
}

/* Bytes one device sends in a ring collective over t ranks for a tensor of V
 * bytes ("Sequence Parallelism math", section "Why the byte count is
 * identical"): reduce-scatter and all-gather each move (t-1)/t * V, an
 * all-reduce is the two phases, 2(t-1)/t * V.
 *   kind 0: reduce-scatter, 1: all-gather, 2: all-reduce */
double orc_ring_bytes(int32_t t, int32_t kind, double V)
{
    double phase = (double)(t - 1) / (double)t * V;
    return kind == 2 ? 2.0 * phase : phase;
}
