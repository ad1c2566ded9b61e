// C-ABI entry points of the tensor-core kernels (declared in sp_region.h):
// the row-parallel linear whose reduce-scatter is the GEMM's own
// accumulation, with the SP region's bias, dropout and residual add in its
// epilogue; the column-parallel linear whose all-gather is its A-operand
// prologue; and ring attention over the context-parallel ranks.  Argument
// validation, tensor maps and launch; the arithmetic is in sp_gemm2.cuh (CTA
// pairs), sp_gemm.cuh (one CTA, narrow outputs) and sp_attn.cuh.
#include <cuda.h>
#include <math.h>
#include <string.h>

#include <atomic>

#include "sp_attn.cuh"
#include "sp_gemm.cuh"
#include "sp_gemm2.cuh"
#include "sp_host.h"
#include "sp_plans.h"
#include "sp_region.h"

using namespace spk;
using namespace spk_host;

namespace spk {
SPK_ERROR_WORD_ACCESSOR(error_word_gemm)
}  // namespace spk

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled from the driver, found once through the runtime
// (the library links no driver library of its own)
EncodeTiledFn encode_tiled()
{
    static EncodeTiledFn fn = []() -> EncodeTiledFn {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000,
                                             cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    return fn;
}

// Map of a bf16 matrix [rows][cols] (row stride ld elements), boxes of 64
// columns x box_rows rows, 128-byte swizzle, zero fill outside the matrix.
bool make_map(CUtensorMap* m, const void* base, long long rows, long long cols, long long ld,
              int box_rows)
{
    EncodeTiledFn f = encode_tiled();
    if (!f) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kGemmBK, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t tail_bytes() { return (sizeof(GemmTail) + 127) & ~(size_t)127; }

template <int BN, int EPI>
int launch_gemm(GemmArgs a, const GemmMaps& maps, const DevInfo& dev, cudaStream_t st)
{
    constexpr size_t kStage = (size_t)kGemmBM * kGemmBK * 2 + (size_t)BN * kGemmBK * 2;
    const size_t fixed = 1024 + tail_bytes();   // alignment slack, barriers
    if ((size_t)dev.smem_optin <= fixed + 2 * kStage) return SP_ERR_UNSUPPORTED;
    int S = (int)(((size_t)dev.smem_optin - fixed) / kStage);
    if (S > 16) S = 16;
    a.stages = S;
    const size_t smem = fixed + (size_t)S * kStage;
    const void* kern = (const void*)k_tp_gemm<BN, EPI>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess) {
        cudaGetLastError();
        return SP_ERR_CUDA;
    }
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    // persistent: one CTA per SM at most, each looping over tiles
    const long long tiles = (long long)((a.N + BN - 1) / BN) * ((a.M + kGemmBM - 1) / kGemmBM);
    if (tiles < 1) return SP_OK;
    cfg.gridDim = dim3((unsigned)(tiles < dev.sms ? tiles : dev.sms));
    cfg.blockDim = dim3(kGemmThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    void* params[] = {&a, const_cast<GemmMaps*>(&maps)};
    if (cudaLaunchKernelExC(&cfg, kern, params) != cudaSuccess) {
        cudaGetLastError();
        return SP_ERR_CUDA;
    }
    return SP_OK;
}

// Persistent launch of k_tp_gemm2: as many CTA pairs as can be resident at
// once (a pair needs two SMs of one TPC), at most one per 256 x 256 tile.
template <int EPI>
int launch_gemm2(GemmArgs a, const GemmMaps& maps, const DevInfo& dev, cudaStream_t st)
{
    constexpr size_t kStage = (size_t)(kGemmBM + kGemm2HalfN) * kGemmBK * 2;
    const size_t fixed = 1024 + ((sizeof(GemmTail2) + 127) & ~(size_t)127);
    if ((size_t)dev.smem_optin <= fixed + 2 * kStage) return SP_ERR_UNSUPPORTED;
    int S = (int)(((size_t)dev.smem_optin - fixed) / kStage);
    if (S > kGemm2MaxStages) S = kGemm2MaxStages;
    a.stages = S;
    const size_t smem = fixed + (size_t)S * kStage;
    const void* kern = (const void*)k_tp_gemm2<EPI>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess) {
        cudaGetLastError();
        return SP_ERR_CUDA;
    }
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kGemm2Threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;   // the occupancy query takes the cluster shape alone
    cfg.gridDim = dim3((unsigned)(dev.sms & ~1));
    // clusters resident at once, per device and kernel (host threads may
    // race to fill an entry; they store the same value)
    static std::atomic<int> pairs_cache[64][2];
    int pairs = dev.id >= 0 && dev.id < 64 ? pairs_cache[dev.id][EPI].load() : 0;
    if (pairs <= 0) {
        if (cudaOccupancyMaxActiveClusters(&pairs, kern, &cfg) != cudaSuccess || pairs <= 0) {
            cudaGetLastError();
            return SP_ERR_UNSUPPORTED;
        }
        if (dev.id >= 0 && dev.id < 64) pairs_cache[dev.id][EPI].store(pairs);
    }
    const long long tiles = ((a.M + 2 * kGemmBM - 1) / (2 * kGemmBM)) *
                            (long long)((a.N + kGemm2BN - 1) / kGemm2BN);
    if (tiles < 1) return SP_OK;
    const long long np = tiles < pairs ? tiles : pairs;
    cfg.gridDim = dim3((unsigned)(2 * np));
    cfg.numAttrs = 2;
    void* params[] = {&a, const_cast<GemmMaps*>(&maps)};
    if (cudaLaunchKernelExC(&cfg, kern, params) != cudaSuccess) {
        cudaGetLastError();
        return SP_ERR_CUDA;
    }
    return SP_OK;
}

template <int EPI>
int launch_gemm_bn(const GemmArgs& a, const GemmMaps& maps, const DevInfo& dev, cudaStream_t st,
                   int bn)
{
    return bn == 256 ? launch_gemm2<EPI>(a, maps, dev, st)
                     : launch_gemm<128, EPI>(a, maps, dev, st);
}

// output features per tile: 256 (a CTA pair, k_tp_gemm2) unless the output
// is narrower (one CTA, k_tp_gemm with 128-feature tiles)
int pick_bn(long long n) { return n >= 256 ? 256 : 128; }

int check_gemm_cfg(const sp_cfg* cfg)
{
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if (cfg->dtype != SP_BF16 || cfg->res_f32) return SP_ERR_UNSUPPORTED;
    return SP_OK;
}

// ---------------------------------------------------------------------------
// Ring attention: shape checks, the work split and the launch
// ---------------------------------------------------------------------------

int check_attn_shape(const sp_cfg* cfg, int heads)
{
    int rc = check_gemm_cfg(cfg);
    if (rc) return rc;
    if (heads < 1) return SP_ERR_INVALID_ARG;
    if (!(cfg->row_begin == 0 && cfg->row_end == 0)) return SP_ERR_INVALID_ARG;
    if (cfg->h != (int64_t)heads * kAttnD) return SP_ERR_UNSUPPORTED;   // head dim 128
    const long long S = cfg->s, per = S / cfg->t;
    if (S % kAttnBM || per % kAttnBN) return SP_ERR_UNSUPPORTED;
    const long long bh = cfg->b * (long long)heads;
    if (bh * S >= (1LL << 31)) return SP_ERR_UNSUPPORTED;
    return SP_OK;
}

constexpr int kAttnMaxSplit = 8;      // pieces per split unit, at most
constexpr int kAttnMinPiece = 4;      // ring steps (key tiles) per piece, at least

// The work of one call: units of QT query tiles of one head, every ring step.
// They run one CTA each (one CTA per SM), so `units` CTAs take
// ceil(units / sms) rounds of the slowest SM.  With `split` allowed, the
// units of the last, partly filled round are cut into k contiguous ranges of
// ring steps, the k that leaves the shortest last round (ceil(R k / sms) / k
// unit times for R leftover units), and combined afterwards.
struct AttnPlan {
    int qt;
    int nx;                  // units per head
    long long units;
    long long full_units;    // whole units
    long long tail_units;    // split units
    int split;               // pieces per split unit (1: none)
    size_t ws_bytes;         // partial results of the pieces
};

void attn_plan(const sp_cfg* cfg, int heads, int sms, bool allow_split, AttnPlan* p)
{
    const long long S = cfg->s, per = S / cfg->t;
    const long long bh = cfg->b * (long long)heads;
    // two query tiles per CTA when a rank's block holds an even number of
    // them (both then visit the key tiles in the same ring order)
    p->qt = per % (2 * kAttnBM) == 0 ? 2 : 1;
    p->nx = (int)(S / (p->qt * kAttnBM));
    p->units = (long long)p->nx * bh;
    p->full_units = p->units;
    p->tail_units = 0;
    p->split = 1;
    p->ws_bytes = 0;
    const long long rem = sms > 0 ? p->units % sms : 0;
    if (!allow_split || rem == 0) return;
    const long long n_tiles = S / kAttnBN;
    int best_k = 1;
    double best = 1.0;   // the last round, in unit times, without a split
    for (int k = 2; k <= kAttnMaxSplit && n_tiles / k >= kAttnMinPiece; ++k) {
        const double tt = (double)((rem * k + sms - 1) / sms) / k;
        if (tt < best - 1e-9) {
            best = tt;
            best_k = k;
        }
    }
    if (best_k == 1) return;
    p->split = best_k;
    p->tail_units = rem;
    p->full_units = p->units - rem;
    p->ws_bytes = (size_t)rem * best_k * (size_t)(p->qt * kAttnBM) * (kAttnD + 2) * sizeof(float);
}

int attn_fwd(const sp_cfg* cfg, int heads, float scale, const void* q, const void* k,
             const void* v, void* out, float* lse, void* workspace, size_t workspace_bytes,
             bool allow_split, void* stream)
{
    int rc = check_attn_shape(cfg, heads);
    if (rc) return rc;
    if (!q || !k || !v || !out || !(scale > 0.0f) || !isfinite(scale)) return SP_ERR_INVALID_ARG;
    for (const void* p : {q, k, v, (const void*)out})
        if (!aligned(p, 16)) return SP_ERR_INVALID_ARG;
    if (lse && !aligned(lse, 4)) return SP_ERR_INVALID_ARG;
    if (workspace && !aligned(workspace, 16)) return SP_ERR_INVALID_ARG;
    DevInfo dev;
    if ((rc = use_device_of(out, &dev))) return rc;
    AttnPlan pl;
    attn_plan(cfg, heads, dev.sms, allow_split, &pl);
    if (pl.ws_bytes && (!workspace || workspace_bytes < pl.ws_bytes)) return SP_ERR_INVALID_ARG;

    const long long S = cfg->s, per = S / cfg->t;
    const long long bh = cfg->b * (long long)heads;
    AttnMaps maps;
    memset(&maps, 0, sizeof(maps));
    if (!make_map(&maps.q, q, bh * S, kAttnD, kAttnD, kAttnBM) ||
        !make_map(&maps.k, k, bh * S, kAttnD, kAttnD, kAttnBN) ||
        !make_map(&maps.v, v, bh * S, kAttnD, kAttnD, kAttnBN))
        return SP_ERR_INVALID_ARG;
    AttnArgs a;
    memset(&a, 0, sizeof(a));
    a.s = S;
    a.t = cfg->t;
    a.tiles_per_block = (int)(per / kAttnBN);
    a.scale_log2 = (float)((double)scale * 1.4426950408889634);
    a.out = out;
    a.lse = lse;
    a.nx = pl.nx;
    a.full_units = (int)pl.full_units;
    a.split = pl.split;
    const size_t rows_per_unit = (size_t)pl.qt * kAttnBM;
    const long long pieces = pl.tail_units * pl.split;
    if (pieces) {
        a.part_o = static_cast<float*>(workspace);
        a.part_ml = a.part_o + (size_t)pieces * rows_per_unit * kAttnD;
    }
    const int qt = pl.qt;
    const size_t smem =
        1024 + (size_t)(qt + 4) * kAttnTile +
        (((qt == 2 ? sizeof(AttnTail<2>) : sizeof(AttnTail<1>)) + 127) & ~(size_t)127);
    if (smem > (size_t)dev.smem_optin) return SP_ERR_UNSUPPORTED;
    const void* kern = qt == 2 ? (const void*)k_ring_attn<2> : (const void*)k_ring_attn<1>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess) {
        cudaGetLastError();
        return SP_ERR_CUDA;
    }
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3((unsigned)(pl.full_units + pieces));
    lc.blockDim = dim3(attn_threads(qt));
    lc.dynamicSmemBytes = smem;
    lc.stream = static_cast<cudaStream_t>(stream);
    lc.attrs = attr;
    lc.numAttrs = 1;
    void* params[] = {&a, &maps};
    if (cudaLaunchKernelExC(&lc, kern, params) != cudaSuccess) {
        cudaGetLastError();
        return SP_ERR_CUDA;
    }
    if (!pieces) return SP_OK;
    // the split units' rows, one warp each
    int rpu = (int)rows_per_unit;
    long long rows = pl.tail_units * (long long)rows_per_unit;
    constexpr int kWarpsPerBlock = kAttnMergeThreads / 32;
    lc.gridDim = dim3((unsigned)((rows + kWarpsPerBlock - 1) / kWarpsPerBlock));
    lc.blockDim = dim3(kAttnMergeThreads);
    lc.dynamicSmemBytes = 0;
    void* mparams[] = {&a, &rpu, &rows};
    if (cudaLaunchKernelExC(&lc, (const void*)k_attn_merge, mparams) != cudaSuccess) {
        cudaGetLastError();
        return SP_ERR_CUDA;
    }
    return SP_OK;
}

}  // namespace

extern "C" {

int sp_rowpar_linear_rs_fwd(const sp_cfg* cfg, int64_t f, const void* x, const void* w,
                            const void* bias, const void* residual, void* residual_out,
                            uint32_t* mask_bits, void* stream)
{
    int rc = check_gemm_cfg(cfg);
    if (rc) return rc;
    if (!x || !w || !residual || !residual_out) return SP_ERR_INVALID_ARG;
    if (f < 1 || f % cfg->t) return SP_ERR_INVALID_ARG;
    if (f % 8 || cfg->h % 8 || f > (1LL << 31) - 64) return SP_ERR_UNSUPPORTED;
    if (!mask_bits && cfg->p_drop > 0.0f) return SP_ERR_INVALID_ARG;
    for (const void* p : {x, w, bias, residual, (const void*)residual_out})
        if (p && !aligned(p, 16)) return SP_ERR_INVALID_ARG;
    if (mask_bits && !aligned(mask_bits, 4)) return SP_ERR_INVALID_ARG;
    DevInfo dev;
    if ((rc = use_device_of(residual_out, &dev))) return rc;

    long long row0 = 0, rows = 0;
    call_rows(cfg, &row0, &rows);
    const long long h = cfg->h;
    const int bn = pick_bn(h);
    GemmMaps maps;
    memset(&maps, 0, sizeof(maps));
    // x: this call's rows [rows][f]; the t ranks' slices are its column
    // blocks, so one map covers every rank
    if (!make_map(&maps.a[0], x, rows, f, f, kGemmBM) ||
        !make_map(&maps.b, w, h, f, f, bn == 256 ? kGemm2HalfN : bn))
        return SP_ERR_INVALID_ARG;
    GemmArgs a;
    memset(&a, 0, sizeof(a));
    a.M = rows;
    a.N = (int)h;
    a.K = (int)f;
    a.rows_per_shard = (int)(rows > 0x7FFFFFFF ? 0x7FFFFFFF : rows);
    a.nmaps = 1;
    a.out = residual_out;
    a.bias = bias;
    a.residual = residual;
    a.mask = reinterpret_cast<uint8_t*>(mask_bits);
    a.mask_row_bytes = (int)(4 * ((h + 31) / 32));
    a.row0 = row0;
    a.scale = 1.0f / (1.0f - cfg->p_drop);
    a.thr = drop_threshold(cfg->p_drop);
    a.off_lo = (uint32_t)cfg->offset;
    a.off_hi = (uint32_t)(cfg->offset >> 32);
    const uint32_t seed_lo = (uint32_t)cfg->seed, seed_hi = (uint32_t)(cfg->seed >> 32);
    for (int r = 0; r < 10; ++r) {   // Philox key schedule: Weyl increments per round
        a.keys[r][0] = seed_lo + (uint32_t)r * 0x9E3779B9u;
        a.keys[r][1] = seed_hi + (uint32_t)r * 0xBB67AE85u;
    }
    a.dropout = cfg->p_drop > 0.0f ? 1 : 0;
    return launch_gemm_bn<0>(a, maps, dev, static_cast<cudaStream_t>(stream), bn);
}

int sp_ag_colpar_linear_fwd(const sp_cfg* cfg, int64_t f_out, const void* const* shards,
                            const void* w, void* out, void* stream)
{
    int rc = check_gemm_cfg(cfg);
    if (rc) return rc;
    if (!shards || !w || !out || f_out < 1) return SP_ERR_INVALID_ARG;
    if (!(cfg->row_begin == 0 && cfg->row_end == 0)) return SP_ERR_INVALID_ARG;
    const int t = cfg->t;
    const long long N = cfg->s * cfg->b, per = N / t, h = cfg->h;
    if (t > kGemmMaxShards) return SP_ERR_UNSUPPORTED;
    if (t > 1 && per % kGemmBM) return SP_ERR_UNSUPPORTED;   // a tile lies in one shard
    if (h % 8 || f_out % 8 || h > (1LL << 31) - 64 || f_out > (1LL << 31) - 256)
        return SP_ERR_UNSUPPORTED;
    for (int r = 0; r < t; ++r)
        if (!shards[r] || !aligned(shards[r], 16)) return SP_ERR_INVALID_ARG;
    if (!aligned(w, 16) || !aligned(out, 16)) return SP_ERR_INVALID_ARG;
    DevInfo dev;
    if ((rc = use_device_of(out, &dev))) return rc;

    const int bn = pick_bn(f_out);
    GemmMaps maps;
    memset(&maps, 0, sizeof(maps));
    for (int r = 0; r < t; ++r)
        if (!make_map(&maps.a[r], shards[r], per, h, h, kGemmBM)) return SP_ERR_INVALID_ARG;
    if (!make_map(&maps.b, w, f_out, h, h, bn == 256 ? kGemm2HalfN : bn)) return SP_ERR_INVALID_ARG;
    GemmArgs a;
    memset(&a, 0, sizeof(a));
    a.M = N;
    a.N = (int)f_out;
    a.K = (int)h;
    a.rows_per_shard = (int)per;
    a.nmaps = t;
    a.out = out;
    return launch_gemm_bn<1>(a, maps, dev, static_cast<cudaStream_t>(stream), bn);
}

int sp_ring_attention_fwd(const sp_cfg* cfg, int32_t heads, float scale, const void* q,
                          const void* k, const void* v, void* out, float* lse, void* stream)
{
    return attn_fwd(cfg, heads, scale, q, k, v, out, lse, nullptr, 0, false, stream);
}

int sp_ring_attention_fwd_ws(const sp_cfg* cfg, int32_t heads, float scale, const void* q,
                             const void* k, const void* v, void* out, float* lse,
                             void* workspace, size_t workspace_bytes, void* stream)
{
    return attn_fwd(cfg, heads, scale, q, k, v, out, lse, workspace, workspace_bytes, true,
                    stream);
}

int sp_ring_attention_workspace_bytes(const sp_cfg* cfg, int32_t heads, int32_t device,
                                      size_t* bytes)
{
    int rc = check_attn_shape(cfg, heads);
    if (rc) return rc;
    if (!bytes) return SP_ERR_INVALID_ARG;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess) {
        cudaGetLastError();
        return SP_ERR_CUDA;
    }
    AttnPlan pl;
    attn_plan(cfg, heads, sms, true, &pl);
    *bytes = pl.ws_bytes;
    return SP_OK;
}

}  // extern "C"
