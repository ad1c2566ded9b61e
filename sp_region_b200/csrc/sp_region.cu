// C-ABI entry points of the SP boundary library (declared in sp_region.h):
// argument validation, kernel selection and launch.  All device work goes
// through the kernels in sp_fwd.cuh, sp_bwd.cuh and sp_gather.cuh; nothing
// here computes on the host except the activation-memory closed forms.
#include <math.h>
#include <string.h>

#include <algorithm>

#include "sp_region.h"
#include "sp_bwd.cuh"
#include "sp_device.cuh"
#include "sp_entry.cuh"
#include "sp_fwd.cuh"
#include "sp_gather.cuh"
#include "sp_host.h"
#include "sp_plans.h"

using namespace spk;
using namespace spk_host;

namespace spk {
SPK_ERROR_WORD_ACCESSOR(error_word_host)
}  // namespace spk

namespace spk_host {

// Make the device that owns `p` current for this library's CUDA runtime and
// read its limits.  The caller's framework may have another device current,
// so the data decides.
int use_device_of(const void* p, DevInfo* d)
{
    cudaPointerAttributes at;
    cudaError_t e = cudaPointerGetAttributes(&at, p);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return SP_ERR_INVALID_ARG;
    }
    if (at.type != cudaMemoryTypeDevice && at.type != cudaMemoryTypeManaged)
        return SP_ERR_INVALID_ARG;
    d->id = at.device;
    if (cudaSetDevice(d->id) != cudaSuccess) return SP_ERR_CUDA;
    if (cudaDeviceGetAttribute(&d->sms, cudaDevAttrMultiProcessorCount, d->id) != cudaSuccess)
        return SP_ERR_CUDA;
    if (cudaDeviceGetAttribute(&d->smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin,
                               d->id) != cudaSuccess)
        return SP_ERR_CUDA;
    return SP_OK;
}

int check_cfg(const sp_cfg* c)
{
    if (!c) return SP_ERR_INVALID_ARG;
    if (c->s < 1 || c->b < 1 || c->h < 1) return SP_ERR_INVALID_ARG;
    if (c->t < 1 || c->t > SP_MAX_T) return SP_ERR_INVALID_ARG;
    if (c->s % c->t) return SP_ERR_INVALID_ARG;
    if (c->dtype != SP_F32 && c->dtype != SP_BF16) return SP_ERR_INVALID_ARG;
    if (c->norm != SP_LAYERNORM && c->norm != SP_RMSNORM) return SP_ERR_INVALID_ARG;
    if (!(c->p_drop >= 0.0f && c->p_drop < 1.0f)) return SP_ERR_INVALID_ARG;
    if (!(c->eps > 0.0f) || !isfinite(c->eps)) return SP_ERR_INVALID_ARG;
    // Philox counter word 1 holds the token row, word 0 holds j >> 2
    if (c->s > (1LL << 32) || c->b > (1LL << 32)) return SP_ERR_INVALID_ARG;
    if (c->s * c->b > 0xFFFFFFFFLL) return SP_ERR_INVALID_ARG;
    if (c->h > (1LL << 24)) return SP_ERR_INVALID_ARG;
    if (!(c->row_begin == 0 && c->row_end == 0) &&
        !(c->row_begin >= 0 && c->row_begin < c->row_end && c->row_end <= c->s * c->b))
        return SP_ERR_INVALID_ARG;
    if (c->res_f32 != 0 && c->res_f32 != 1) return SP_ERR_INVALID_ARG;
    return SP_OK;
}

// The token rows [*r0, *r0 + *nrows) a call processes.
void call_rows(const sp_cfg* c, long long* r0, long long* nrows)
{
    if (c->row_begin == 0 && c->row_end == 0) {
        *r0 = 0;
        *nrows = c->s * c->b;
    } else {
        *r0 = c->row_begin;
        *nrows = c->row_end - c->row_begin;
    }
}

int elem_bytes(const sp_cfg* c) { return c->dtype == SP_F32 ? 4 : 2; }

// bytes per element of the residual stream tensors (fp32 when res_f32)
int res_elem_bytes(const sp_cfg* c) { return c->res_f32 ? 4 : elem_bytes(c); }

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

uint32_t drop_threshold(float p) { return (uint32_t)floor((double)p * 4294967296.0); }

}  // namespace spk_host

namespace {

constexpr int kGeneralThreads = 256;

size_t round128(size_t x) { return (x + 127) & ~(size_t)127; }

size_t ring_tail_bytes() { return round128(sizeof(RingTail)); }

// Rows covered at once by a general-kernel launch (its grid).
long long general_grid(long long rows, int sms)
{
    const long long g = (long long)sms * 4;
    return rows < g ? rows : g;
}


// Preference order when the caller gives no hint: the first feasible plan
// wins.  A hinted plan is tried first.  Plans that split a row across a
// 2-CTA cluster come last: their per-row exchange of partial sums between
// SMs costs more than it saves wherever a one-CTA plan fits, so they serve
// rows too wide for one CTA (h > 16384 in bf16).
// (measured on B200 for h = 4096 ... 12288: more rows in flight per SM wins
// while the registers and the ring's stages allow it)
constexpr int kFwdOrder[] = {10, 4, 9, 6, 8, 1, 2, 11, 0, 3, 5, 7, 12, 13, 15, 14, 16, 17, 18};
// the entry into a TP region streams one segment per row, so its per-row
// reductions dominate and more rows in flight per SM pay off first
constexpr int kFwdEntryOrder[] = {13, 12, 11, 10, 4, 9, 6, 8, 1, 2, 0, 3, 5, 7, 15, 14, 16,
                                  17, 18};
// backward: tensor-memory accumulators first; they leave shared memory to the
// ring (measured on B200 for bf16 rows of h = 12288, t = 16: 2 -> 8 stages,
// 4.9 -> 6.6 TB/s).  Plan 23 (two groups of 4-vector threads) tiles rows of
// 1024 vectors exactly: h = 8192 went 5.60 -> 5.69 TB/s over plan 18.
constexpr int kBwdOrder[] = {19, 15, 23, 18, 16, 17, 21, 20, 22, 11, 8, 9, 12,
                             2, 3, 5, 10, 6, 1, 0, 4, 7, 13, 14};

int group_threads(int hv, int V)
{
    const int per = (hv + V - 1) / V;
    return (per + 31) / 32 * 32;
}

long long ring_stages(long long smem_optin, long long fixed, uint32_t stage_stride)
{
    if (smem_optin <= fixed) return 0;
    long long S = (smem_optin - fixed) / stage_stride;
    return S > 64 ? 64 : S;
}

// entry kernel: V = 4 vectors per thread in bf16, 2 in fp32 (registers)
template <typename T>
const void* entry_kernel_t(bool ln, bool exact)
{
    constexpr int V = sizeof(T) == 2 ? 4 : 2;
    if (ln)
        return exact ? (const void*)k_norm_ag<T, V, true, true>
                     : (const void*)k_norm_ag<T, V, true, false>;
    return exact ? (const void*)k_norm_ag<T, V, false, true>
                 : (const void*)k_norm_ag<T, V, false, false>;
}

// kernel of a fast plan for the I/O dtype and norm (defined by the
// instantiation units sp_inst_fwd.cu / sp_inst_bwd.cu)
const void* fwd_kernel_of(int dtype, bool ln, int id, bool exact)
{
    if (dtype == SP_BF16) return ln ? fwd_kernel_bf16_ln(id, exact) : fwd_kernel_bf16_rms(id, exact);
    return ln ? fwd_kernel_f32_ln(id, exact) : fwd_kernel_f32_rms(id, exact);
}

const void* bwd_kernel_of(int dtype, bool ln, int id, bool exact)
{
    if (dtype == SP_BF16) return ln ? bwd_kernel_bf16_ln(id, exact) : bwd_kernel_bf16_rms(id, exact);
    return ln ? bwd_kernel_f32_ln(id, exact) : bwd_kernel_f32_rms(id, exact);
}

// Every launch allows programmatic dependent launch: the kernel may be
// scheduled while the previous kernel in the stream is still running, and
// waits in-kernel (griddepcontrol.wait) before touching global memory.
int launch_kernel_args(const void* kern, int grid, int block, size_t smem, cudaStream_t st,
                       void** params)
{
    if (!kern) return SP_ERR_UNSUPPORTED;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess) {
        cudaGetLastError();
        return SP_ERR_CUDA;
    }
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelExC(&cfg, kern, params) != cudaSuccess) {
        cudaGetLastError();
        return SP_ERR_CUDA;
    }
    return SP_OK;
}

int launch_kernel(const void* kern, int grid, int block, size_t smem, cudaStream_t st,
                  void* args)
{
    void* params[] = {args};
    return launch_kernel_args(kern, grid, block, smem, st, params);
}

// A persistent launch of clusters of `cs` CTAs: as many clusters as fit on
// the device at once (at most `rows`), each CTA one SM.  *grid returns the
// CTA count.
int launch_clusters(const void* kern, long long rows, int cs, int block, size_t smem,
                    cudaStream_t st, void* args, int* grid)
{
    if (!kern) return SP_ERR_UNSUPPORTED;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess) {
        cudaGetLastError();
        return SP_ERR_CUDA;
    }
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)cs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    cfg.gridDim = dim3(cs);
    int max_clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&max_clusters, kern, &cfg) != cudaSuccess ||
        max_clusters < 1) {
        cudaGetLastError();
        return SP_ERR_UNSUPPORTED;
    }
    const long long ncl = rows < max_clusters ? rows : max_clusters;
    cfg.gridDim = dim3((unsigned)(ncl * cs));
    *grid = (int)(ncl * cs);
    void* params[] = {args};
    if (cudaLaunchKernelExC(&cfg, kern, params) != cudaSuccess) {
        cudaGetLastError();
        return SP_ERR_CUDA;
    }
    return SP_OK;
}

// A fast launch: the chosen plan, its block and grid, and its dynamic shared
// memory (the layout offsets are written into the kernel arguments).
struct FastLaunch {
    int plan = -1;
    int block = 0;
    int grid = 0;
    int groups = 1;
    int cs = 1;
    bool exact = false;   // C * V covers the row (slice) exactly
    size_t smem = 0;
};

FastLaunch plan_fwd(FwdArgs& a, const DevInfo& dev, int E, int hint)
{
    FastLaunch L;
    const size_t tailb = ring_tail_bytes();
    const size_t pstride = round128((size_t)a.h * E);
    int order[1 + kNumFwdPlans];
    int no = 0;
    if (hint >= 1 && hint <= kNumFwdPlans) order[no++] = hint - 1;
    if (a.t == 0)
        for (int id : kFwdEntryOrder) order[no++] = id;
    else
        for (int id : kFwdOrder) order[no++] = id;
    for (int oi = 0; oi < no; ++oi) {
        const int id = order[oi];
        const Plan& p = kFwdPlans[id];
        if (a.hv % p.CS) continue;
        if (a.res_f32 && p.V >= 4 && p.maxT <= 544) continue;   // compiled without it
        const int C = group_threads(a.hv / p.CS, p.V);
        if (p.G * C + 32 > p.maxT) continue;
        // each CTA stages and keeps parameters for its 1/CS of the row
        const uint32_t seg_max = a.res_seg_bytes > a.seg_bytes ? a.res_seg_bytes : a.seg_bytes;
        const uint32_t stride = (uint32_t)round128(seg_max / p.CS);
        const size_t pstride_c = round128((size_t)a.h * E / p.CS);
        long long S = ring_stages(dev.smem_optin, (long long)(tailb + 3 * pstride_c), stride);
        S -= S % p.G;                 // G sub-rings of S / G stages each
        if (S < 2 * p.G) continue;
        a.stage_stride = stride;
        a.stages = (int)S;
        a.param_off = (uint32_t)(S * a.stage_stride);
        a.param_stride = (uint32_t)pstride_c;
        a.tail_off = (uint32_t)(a.param_off + 3 * pstride_c);
        L.plan = id;
        L.block = p.G * C + 32;
        L.grid = (int)(a.rows < dev.sms ? a.rows : dev.sms);
        L.groups = p.G;
        L.cs = p.CS;
        L.exact = C * p.V == a.hv / p.CS;
        L.smem = (size_t)a.tail_off + tailb;
        return L;
    }
    (void)pstride;
    return L;
}

FastLaunch plan_bwd(BwdArgs& a, const DevInfo& dev, int E, int hint)
{
    FastLaunch L;
    const size_t tailb = ring_tail_bytes();
    const size_t pstride = round128((size_t)a.h * E);
    int order[1 + kNumBwdPlans];
    int no = 0;
    if (hint >= 1 && hint <= kNumBwdPlans) order[no++] = hint - 1;
    for (int id : kBwdOrder) order[no++] = id;
    for (int oi = 0; oi < no; ++oi) {
        const int id = order[oi];
        const Plan& p = kBwdPlans[id];
        if (p.CS != 1) continue;
        const int C = group_threads(a.hv, p.V);
        if (p.G * C + 32 > p.maxT) continue;
        uint32_t tcols = 0;
        if (p.acc == 2) {
            // 24 columns per vector for each warp; the warps of a lane
            // quarter sit side by side; allocations are powers of 2 >= 32
            const int per_quarter = ((p.G * C / 32) + 3) / 4;
            const int need = per_quarter * 24 * p.V;
            if (need > 512) continue;
            tcols = 32;
            while ((int)tcols < need) tcols <<= 1;
        }
        const size_t accb = p.acc == 1 ? (size_t)3 * 2 * a.hv * sizeof(float4) : 0;
        long long S = ring_stages(dev.smem_optin, (long long)(tailb + pstride + accb),
                                  a.stage_stride);
        S -= S % p.G;                 // G sub-rings of S / G stages each
        if (S < 2 * p.G) continue;
        a.stages = (int)S;
        a.tmem_cols = tcols;
        // tensor-memory groups fold their sums in the CTA when the staging
        // ((G-1) x 3 x 2 planes of 16 bytes per vector) fits in the ring
        a.fold = (p.acc == 2 && p.G > 1 &&
                  (size_t)(p.G - 1) * 96 * (size_t)a.hv <= (size_t)S * a.stage_stride)
                     ? 1 : 0;
        a.param_off = (uint32_t)(S * a.stage_stride);
        a.acc_off = (uint32_t)(a.param_off + pstride);
        a.tail_off = (uint32_t)(a.acc_off + accb);
        L.plan = id;
        L.block = p.G * C + 32;
        L.grid = (int)(a.rows < dev.sms ? a.rows : dev.sms);
        L.groups = p.G;
        L.exact = C * p.V == a.hv;
        L.smem = (size_t)a.tail_off + tailb;
        return L;
    }
    return L;
}

}  // namespace

extern "C" {

int sp_plan_count(int32_t* fwd_plans, int32_t* bwd_plans)
{
    if (!fwd_plans || !bwd_plans) return SP_ERR_INVALID_ARG;
    *fwd_plans = kNumFwdPlans;
    *bwd_plans = kNumBwdPlans;
    return SP_OK;
}

const char* sp_status_string(int status)
{
    switch (status) {
    case SP_OK: return "ok";
    case SP_ERR_INVALID_ARG: return "invalid argument";
    case SP_ERR_UNSUPPORTED: return "unsupported configuration";
    case SP_ERR_CUDA: return "CUDA error";
    case SP_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    default: return "unknown status";
    }
}

int sp_activation_bytes(int64_t s, int64_t b, int64_t h, int64_t a, int32_t t, int32_t mode,
                        double bytes_per_elem, double* out)
{
    if (!out || s < 1 || b < 1 || h < 1 || a < 0 || t < 1) return SP_ERR_INVALID_ARG;
    if (!(bytes_per_elem > 0.0)) return SP_ERR_INVALID_ARG;
    const double sbh = (double)s * (double)b * (double)h;
    const double attn = 5.0 * (double)a * (double)s / (double)h;   // 5as/h
    double c;
    switch (mode) {
    case 0: c = 34.0 + attn; break;                                   // A_layer
    case 1: c = 10.0 + 24.0 / (double)t + attn / (double)t; break;    // A_TP
    case 2: c = (34.0 + attn) / (double)t; break;                     // A_TP+SP
    default: return SP_ERR_INVALID_ARG;
    }
    *out = c * sbh * bytes_per_elem;
    return SP_OK;
}

}  // extern "C"

namespace {

// The forward with an explicit number of partial sums: cfg->t for the exit
// of a tensor-parallel region, 0 for the entry into one (norm, then
// all-gather; residual_out is then NULL and there is no dropout).
int fwd_impl(const sp_cfg* cfg, int nparts, const void* const* partials, const void* bias,
             const void* residual, const void* gamma, const void* beta, void* residual_out,
             void* const* gathered, int32_t n_gathered, uint32_t* mask_bits, float* mean,
             float* rstd, void* stream)
{
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if ((nparts > 0 && (!partials || !residual_out)) || !residual || !gamma || !gathered)
        return SP_ERR_INVALID_ARG;
    if (n_gathered < 1 || n_gathered > SP_MAX_T) return SP_ERR_INVALID_ARG;
    const int E = elem_bytes(cfg);
    const bool ln = cfg->norm == SP_LAYERNORM;
    bool all16 = true;
    for (int k = 0; k < nparts; ++k) {
        if (!partials[k] || !aligned(partials[k], E)) return SP_ERR_INVALID_ARG;
        all16 = all16 && aligned(partials[k], 16);
    }
    for (int q = 0; q < n_gathered; ++q) {
        if (!gathered[q] || !aligned(gathered[q], E)) return SP_ERR_INVALID_ARG;
        all16 = all16 && aligned(gathered[q], 16);
    }
    const int Er = res_elem_bytes(cfg);
    const void* elem_ptrs[] = {gamma, bias, ln ? beta : nullptr};
    for (const void* p : elem_ptrs) {
        if (p && !aligned(p, E)) return SP_ERR_INVALID_ARG;
        all16 = all16 && (!p || aligned(p, 16));
    }
    for (const void* p : {residual, (const void*)residual_out}) {   // the residual stream
        if (p && !aligned(p, Er)) return SP_ERR_INVALID_ARG;
        all16 = all16 && (!p || aligned(p, 16));
    }
    if ((mask_bits && !aligned(mask_bits, 4)) || (mean && !aligned(mean, 4)) ||
        (rstd && !aligned(rstd, 4)))
        return SP_ERR_INVALID_ARG;

    DevInfo dev;
    if ((rc = use_device_of(residual, &dev))) return rc;

    long long row0 = 0, rows = 0;
    call_rows(cfg, &row0, &rows);
    const int h = (int)cfg->h;
    FwdArgs a;
    memset(&a, 0, sizeof(a));
    for (int k = 0; k < nparts; ++k) a.parts[k] = partials[k];
    for (int q = 0; q < n_gathered; ++q) a.gathered[q] = gathered[q];
    a.bias = bias;
    a.residual = residual;
    a.gamma = gamma;
    a.beta = ln ? beta : nullptr;
    a.residual_out = residual_out;
    a.mask = reinterpret_cast<uint8_t*>(mask_bits);
    a.mean = ln ? mean : nullptr;
    a.rstd = rstd;
    a.rows = rows;
    a.row0 = row0;
    a.h = h;
    a.hv = h / 8;
    a.t = nparts;
    a.n_gathered = n_gathered;
    a.seg_bytes = (uint32_t)(h * E);
    a.res_seg_bytes = (uint32_t)(h * Er);
    a.res_f32 = Er != E ? 1 : 0;
    a.stage_stride = (uint32_t)round128(a.res_seg_bytes > a.seg_bytes ? a.res_seg_bytes
                                                                       : a.seg_bytes);
    a.mask_row_bytes = 4 * ((h + 31) / 32);
    a.eps = cfg->eps;
    a.inv_h = (float)(1.0 / (double)h);
    a.scale = 1.0f / (1.0f - cfg->p_drop);
    a.thr = drop_threshold(cfg->p_drop);
    a.seed_lo = (uint32_t)cfg->seed;
    a.seed_hi = (uint32_t)(cfg->seed >> 32);
    a.off_lo = (uint32_t)cfg->offset;
    a.off_hi = (uint32_t)(cfg->offset >> 32);
    for (int r = 0; r < 10; ++r) {   // Philox key schedule: Weyl increments per round
        a.keys[r][0] = a.seed_lo + (uint32_t)r * 0x9E3779B9u;
        a.keys[r][1] = a.seed_hi + (uint32_t)r * 0xBB67AE85u;
    }
    a.dropout = cfg->p_drop > 0.0f ? 1 : 0;
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    // the entry (no partial sums) without a plan hint: registers instead of
    // a staging ring, G groups of C threads per CTA
    if (nparts == 0 && cfg->fwd_plan == 0 && !a.res_f32 && h % 8 == 0 && all16) {
        const int V = E == 2 ? 4 : 2;
        const int C = group_threads(h / 8, V);
        if (C <= kEntryThreads) {
            EntryArgs e;
            memset(&e, 0, sizeof(e));
            e.x = residual;
            e.gamma = gamma;
            e.beta = ln ? beta : nullptr;
            for (int q = 0; q < n_gathered; ++q) e.gathered[q] = gathered[q];
            e.mean = ln ? mean : nullptr;
            e.rstd = rstd;
            e.rows = rows;
            e.row0 = row0;
            e.hv = h / 8;
            e.C = C;
            e.n_gathered = n_gathered;
            e.seg_bytes = (uint32_t)(h * E);
            e.param_stride = (uint32_t)round128((size_t)h * E);
            e.inv_h = a.inv_h;
            e.eps = cfg->eps;
            const int G = std::min(8, kEntryThreads / C);
            const size_t smem = 2 * (size_t)e.param_stride + (size_t)2 * G * 64 * sizeof(float);
            const bool exact = C * V == h / 8;
            const void* kern = cfg->dtype == SP_BF16 ? entry_kernel_t<__nv_bfloat16>(ln, exact)
                                                     : entry_kernel_t<float>(ln, exact);
            const int grid = (int)(rows < dev.sms ? rows : dev.sms);
            return launch_kernel(kern, grid, G * C, smem, st, &e);
        }
    }

    if (h % 8 == 0 && all16) {
        const FastLaunch L = plan_fwd(a, dev, E, cfg->fwd_plan);
        if (L.plan >= 0) {
            const void* kern = fwd_kernel_of(cfg->dtype, ln, L.plan, L.exact);
            if (L.cs > 1) {
                int grid = 0;
                return launch_clusters(kern, rows, L.cs, L.block, L.smem, st, &a, &grid);
            }
            return launch_kernel(kern, L.grid, L.block, L.smem, st, &a);
        }
    }
    // general kernel: any h, element-aligned pointers
    const size_t smem = (size_t)h * 4 + (size_t)a.mask_row_bytes;
    if (smem > (size_t)dev.smem_optin - 1024) return SP_ERR_UNSUPPORTED;
    const int grid = (int)general_grid(rows, dev.sms);
    const void* kern;
    if (cfg->dtype == SP_BF16)
        kern = ln ? (const void*)k_fwd_general<__nv_bfloat16, true>
                  : (const void*)k_fwd_general<__nv_bfloat16, false>;
    else
        kern = ln ? (const void*)k_fwd_general<float, true>
                  : (const void*)k_fwd_general<float, false>;
    return launch_kernel(kern, grid, kGeneralThreads, smem, st, &a);
}

}  // namespace

namespace {
// ---------------------------------------------------------------------------
// Backward launch decision, shared by the two backward entry points and the
// workspace query: the kernel, its launch shape and the workspace slices
// (3 * h fp32 each) it writes.
// ---------------------------------------------------------------------------
constexpr int kBwdGeneralThreads = 1024;

struct BwdChoice {
    bool fast = false;
    FastLaunch L;            // fast kernel: plan, block, grid, shared memory
    long long slices = 0;    // workspace slices written
    size_t general_smem = 0;
};

// The shape fields of the backward's arguments (everything but pointers).
void bwd_shape(const sp_cfg* cfg, BwdArgs* a)
{
    memset(a, 0, sizeof(*a));
    long long row0 = 0, rows = 0;
    call_rows(cfg, &row0, &rows);
    const int h = (int)cfg->h;
    const int E = elem_bytes(cfg), Er = res_elem_bytes(cfg);
    a->rows = rows;
    a->row0 = row0;
    a->h = h;
    a->hv = h / 8;
    a->t = cfg->t;
    a->seg_bytes = (uint32_t)(h * E);
    a->res_seg_bytes = (uint32_t)(h * Er);
    a->res_f32 = Er != E ? 1 : 0;
    a->stage_stride = (uint32_t)round128(a->res_seg_bytes > a->seg_bytes ? a->res_seg_bytes
                                                                          : a->seg_bytes);
    a->mask_row_bytes = 4 * ((h + 31) / 32);
    a->inv_h = (float)(1.0 / (double)h);
    a->scale = 1.0f / (1.0f - cfg->p_drop);
}

// fast_ok: every [s,b,h] pointer is 16-byte aligned.  Fills the planner's
// fields of *a (stages, offsets, fold).  SP_ERR_UNSUPPORTED when no kernel
// takes the shape.
int choose_bwd(const sp_cfg* cfg, const DevInfo& dev, bool fast_ok, BwdArgs& a, BwdChoice* ch)
{
    *ch = BwdChoice();
    const int h = (int)cfg->h;
    if (fast_ok && h % 8 == 0) {
        const FastLaunch L = plan_bwd(a, dev, elem_bytes(cfg), cfg->bwd_plan);
        if (L.plan >= 0) {
            ch->fast = true;
            ch->L = L;
            // one slice per CTA (shared-memory sums, or tensor-memory sums
            // folded in the CTA), else one per consumer group
            ch->slices = (long long)L.grid *
                         ((kBwdPlans[L.plan].acc == 1 || a.fold) ? 1 : L.groups);
            return SP_OK;
        }
    }
    const size_t smem = (size_t)h * 4;
    if (smem > (size_t)dev.smem_optin - 1024) return SP_ERR_UNSUPPORTED;
    ch->general_smem = smem;
    ch->slices = a.rows < dev.sms ? a.rows : dev.sms;   // one CTA per SM at most
    return SP_OK;
}

int noalloc_scratch(int dev, size_t need, void** out);

// The backward; workspace == nullptr takes the scratch from the library's
// fixed device array (sp_rs_norm_dropout_bwd_noalloc).
int bwd_impl(const sp_cfg* cfg, const void* const* dn_partials, const void* dR_next,
             const void* residual_out, const void* gamma, const uint32_t* mask_bits,
             const float* mean, const float* rstd, void* dresidual_in, void* const* dY,
             int n_dY, float* dgamma, float* dbeta, float* dbias, void* workspace,
             size_t workspace_bytes, void* stream)
{
    int rc = check_cfg(cfg);
    if (rc) return rc;
    const bool ln = cfg->norm == SP_LAYERNORM;
    if (!dn_partials || !residual_out || !gamma || !rstd || !dresidual_in || !dgamma)
        return SP_ERR_INVALID_ARG;
    if (ln && !mean) return SP_ERR_INVALID_ARG;
    if (!mask_bits && cfg->p_drop > 0.0f) return SP_ERR_INVALID_ARG;
    const int E = elem_bytes(cfg);
    bool all16 = true;
    for (int k = 0; k < cfg->t; ++k) {
        if (!dn_partials[k] || !aligned(dn_partials[k], E)) return SP_ERR_INVALID_ARG;
        all16 = all16 && aligned(dn_partials[k], 16);
    }
    const int Er = res_elem_bytes(cfg);
    if (n_dY < 0 || n_dY > SP_MAX_T || (n_dY > 0 && !dY)) return SP_ERR_INVALID_ARG;
    for (int q = 0; q < n_dY; ++q) {
        if (!dY[q] || !aligned(dY[q], E)) return SP_ERR_INVALID_ARG;
        all16 = all16 && aligned(dY[q], 16);
    }
    if (!aligned(gamma, E)) return SP_ERR_INVALID_ARG;
    all16 = all16 && aligned(gamma, 16);
    for (const void* p : {dR_next, residual_out, (const void*)dresidual_in}) {   // residual stream
        if (p && !aligned(p, Er)) return SP_ERR_INVALID_ARG;
        all16 = all16 && (!p || aligned(p, 16));
    }
    const void* f4_ptrs[] = {mask_bits, mean, rstd, dgamma, dbeta, dbias};
    for (const void* p : f4_ptrs)
        if (p && !aligned(p, 4)) return SP_ERR_INVALID_ARG;
    if (workspace && !aligned(workspace, 16)) return SP_ERR_INVALID_ARG;

    DevInfo dev;
    if ((rc = use_device_of(residual_out, &dev))) return rc;

    const int h = (int)cfg->h;
    BwdArgs a;
    bwd_shape(cfg, &a);
    BwdChoice ch;
    if ((rc = choose_bwd(cfg, dev, all16, a, &ch))) return rc;
    const size_t need = (size_t)ch.slices * 3 * h * sizeof(float);
    if (!workspace) {
        if ((rc = noalloc_scratch(dev.id, need, &workspace))) return rc;
    } else if (need > workspace_bytes) {
        return SP_ERR_INVALID_ARG;
    }
    for (int k = 0; k < cfg->t; ++k) a.dparts[k] = dn_partials[k];
    a.drnext = dR_next;
    a.x = residual_out;
    a.gamma = gamma;
    a.mask = reinterpret_cast<const uint8_t*>(mask_bits);
    a.mean = ln ? mean : nullptr;
    a.rstd = rstd;
    a.dres = dresidual_in;
    for (int q = 0; q < n_dY; ++q) a.dY[q] = dY[q];
    a.n_dY = n_dY;
    a.ws = static_cast<float*>(workspace);
    a.want_dbeta = (ln && dbeta) ? 1 : 0;
    a.want_dbias = dbias ? 1 : 0;
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    if (ch.fast) {
        const void* kern = bwd_kernel_of(cfg->dtype, ln, ch.L.plan, ch.L.exact);
        if ((rc = launch_kernel(kern, ch.L.grid, ch.L.block, ch.L.smem, st, &a))) return rc;
    } else {
        const void* kern;
        if (cfg->dtype == SP_BF16)
            kern = ln ? (const void*)k_bwd_general<__nv_bfloat16, true>
                      : (const void*)k_bwd_general<__nv_bfloat16, false>;
        else
            kern = ln ? (const void*)k_bwd_general<float, true>
                      : (const void*)k_bwd_general<float, false>;
        if ((rc = launch_kernel(kern, (int)ch.slices, kBwdGeneralThreads, ch.general_smem, st,
                                &a)))
            return rc;
    }
    const int tiles = (h + 31) / 32;
    const float* ws_c = a.ws;
    int nparts = (int)ch.slices, hh = h;
    float* outs[3] = {dgamma, a.want_dbeta ? dbeta : nullptr, a.want_dbias ? dbias : nullptr};
    void* params[] = {&ws_c, &nparts, &hh, &outs[0], &outs[1], &outs[2]};
    return launch_kernel_args((const void*)k_colreduce, 3 * tiles, kColreduceWarps * 32, 0, st,
                              params);
}

}  // namespace

extern "C" {

int sp_rs_bias_dropout_add_norm_fwd(const sp_cfg* cfg, const void* const* partials,
                                    const void* bias, const void* residual, const void* gamma,
                                    const void* beta, void* residual_out, void* const* gathered,
                                    int32_t n_gathered, uint32_t* mask_bits, float* mean,
                                    float* rstd, void* stream)
{
    if (!cfg) return SP_ERR_INVALID_ARG;
    return fwd_impl(cfg, cfg->t, partials, bias, residual, gamma, beta, residual_out, gathered,
                    n_gathered, mask_bits, mean, rstd, stream);
}

int sp_norm_all_gather_fwd(const sp_cfg* cfg, const void* x, const void* gamma,
                           const void* beta, void* const* gathered, int32_t n_gathered,
                           float* mean, float* rstd, void* stream)
{
    if (!cfg) return SP_ERR_INVALID_ARG;
    sp_cfg c = *cfg;
    c.p_drop = 0.0f;   // the entry has no dropout
    return fwd_impl(&c, 0, nullptr, nullptr, x, gamma, beta, nullptr, gathered, n_gathered,
                    nullptr, mean, rstd, stream);
}

int sp_linear_rs_bias_dropout_add_norm_fwd(const sp_cfg* cfg, int64_t f, const void* x,
                                           const void* w, const void* bias,
                                           const void* residual, const void* gamma,
                                           const void* beta, void* residual_out,
                                           void* const* gathered, int32_t n_gathered,
                                           uint32_t* mask_bits, float* mean, float* rstd,
                                           void* stream)
{
    if (!cfg || !gamma || !gathered || n_gathered < 1 || n_gathered > SP_MAX_T)
        return SP_ERR_INVALID_ARG;
    int rc = sp_rowpar_linear_rs_fwd(cfg, f, x, w, bias, residual, residual_out, mask_bits,
                                     stream);
    if (rc) return rc;
    // the stored residual sum is the norm's input; the entry kernel
    // normalises each row and writes it to every gathered buffer
    sp_cfg c = *cfg;
    c.fwd_plan = 0;
    return sp_norm_all_gather_fwd(&c, residual_out, gamma, beta, gathered, n_gathered, mean,
                                  rstd, stream);
}

int sp_all_gather(const sp_cfg* cfg, const void* const* shards, void* const* outs,
                  int32_t n_out, void* stream)
{
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if (!shards || !outs || n_out < 1 || n_out > SP_MAX_T) return SP_ERR_INVALID_ARG;
    const int E = elem_bytes(cfg);
    const long long rows = cfg->s * cfg->b;
    const long long shard_elems = rows / cfg->t * cfg->h;
    const long long shard_bytes = shard_elems * E;
    bool vec = (shard_bytes % 16) == 0;
    for (int r = 0; r < cfg->t; ++r) {
        if (!shards[r] || !aligned(shards[r], E)) return SP_ERR_INVALID_ARG;
        vec = vec && aligned(shards[r], 16);
    }
    for (int q = 0; q < n_out; ++q) {
        if (!outs[q] || !aligned(outs[q], E)) return SP_ERR_INVALID_ARG;
        vec = vec && aligned(outs[q], 16);
    }
    DevInfo dev;
    if ((rc = use_device_of(shards[0], &dev))) return rc;
    GatherArgs a;
    memset(&a, 0, sizeof(a));
    for (int r = 0; r < cfg->t; ++r) a.shards[r] = shards[r];
    for (int q = 0; q < n_out; ++q) a.outs[q] = outs[q];
    a.t = cfg->t;
    a.n_out = n_out;
    a.unit_bytes = vec ? 16 : E;
    a.shard_units = shard_bytes / a.unit_bytes;
    if (vec) {
        // bulk copies through shared memory, one issuing thread per SM
        const long long chunks =
            (shard_bytes + kAgChunk - 1) / kAgChunk * (long long)cfg->t;
        if (chunks < 1) return SP_OK;
        const size_t smem = (size_t)kAgSlots * kAgChunk;
        if (smem > (size_t)dev.smem_optin) return SP_ERR_UNSUPPORTED;
        const void* kern = (const void*)k_all_gather_bulk;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess) {
            cudaGetLastError();
            return SP_ERR_CUDA;
        }
        const int grid = (int)(chunks < dev.sms ? chunks : dev.sms);
        return launch_kernel(kern, grid, 32, smem, static_cast<cudaStream_t>(stream), &a);
    }
    const long long total = a.shard_units * a.t;
    long long grid = (total + 511) / 512;
    const long long cap = (long long)dev.sms * 4;
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    // unaligned buffers: the element-wise copy
    const void* kern = E == 4 ? (const void*)k_all_gather<uint32_t>
                              : (const void*)k_all_gather<uint16_t>;
    return launch_kernel(kern, (int)grid, 512, 0, static_cast<cudaStream_t>(stream), &a);
}

int sp_bwd_workspace_bytes(const sp_cfg* cfg, int32_t device, size_t* bytes)
{
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if (!bytes) return SP_ERR_INVALID_ARG;
    DevInfo dev;
    dev.id = device;
    if (cudaDeviceGetAttribute(&dev.sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess ||
        cudaDeviceGetAttribute(&dev.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin,
                               device) != cudaSuccess) {
        cudaGetLastError();
        return SP_ERR_CUDA;
    }
    // the slices of the kernel the backward picks for 16-byte aligned
    // pointers, or of the general kernel (misaligned pointers), whichever is
    // larger
    BwdArgs a;
    bwd_shape(cfg, &a);
    BwdChoice fast, general;
    const int rf = choose_bwd(cfg, dev, true, a, &fast);
    const int rg = choose_bwd(cfg, dev, false, a, &general);
    if (rf && rg) return rf;
    long long slices = rf ? 0 : fast.slices;
    if (!rg && general.slices > slices) slices = general.slices;
    *bytes = (size_t)slices * 3 * (size_t)cfg->h * sizeof(float);
    return SP_OK;
}

int sp_rs_norm_dropout_bwd(const sp_cfg* cfg, const void* const* dn_partials,
                           const void* dR_next, const void* residual_out, const void* gamma,
                           const uint32_t* mask_bits, const float* mean, const float* rstd,
                           void* dresidual_in, void* dY, float* dgamma, float* dbeta,
                           float* dbias, void* workspace, size_t workspace_bytes, void* stream)
{
    if (!workspace) return SP_ERR_INVALID_ARG;
    return bwd_impl(cfg, dn_partials, dR_next, residual_out, gamma, mask_bits, mean, rstd,
                    dresidual_in, &dY, dY ? 1 : 0, dgamma, dbeta, dbias, workspace,
                    workspace_bytes, stream);
}

int sp_rs_norm_dropout_bwd_ag(const sp_cfg* cfg, const void* const* dn_partials,
                              const void* dR_next, const void* residual_out, const void* gamma,
                              const uint32_t* mask_bits, const float* mean, const float* rstd,
                              void* dresidual_in, void* const* dY, int32_t n_dY, float* dgamma,
                              float* dbeta, float* dbias, void* workspace,
                              size_t workspace_bytes, void* stream)
{
    if (!workspace || n_dY < 1) return SP_ERR_INVALID_ARG;
    return bwd_impl(cfg, dn_partials, dR_next, residual_out, gamma, mask_bits, mean, rstd,
                    dresidual_in, dY, n_dY, dgamma, dbeta, dbias, workspace, workspace_bytes,
                    stream);
}

int sp_device_error(int32_t device, int32_t* code, int32_t clear)
{
    if (!code) return SP_ERR_INVALID_ARG;
    if (cudaSetDevice(device) != cudaSuccess) {
        cudaGetLastError();
        return SP_ERR_INVALID_ARG;
    }
    // every unit's word, in a fixed order; the first nonzero one is reported
    int (*const words[])(unsigned*, int) = {
        error_word_host,         error_word_fwd_bf16_ln, error_word_fwd_bf16_rms,
        error_word_fwd_f32_ln,   error_word_fwd_f32_rms, error_word_bwd_bf16_ln,
        error_word_bwd_bf16_rms, error_word_bwd_f32_ln,  error_word_bwd_f32_rms,
        error_word_gemm};
    unsigned first = 0;
    for (auto fn : words) {
        unsigned v = 0;
        if (fn(&v, clear) != 0) {
            cudaGetLastError();
            return SP_ERR_CUDA;
        }
        if (!first) first = v;
    }
    *code = (int32_t)first;
    return SP_OK;
}

int sp_debug_wait_timeout(int64_t limit_ns, int32_t* status, void* stream)
{
    if (!status || limit_ns < 0 || limit_ns > 10000000000LL) return SP_ERR_INVALID_ARG;
    DevInfo dev;
    int rc = use_device_of(status, &dev);
    if (rc) return rc;
    unsigned long long lim = (unsigned long long)limit_ns;
    int* st = reinterpret_cast<int*>(status);
    void* params[] = {&lim, &st};
    return launch_kernel_args((const void*)k_wait_selftest, 1, 32, 0,
                              static_cast<cudaStream_t>(stream), params);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Backward without caller-provided scratch.
//
// Some callers cannot allocate device memory at the point where they run the
// backward: code inside a memory-capped arena that owns every byte, a
// runtime whose allocator must not be re-entered from this call, or a host
// loop that may not synchronise (cudaMalloc and cudaFree can synchronise the
// device).  For them the scratch of the parameter-gradient partial sums lives
// in one fixed array in this library's device image instead of a buffer they
// pass in.  The array is reserved on every GPU that loads the library and is
// held until the process exits.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;   // 64 MiB per GPU

}  // namespace

// Host code must not use this name as a device address: it is the host-side
// stand-in of the symbol.  Its device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchBytes / sizeof(float)];

namespace {

// Device address of the scratch array on device `dev`, which the caller has
// made current, once `need` bytes are known to fit.  The address is looked up
// on every call (cheap once the library's device code is loaded), so it stays
// right if the device's context is torn down and created again.
int noalloc_scratch(int dev, size_t need, void** out)
{
    (void)dev;
    if (need > kNoAllocScratchBytes) return SP_ERR_UNSUPPORTED;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
        cudaGetLastError();
        return SP_ERR_CUDA;
    }
    *out = p;
    return SP_OK;
}

}  // namespace

extern "C" int sp_rs_norm_dropout_bwd_noalloc(
    const sp_cfg* cfg, const void* const* dn_partials, const void* dR_next,
    const void* residual_out, const void* gamma, const uint32_t* mask_bits, const float* mean,
    const float* rstd, void* dresidual_in, void* dY, float* dgamma, float* dbeta, float* dbias,
    void* stream)
{
    // the backward picks its kernel for the actual pointers, then checks that
    // the slices that kernel writes fit the array
    return bwd_impl(cfg, dn_partials, dR_next, residual_out, gamma, mask_bits, mean, rstd,
                    dresidual_in, &dY, dY ? 1 : 0, dgamma, dbeta, dbias, nullptr, 0, stream);
}
