// C-ABI entry points of the SP boundary library (declared in sp_region.h):
// argument validation, kernel selection and launch.  All device work goes
// through the kernels in sp_fwd.cuh, sp_bwd.cuh and sp_gather.cuh; nothing
// here computes on the host except the activation-memory closed forms.
#include <math.h>
#include <string.h>

#include "sp_region.h"
#include "sp_bwd.cuh"
#include "sp_device.cuh"
#include "sp_fwd.cuh"
#include "sp_gather.cuh"

using namespace spk;

namespace {

constexpr int kGeneralThreads = 256;
constexpr int kMaxV = 4;

struct DevInfo {
    int id;
    int sms;
    int smem_optin;
};

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
    return SP_OK;
}

int elem_bytes(const sp_cfg* c) { return c->dtype == SP_F32 ? 4 : 2; }

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

uint32_t drop_threshold(float p)
{
    return (uint32_t)floor((double)p * 4294967296.0);
}

int launch_status()
{
    return cudaGetLastError() == cudaSuccess ? SP_OK : SP_ERR_CUDA;
}

// Fast-kernel shape for a row of hv 8-feature vectors: V vectors per
// consumer thread, C consumer threads (multiple of 32, at most 512).
bool fast_shape(int hv, int* V, int* C)
{
    int v = (hv + kFwdMaxConsumers - 1) / kFwdMaxConsumers;
    if (v < 1) v = 1;
    if (v > kMaxV) return false;
    int c = (hv + v - 1) / v;
    c = (c + 31) / 32 * 32;
    *V = v;
    *C = c;
    return true;
}

template <typename T, bool LN>
int launch_fwd_fast(const FwdArgs& a, int V, int C, int grid, size_t smem, cudaStream_t st)
{
    auto pick = [&](auto kern) -> int {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem) != cudaSuccess)
            return SP_ERR_CUDA;
        kern<<<grid, C + 32, smem, st>>>(a);
        return launch_status();
    };
    switch (V) {
    case 1: return pick(k_fwd_tma<T, 1, LN>);
    case 2: return pick(k_fwd_tma<T, 2, LN>);
    case 3: return pick(k_fwd_tma<T, 3, LN>);
    default: return pick(k_fwd_tma<T, 4, LN>);
    }
}

template <typename T, bool LN>
int launch_bwd_fast(const BwdArgs& a, int V, int C, int grid, size_t smem, cudaStream_t st)
{
    auto pick = [&](auto kern) -> int {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem) != cudaSuccess)
            return SP_ERR_CUDA;
        kern<<<grid, C + 32, smem, st>>>(a);
        return launch_status();
    };
    switch (V) {
    case 1: return pick(k_bwd_tma<T, 1, LN, false>);
    case 2: return pick(k_bwd_tma<T, 2, LN, true>);
    case 3: return pick(k_bwd_tma<T, 3, LN, true>);
    default: return pick(k_bwd_tma<T, 4, LN, true>);
    }
}

size_t ring_tail_bytes() { return (sizeof(RingTail) + 127) & ~(size_t)127; }

size_t round128(size_t x) { return (x + 127) & ~(size_t)127; }

// accumulators in shared memory once a thread owns two or more vectors
bool bwd_acc_in_smem(int V) { return V >= 2; }

// Rows a general-kernel launch covers at once (grid), per device.
long long general_grid(long long rows, int sms)
{
    const long long g = (long long)sms * 4;
    return rows < g ? rows : g;
}

long long fast_grid(long long rows, int sms) { return rows < sms ? rows : sms; }

}  // namespace

extern "C" {

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

int sp_rs_bias_dropout_add_norm_fwd(const sp_cfg* cfg, const void* const* partials,
                                    const void* bias, const void* residual, const void* gamma,
                                    const void* beta, void* residual_out, void* const* gathered,
                                    int32_t n_gathered, uint32_t* mask_bits, float* mean,
                                    float* rstd, void* stream)
{
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if (!partials || !residual || !gamma || !residual_out || !gathered) return SP_ERR_INVALID_ARG;
    if (n_gathered < 1 || n_gathered > SP_MAX_T) return SP_ERR_INVALID_ARG;
    const int E = elem_bytes(cfg);
    const bool ln = cfg->norm == SP_LAYERNORM;
    bool all16 = true;
    for (int k = 0; k < cfg->t; ++k) {
        if (!partials[k] || !aligned(partials[k], E)) return SP_ERR_INVALID_ARG;
        all16 = all16 && aligned(partials[k], 16);
    }
    for (int q = 0; q < n_gathered; ++q) {
        if (!gathered[q] || !aligned(gathered[q], E)) return SP_ERR_INVALID_ARG;
        all16 = all16 && aligned(gathered[q], 16);
    }
    const void* elem_ptrs[] = {residual, gamma, residual_out, bias, ln ? beta : nullptr};
    for (const void* p : elem_ptrs) {
        if (p && !aligned(p, E)) return SP_ERR_INVALID_ARG;
        all16 = all16 && (!p || aligned(p, 16));
    }
    if ((mask_bits && !aligned(mask_bits, 4)) || (mean && !aligned(mean, 4)) ||
        (rstd && !aligned(rstd, 4)))
        return SP_ERR_INVALID_ARG;

    DevInfo dev;
    if ((rc = use_device_of(residual, &dev))) return rc;

    const long long rows = cfg->s * cfg->b;
    const int h = (int)cfg->h;
    FwdArgs a;
    memset(&a, 0, sizeof(a));
    for (int k = 0; k < cfg->t; ++k) a.parts[k] = partials[k];
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
    a.h = h;
    a.hv = h / 8;
    a.t = cfg->t;
    a.n_gathered = n_gathered;
    a.seg_bytes = (uint32_t)(h * E);
    a.stage_stride = (a.seg_bytes + 127u) & ~127u;
    a.mask_row_bytes = 4 * ((h + 31) / 32);
    a.eps = cfg->eps;
    a.h_f = (float)h;
    a.scale = 1.0f / (1.0f - cfg->p_drop);
    a.thr = drop_threshold(cfg->p_drop);
    a.seed_lo = (uint32_t)cfg->seed;
    a.seed_hi = (uint32_t)(cfg->seed >> 32);
    a.off_lo = (uint32_t)cfg->offset;
    a.off_hi = (uint32_t)(cfg->offset >> 32);
    a.dropout = cfg->p_drop > 0.0f ? 1 : 0;
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    int V = 0, C = 0;
    if (h % 8 == 0 && all16 && fast_shape(h / 8, &V, &C)) {
        const size_t tailb = ring_tail_bytes();
        const size_t pstride = round128((size_t)h * E);
        long long S = ((long long)dev.smem_optin - (long long)(tailb + 3 * pstride)) /
                      a.stage_stride;
        if (S > 64) S = 64;
        if (S >= 2) {
            a.stages = (int)S;
            a.param_off = (uint32_t)(S * a.stage_stride);
            a.param_stride = (uint32_t)pstride;
            a.tail_off = (uint32_t)(a.param_off + 3 * pstride);
            const size_t smem = (size_t)a.tail_off + tailb;
            const int grid = (int)fast_grid(rows, dev.sms);
            if (cfg->dtype == SP_BF16)
                return ln ? launch_fwd_fast<__nv_bfloat16, true>(a, V, C, grid, smem, st)
                          : launch_fwd_fast<__nv_bfloat16, false>(a, V, C, grid, smem, st);
            return ln ? launch_fwd_fast<float, true>(a, V, C, grid, smem, st)
                      : launch_fwd_fast<float, false>(a, V, C, grid, smem, st);
        }
    }
    // general kernel
    const size_t smem = (size_t)h * 4 + (size_t)a.mask_row_bytes;
    if (smem > (size_t)dev.smem_optin - 1024) return SP_ERR_UNSUPPORTED;
    const int grid = (int)general_grid(rows, dev.sms);
    auto go = [&](auto kern) -> int {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem) != cudaSuccess)
            return SP_ERR_CUDA;
        kern<<<grid, kGeneralThreads, smem, st>>>(a);
        return launch_status();
    };
    if (cfg->dtype == SP_BF16)
        return ln ? go(k_fwd_general<__nv_bfloat16, true>) : go(k_fwd_general<__nv_bfloat16, false>);
    return ln ? go(k_fwd_general<float, true>) : go(k_fwd_general<float, false>);
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
    const long long total = a.shard_units * a.t;
    long long grid = (total + 511) / 512;
    const long long cap = (long long)dev.sms * 4;
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (vec)
        k_all_gather<uint4><<<(int)grid, 512, 0, st>>>(a);
    else if (E == 4)
        k_all_gather<uint32_t><<<(int)grid, 512, 0, st>>>(a);
    else
        k_all_gather<uint16_t><<<(int)grid, 512, 0, st>>>(a);
    return launch_status();
}

int sp_bwd_workspace_bytes(const sp_cfg* cfg, int32_t device, size_t* bytes)
{
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if (!bytes) return SP_ERR_INVALID_ARG;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess) {
        cudaGetLastError();
        return SP_ERR_CUDA;
    }
    const long long rows = cfg->s * cfg->b;
    const long long g = general_grid(rows, sms);   // >= the fast kernel's grid
    *bytes = (size_t)g * 3 * (size_t)cfg->h * sizeof(float);
    return SP_OK;
}

int sp_rs_norm_dropout_bwd(const sp_cfg* cfg, const void* const* dn_partials,
                           const void* dR_next, const void* residual_out, const void* gamma,
                           const uint32_t* mask_bits, const float* mean, const float* rstd,
                           void* dresidual_in, void* dY, float* dgamma, float* dbeta,
                           float* dbias, void* workspace, size_t workspace_bytes, void* stream)
{
    int rc = check_cfg(cfg);
    if (rc) return rc;
    const bool ln = cfg->norm == SP_LAYERNORM;
    if (!dn_partials || !residual_out || !gamma || !rstd || !dresidual_in || !dY || !dgamma ||
        !workspace)
        return SP_ERR_INVALID_ARG;
    if (ln && !mean) return SP_ERR_INVALID_ARG;
    if (!mask_bits && cfg->p_drop > 0.0f) return SP_ERR_INVALID_ARG;
    const int E = elem_bytes(cfg);
    bool all16 = true;
    for (int k = 0; k < cfg->t; ++k) {
        if (!dn_partials[k] || !aligned(dn_partials[k], E)) return SP_ERR_INVALID_ARG;
        all16 = all16 && aligned(dn_partials[k], 16);
    }
    const void* elem_ptrs[] = {dR_next, residual_out, gamma, dresidual_in, dY};
    for (const void* p : elem_ptrs) {
        if (p && !aligned(p, E)) return SP_ERR_INVALID_ARG;
        all16 = all16 && (!p || aligned(p, 16));
    }
    const void* f4_ptrs[] = {mask_bits, mean, rstd, dgamma, dbeta, dbias};
    for (const void* p : f4_ptrs)
        if (p && !aligned(p, 4)) return SP_ERR_INVALID_ARG;
    if (!aligned(workspace, 16)) return SP_ERR_INVALID_ARG;

    DevInfo dev;
    if ((rc = use_device_of(residual_out, &dev))) return rc;

    const long long rows = cfg->s * cfg->b;
    const int h = (int)cfg->h;
    BwdArgs a;
    memset(&a, 0, sizeof(a));
    for (int k = 0; k < cfg->t; ++k) a.dparts[k] = dn_partials[k];
    a.drnext = dR_next;
    a.x = residual_out;
    a.gamma = gamma;
    a.mask = reinterpret_cast<const uint8_t*>(mask_bits);
    a.mean = ln ? mean : nullptr;
    a.rstd = rstd;
    a.dres = dresidual_in;
    a.dY = dY;
    a.ws = static_cast<float*>(workspace);
    a.rows = rows;
    a.h = h;
    a.hv = h / 8;
    a.t = cfg->t;
    a.seg_bytes = (uint32_t)(h * E);
    a.stage_stride = (a.seg_bytes + 127u) & ~127u;
    a.mask_row_bytes = 4 * ((h + 31) / 32);
    a.h_f = (float)h;
    a.scale = 1.0f / (1.0f - cfg->p_drop);
    a.want_dbeta = (ln && dbeta) ? 1 : 0;
    a.want_dbias = dbias ? 1 : 0;
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    int grid = 0;
    int V = 0, C = 0;
    bool launched = false;
    if (h % 8 == 0 && all16 && fast_shape(h / 8, &V, &C)) {
        const size_t tailb = ring_tail_bytes();
        const size_t pstride = round128((size_t)h * E);
        const size_t accb = bwd_acc_in_smem(V) ? (size_t)3 * 2 * a.hv * sizeof(float4) : 0;
        long long S = ((long long)dev.smem_optin - (long long)(tailb + pstride + accb)) /
                      a.stage_stride;
        if (S > 64) S = 64;
        if (S >= 2) {
            a.stages = (int)S;
            a.param_off = (uint32_t)(S * a.stage_stride);
            a.acc_off = (uint32_t)(a.param_off + pstride);
            a.tail_off = (uint32_t)(a.acc_off + accb);
            grid = (int)fast_grid(rows, dev.sms);
            if ((size_t)grid * 3 * h * sizeof(float) > workspace_bytes) return SP_ERR_INVALID_ARG;
            const size_t smem = (size_t)a.tail_off + tailb;
            if (cfg->dtype == SP_BF16)
                rc = ln ? launch_bwd_fast<__nv_bfloat16, true>(a, V, C, grid, smem, st)
                        : launch_bwd_fast<__nv_bfloat16, false>(a, V, C, grid, smem, st);
            else
                rc = ln ? launch_bwd_fast<float, true>(a, V, C, grid, smem, st)
                        : launch_bwd_fast<float, false>(a, V, C, grid, smem, st);
            if (rc) return rc;
            launched = true;
        }
    }
    if (!launched) {
        const size_t smem = (size_t)h * 4;
        if (smem > (size_t)dev.smem_optin - 1024) return SP_ERR_UNSUPPORTED;
        grid = (int)general_grid(rows, dev.sms);
        if ((size_t)grid * 3 * h * sizeof(float) > workspace_bytes) return SP_ERR_INVALID_ARG;
        auto go = [&](auto kern) -> int {
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)smem) != cudaSuccess)
                return SP_ERR_CUDA;
            kern<<<grid, kGeneralThreads, smem, st>>>(a);
            return launch_status();
        };
        if (cfg->dtype == SP_BF16)
            rc = ln ? go(k_bwd_general<__nv_bfloat16, true>) : go(k_bwd_general<__nv_bfloat16, false>);
        else
            rc = ln ? go(k_bwd_general<float, true>) : go(k_bwd_general<float, false>);
        if (rc) return rc;
    }
    const long long n = 3LL * h;
    k_colreduce<<<(int)((n + 255) / 256), 256, 0, st>>>(a.ws, grid, h, dgamma,
                                                        a.want_dbeta ? dbeta : nullptr,
                                                        a.want_dbias ? dbias : nullptr);
    return launch_status();
}

int sp_device_error(int32_t device, int32_t* code, int32_t clear)
{
    if (!code) return SP_ERR_INVALID_ARG;
    if (cudaSetDevice(device) != cudaSuccess) {
        cudaGetLastError();
        return SP_ERR_INVALID_ARG;
    }
    unsigned v = 0;
    if (cudaMemcpyFromSymbol(&v, g_error, sizeof(v)) != cudaSuccess) return SP_ERR_CUDA;
    *code = (int32_t)v;
    if (clear) {
        const unsigned zero = 0;
        if (cudaMemcpyToSymbol(g_error, &zero, sizeof(zero)) != cudaSuccess) return SP_ERR_CUDA;
    }
    return SP_OK;
}

int sp_debug_wait_timeout(int64_t limit_ns, int32_t* status, void* stream)
{
    if (!status || limit_ns < 0 || limit_ns > 10000000000LL) return SP_ERR_INVALID_ARG;
    DevInfo dev;
    int rc = use_device_of(status, &dev);
    if (rc) return rc;
    k_wait_selftest<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
        (unsigned long long)limit_ns, reinterpret_cast<int*>(status));
    return launch_status();
}

}  // extern "C"
