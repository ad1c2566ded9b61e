// Backward of the SP boundary on sm_100a.
//
// The backward of an all-gather is a reduce-scatter and the backward of a
// reduce-scatter is an all-gather ("Sequence Parallelism math", section "The
// collective substitution": the backward pass swaps the two).  Per token row
// n: dn = sum_k dP_k (reduce-scatter of the upstream partial gradients), the
// norm backward from the stored residual sum x and its mean / rstd, the
// residual-stream gradient, the dropout backward from the stored keep bits,
// and dY written in the gathered [s,b,h] layout.  dgamma / dbeta / dbias are
// sums over all rows: per-CTA fp32 partials in a fixed row order, then
// k_colreduce sums the CTAs in index order.
//
// k_bwd_tma mirrors k_fwd_tma: a producer lane streams the t gradient
// partial rows, the x row and (optionally) the dR_next row into a ring of
// shared-memory stages with cp.async.bulk; consumer threads own 8-feature
// vectors.  The x stage is held while the row is processed (it is read twice)
// so the row never sits in registers.  ACC_SMEM keeps the per-CTA parameter
// gradient partials in shared memory when 3 * 8V fp32 registers per thread
// would not fit.
#pragma once

#include "sp_device.cuh"
#include "sp_fwd.cuh"

namespace spk {

struct BwdArgs {
    const void* dparts[kMaxT];
    const void* drnext;
    const void* x;
    const void* gamma;
    const uint8_t* mask;     // bytes: [rows][mask_row_bytes]; NULL: keep all
    const float* mean;
    const float* rstd;
    void* dres;
    void* dY;
    float* ws;               // [gridDim.x][3][h] per-CTA partial sums
    long long rows;
    int h;
    int hv;
    int t;
    int stages;
    uint32_t seg_bytes;
    uint32_t stage_stride;
    int mask_row_bytes;
    uint32_t param_off;      // shared-memory offsets (fast kernel): gamma copy,
    uint32_t acc_off;        //   parameter-gradient accumulators (ACC_SMEM),
    uint32_t tail_off;       //   barriers / scratch
    float h_f;
    float scale;
    int want_dbeta;
    int want_dbias;
};

template <typename T, int V, bool LN, bool ACC_SMEM>
__global__ void __launch_bounds__(kFwdMaxConsumers + 32, 1)
    k_bwd_tma(const __grid_constant__ BwdArgs a)
{
    using Vec = typename IO<T>::Vec;
    extern __shared__ __align__(128) unsigned char smem[];
    RingTail* tail = reinterpret_cast<RingTail*>(smem + a.tail_off);
    // gamma copy (thread-private slots) and, for ACC_SMEM, the per-CTA
    // accumulators [3][2][hv][4] fp32, also thread-private
    unsigned char* sgam = smem + a.param_off;
    float4* accs = reinterpret_cast<float4*>(smem + a.acc_off);
    volatile int* abort = &tail->abort;

    const int C = blockDim.x - 32;
    const int tid = threadIdx.x;
    const int S = a.stages;
    const int nsrc = a.t + 1 + (a.drnext ? 1 : 0);

    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(smem_addr(&tail->full[s]), 1);
            mbar_init(smem_addr(&tail->empty[s]), C / 32);
        }
        tail->abort = 0;
        mbar_init_fence();
    }
    __syncthreads();

    // ------------------------------------------------------------------ producer
    if (tid >= C) {
        if (tid != C) return;
        const uint64_t pol = policy_evict_first();
        uint32_t stage = 0, phase = 1;
        long long issued = 0;
        bool ok = true;
        for (long long n = blockIdx.x; n < a.rows && ok; n += gridDim.x) {
            for (int k = 0; k < nsrc; ++k) {
                if (!mbar_wait(smem_addr(&tail->empty[stage]), phase, abort, ERR_WAIT_EMPTY)) {
                    ok = false;
                    break;
                }
                const void* base = k < a.t ? a.dparts[k] : (k == a.t ? a.x : a.drnext);
                const unsigned char* src =
                    static_cast<const unsigned char*>(base) + (size_t)n * a.seg_bytes;
                const uint32_t bar = smem_addr(&tail->full[stage]);
                mbar_arrive_expect_tx(bar, a.seg_bytes);
                bulk_load(smem_addr(smem + (size_t)stage * a.stage_stride), src, a.seg_bytes,
                          bar, pol);
                ++issued;
                if (++stage == (uint32_t)S) {
                    stage = 0;
                    phase ^= 1;
                }
            }
        }
        if (!ok) {
            long long first = issued > S ? issued - S : 0;
            for (long long i = first; i < issued; ++i) {
                const uint32_t s = (uint32_t)(i % S);
                const uint32_t par = (uint32_t)((i / S) & 1);
                volatile int no_abort = 0;
                if (!mbar_wait(smem_addr(&tail->full[s]), par, &no_abort, ERR_DRAIN)) break;
            }
        }
        return;
    }

    // ------------------------------------------------------------------ consumers
    const int lane = tid & 31;
    const int hv = a.hv;
    float ag[ACC_SMEM ? 1 : V][8], ab[ACC_SMEM ? 1 : V][8], ac[ACC_SMEM ? 1 : V][8];
#pragma unroll
    for (int i = 0; i < V; ++i) {
        const int v = tid + i * C;
        if (v < hv) store_vec<T>(sgam, v, load_vec<T>(a.gamma, v));
        if (!ACC_SMEM) {
#pragma unroll
            for (int e = 0; e < 8; ++e) ag[i][e] = ab[i][e] = ac[i][e] = 0.f;
        } else if (v < hv) {
#pragma unroll
            for (int q = 0; q < 3; ++q) {
                accs[((size_t)q * 2 + 0) * hv + v] = make_float4(0.f, 0.f, 0.f, 0.f);
                accs[((size_t)q * 2 + 1) * hv + v] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
    }
    // thread-private read-modify-write of the shared accumulators
    auto acc_add = [&](int q, int v, const float d[8]) {
        float4* p0 = &accs[((size_t)q * 2 + 0) * hv + v];
        float4* p1 = &accs[((size_t)q * 2 + 1) * hv + v];
        float4 x0 = *p0, x1 = *p1;
        x0.x += d[0]; x0.y += d[1]; x0.z += d[2]; x0.w += d[3];
        x1.x += d[4]; x1.y += d[5]; x1.z += d[6]; x1.w += d[7];
        *p0 = x0;
        *p1 = x1;
    };

    uint32_t stage = 0, phase = 0;
    auto advance = [&]() {
        if (++stage == (uint32_t)S) {
            stage = 0;
            phase ^= 1;
        }
    };
    auto release_at = [&](uint32_t s) {
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_addr(&tail->empty[s]));
    };

    for (long long n = blockIdx.x; n < a.rows; n += gridDim.x) {
        // loads whose latency overlaps the reduction below
        const float rstd = a.rstd[n];
        const float mean = LN ? a.mean[n] : 0.f;
        uint32_t kb[V];
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const int v = tid + i * C;
            kb[i] = (a.mask && v < hv) ? a.mask[(size_t)n * a.mask_row_bytes + v] : 0xFFu;
        }

        // reduce-scatter of the upstream gradient partials
        float dn[V][8];
        for (int k = 0; k < a.t; ++k) {
            mbar_wait(smem_addr(&tail->full[stage]), phase, abort, ERR_WAIT_FULL);
            const unsigned char* buf = smem + (size_t)stage * a.stage_stride;
#pragma unroll
            for (int i = 0; i < V; ++i) {
                const int v = tid + i * C;
                if (v < hv) {
                    float f[8];
                    IO<T>::unpack(load_vec<T>(buf, v), f);
#pragma unroll
                    for (int e = 0; e < 8; ++e) dn[i][e] = (k == 0) ? f[e] : dn[i][e] + f[e];
                }
            }
            release_at(stage);
            advance();
        }

        // pass 1 over x: row sums of g and g*xhat; parameter-gradient partials
        mbar_wait(smem_addr(&tail->full[stage]), phase, abort, ERR_WAIT_FULL);
        const uint32_t sx = stage;
        const unsigned char* xb = smem + (size_t)sx * a.stage_stride;
        advance();
        float sg = 0.f, sgx = 0.f;
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const int v = tid + i * C;
            if (v < hv) {
                float xv[8], g[8], dgm[8];
                IO<T>::unpack(load_vec<T>(xb, v), xv);
                IO<T>::unpack(load_vec<T>(sgam, v), g);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float xh = LN ? (xv[e] - mean) * rstd : xv[e] * rstd;
                    const float gg = dn[i][e] * g[e];
                    sg += gg;
                    sgx += gg * xh;
                    dgm[e] = dn[i][e] * xh;
                }
                if (ACC_SMEM) {
                    acc_add(0, v, dgm);
                    if (a.want_dbeta) acc_add(1, v, dn[i]);
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        ag[ACC_SMEM ? 0 : i][e] += dgm[e];
                        ab[ACC_SMEM ? 0 : i][e] += dn[i][e];
                    }
                }
            }
        }
        const float2 tot = consumer_sum2(make_float2(sg, sgx),
                                         reinterpret_cast<float2*>(tail->red0), C);
        const float mg = tot.x / a.h_f, mgx = tot.y / a.h_f;

        const unsigned char* rb = nullptr;
        uint32_t sr = 0;
        if (a.drnext) {
            mbar_wait(smem_addr(&tail->full[stage]), phase, abort, ERR_WAIT_FULL);
            sr = stage;
            rb = smem + (size_t)sr * a.stage_stride;
            advance();
        }

        // pass 2: input gradient, residual gradient, dropout backward
        unsigned char* dres = static_cast<unsigned char*>(a.dres) + (size_t)n * a.seg_bytes;
        unsigned char* dy = static_cast<unsigned char*>(a.dY) + (size_t)n * a.seg_bytes;
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const int v = tid + i * C;
            if (v < hv) {
                float xv[8], g[8], dr[8], dz[8];
                IO<T>::unpack(load_vec<T>(xb, v), xv);
                IO<T>::unpack(load_vec<T>(sgam, v), g);
                float rn[8];
                if (rb) {
                    IO<T>::unpack(load_vec<T>(rb, v), rn);
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e) rn[e] = 0.f;
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float xh = LN ? (xv[e] - mean) * rstd : xv[e] * rstd;
                    const float gg = dn[i][e] * g[e];
                    const float dx = LN ? rstd * (gg - mg - xh * mgx) : rstd * (gg - xh * mgx);
                    dr[e] = dx + rn[e];
                    dz[e] = ((kb[i] >> e) & 1u) ? dr[e] * a.scale : 0.f;
                }
                store_vec<T>(dres, v, IO<T>::pack(dr));
                store_vec<T>(dy, v, IO<T>::pack(dz));
                if (a.want_dbias) {
                    if (ACC_SMEM) {
                        acc_add(2, v, dz);
                    } else {
#pragma unroll
                        for (int e = 0; e < 8; ++e) ac[ACC_SMEM ? 0 : i][e] += dz[e];
                    }
                }
            }
        }
        release_at(sx);
        if (rb) release_at(sr);
    }

    // this CTA's partial sums -> workspace [cta][q][h]
    float* ws = a.ws + (size_t)blockIdx.x * 3 * a.h;
#pragma unroll
    for (int i = 0; i < V; ++i) {
        const int v = tid + i * C;
        if (v < hv) {
            for (int q = 0; q < 3; ++q) {
                float4 lo, hi;
                if (ACC_SMEM) {
                    lo = accs[((size_t)q * 2 + 0) * hv + v];
                    hi = accs[((size_t)q * 2 + 1) * hv + v];
                } else {
                    const float* s = q == 0 ? ag[ACC_SMEM ? 0 : i]
                                            : (q == 1 ? ab[ACC_SMEM ? 0 : i]
                                                      : ac[ACC_SMEM ? 0 : i]);
                    lo = make_float4(s[0], s[1], s[2], s[3]);
                    hi = make_float4(s[4], s[5], s[6], s[7]);
                }
                float4* dst = reinterpret_cast<float4*>(ws + (size_t)q * a.h + 8 * (size_t)v);
                dst[0] = lo;
                dst[1] = hi;
            }
        }
    }
}

// General backward: any h.  One CTA per row (grid stride); the reduced dn row
// lives in shared memory, the CTA's parameter-gradient partials in its own
// workspace slice (zeroed first, owned column by column by one thread each).
template <typename T, bool LN>
__global__ void __launch_bounds__(256) k_bwd_general(const __grid_constant__ BwdArgs a)
{
    extern __shared__ __align__(128) unsigned char smem[];
    float* dns = reinterpret_cast<float*>(smem);
    __shared__ float red[32];
    const int h = a.h;
    float* ws = a.ws + (size_t)blockIdx.x * 3 * h;
    for (int j = threadIdx.x; j < 3 * h; j += blockDim.x) ws[j] = 0.f;

    for (long long n = blockIdx.x; n < a.rows; n += gridDim.x) {
        const long long base = n * (long long)h;
        const float rstd = a.rstd[n];
        const float mean = LN ? a.mean[n] : 0.f;
        float sg = 0.f, sgx = 0.f;
        for (int j = threadIdx.x; j < h; j += blockDim.x) {
            float d = 0.f;
            for (int k = 0; k < a.t; ++k) d = (k == 0) ? IO<T>::load1(a.dparts[k], base + j)
                                                       : d + IO<T>::load1(a.dparts[k], base + j);
            dns[j] = d;
            const float xv = IO<T>::load1(a.x, base + j);
            const float xh = LN ? (xv - mean) * rstd : xv * rstd;
            const float gg = d * IO<T>::load1(a.gamma, j);
            sg += gg;
            sgx += gg * xh;
            ws[j] += d * xh;
            if (a.want_dbeta) ws[h + j] += d;
        }
        const float mg = block_sum(sg, red) / a.h_f;
        const float mgx = block_sum(sgx, red) / a.h_f;
        for (int j = threadIdx.x; j < h; j += blockDim.x) {
            const float d = dns[j];
            const float xv = IO<T>::load1(a.x, base + j);
            const float xh = LN ? (xv - mean) * rstd : xv * rstd;
            const float gg = d * IO<T>::load1(a.gamma, j);
            const float dx = LN ? rstd * (gg - mg - xh * mgx) : rstd * (gg - xh * mgx);
            const float dr = dx + (a.drnext ? IO<T>::load1(a.drnext, base + j) : 0.f);
            IO<T>::store1(a.dres, base + j, dr);
            uint32_t keep = 1u;
            if (a.mask) keep = (a.mask[(size_t)n * a.mask_row_bytes + (j >> 3)] >> (j & 7)) & 1u;
            const float dz = keep ? dr * a.scale : 0.f;
            IO<T>::store1(a.dY, base + j, dz);
            if (a.want_dbias) ws[2 * h + j] += dz;
        }
        __syncthreads();   // dns is rewritten by the next row
    }
}

// dgamma / dbeta / dbias: fixed-order sum of the per-CTA partials.
__global__ void __launch_bounds__(256)
    k_colreduce(const float* __restrict__ ws, int nparts, int h, float* dgamma, float* dbeta,
                float* dbias)
{
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= 3LL * h) return;
    const int q = (int)(idx / h), j = (int)(idx % h);
    float* out = q == 0 ? dgamma : (q == 1 ? dbeta : dbias);
    if (!out) return;
    const float* p = ws + (size_t)q * h + j;
    const size_t stride = (size_t)3 * h;
    float s = 0.f;
    int g = 0;
    for (; g + 8 <= nparts; g += 8) {
        float v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) v[u] = p[(size_t)(g + u) * stride];
#pragma unroll
        for (int u = 0; u < 8; ++u) s += v[u];
    }
    for (; g < nparts; ++g) s += p[(size_t)g * stride];
    out[j] = s;
}

}  // namespace spk
