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
// would not fit.  With several consumer groups sharing that one set, the
// groups take turns in the CTA's row order (two turn barriers, one for each
// accumulating pass), so the sums keep a fixed order and stay bitwise
// deterministic while the groups' reduce-scatter phases overlap.
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
    long long rows;          // token rows of this call (local index i)
    long long row0;          // global index of local row 0: n = row0 + i
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

template <typename T, int V, int G, int MAXT, bool LN, bool ACC_SMEM>
__global__ void __launch_bounds__(MAXT, 1) k_bwd_tma(const __grid_constant__ BwdArgs a)
{
    using Vec = typename IO<T>::Vec;
    extern __shared__ __align__(128) unsigned char smem[];
    RingTail* tail = reinterpret_cast<RingTail*>(smem + a.tail_off);
    // gamma copy and, for ACC_SMEM, the per-CTA accumulators [3][2][hv][4]
    // fp32; every slot is private to the thread that owns its vector
    unsigned char* sgam = smem + a.param_off;
    float4* accs = reinterpret_cast<float4*>(smem + a.acc_off);
    volatile int* abort = &tail->abort;

    const int C = (blockDim.x - 32) / G;
    const int tid = threadIdx.x;
    const int S = a.stages;
    const int nsrc = a.t + 1 + (a.drnext ? 1 : 0);   // dP_k..., x, [dR_next]

    init_ring(tail, S, C / 32);

    if (tid >= G * C) {
        if (tid == G * C)
            ring_produce<G>(smem, tail, abort, a.rows, nsrc, a.seg_bytes, a.stage_stride, S,
                            [&](int k, long long i) -> const void* {
                                // upstream partials by global row; x and dR_next
                                // are this call's shard, by local row
                                if (k < a.t)
                                    return static_cast<const unsigned char*>(a.dparts[k]) +
                                           (size_t)(a.row0 + i) * a.seg_bytes;
                                return static_cast<const unsigned char*>(k == a.t ? a.x
                                                                                  : a.drnext) +
                                       (size_t)i * a.seg_bytes;
                            });
        return;
    }

    const int g = tid / C;
    const int c = tid - g * C;
    const int lane = tid & 31;
    const int bar_id = 1 + g;
    const int hv = a.hv;
    float ag[ACC_SMEM ? 1 : V][8], ab[ACC_SMEM ? 1 : V][8], ac[ACC_SMEM ? 1 : V][8];
#pragma unroll
    for (int i = 0; i < V; ++i) {
        const int v = c + i * C;
        if (g == 0 && v < hv) store_vec<T>(sgam, v, load_vec<T>(a.gamma, v));
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
    asm volatile("bar.sync %0, %1;" ::"r"(1 + kMaxGroups), "r"(G * C) : "memory");

    auto acc_add = [&](int q, int v, const float d[8]) {
        float4* p0 = &accs[((size_t)q * 2 + 0) * hv + v];
        float4* p1 = &accs[((size_t)q * 2 + 1) * hv + v];
        float4 x0 = *p0, x1 = *p1;
        x0.x += d[0]; x0.y += d[1]; x0.z += d[2]; x0.w += d[3];
        x1.x += d[4]; x1.y += d[5]; x1.z += d[6]; x1.w += d[7];
        *p0 = x0;
        *p1 = x1;
    };
    auto release_at = [&](uint32_t s_) {
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_addr(&tail->empty[s_]));
    };
    // Turns of the shared accumulators, passed around the groups in CTA row
    // order: when row j finishes pass q it arrives on turn[q][next group],
    // and row j waits on turn[q][its own group] for the completion that row
    // j-1 made.  Group g's k-th row (j = g + k*G) waits for completion k of
    // its barrier (k-1 for group 0, whose first row has no predecessor).  A
    // barrier's next completion needs this group's own turn first, so no
    // barrier ever runs two phases ahead of its waiter.
    constexpr bool kTurns = ACC_SMEM && (G > 1);
    auto take_turn = [&](int q, long long j) {
        if (!kTurns || j == 0) return;
        const long long k = (j - g) / G - (g == 0 ? 1 : 0);
        mbar_wait(smem_addr(&tail->turn[q][g]), (uint32_t)(k & 1), abort, ERR_WAIT_FULL);
    };
    auto pass_turn = [&](int q) {
        if (kTurns) {
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_addr(&tail->turn[q][g + 1 == G ? 0 : g + 1]));
        }
    };

    const uint32_t Sg = (uint32_t)(S / G);
    RingPos pos((uint32_t)g * Sg, 0, Sg);
    int parity = 0;
    for (long long j = g;; j += G, parity ^= 1) {
        const long long i_row = blockIdx.x + j * (long long)gridDim.x;   // local row
        if (i_row >= a.rows) break;
        const long long n = a.row0 + i_row;                                // global row
        // loads whose latency overlaps the reduction below
        const float rstd = a.rstd[i_row];
        const float mean = LN ? a.mean[i_row] : 0.f;
        uint32_t kb[V];
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const int v = c + i * C;
            kb[i] = (a.mask && v < hv) ? a.mask[(size_t)i_row * a.mask_row_bytes + v] : 0xFFu;
        }

        // reduce-scatter of the upstream gradient partials, k ascending, from +0
        float dn[V][8];
#pragma unroll
        for (int i = 0; i < V; ++i)
#pragma unroll
            for (int e = 0; e < 8; ++e) dn[i][e] = 0.f;
        for (int k = 0; k < a.t; ++k) {
            mbar_wait(smem_addr(&tail->full[pos.abs()]), pos.phase, abort, ERR_WAIT_FULL);
            const unsigned char* buf = smem + (size_t)pos.abs() * a.stage_stride;
#pragma unroll
            for (int i = 0; i < V; ++i) {
                const int v = c + i * C;
                if (v < hv) {
                    float f[8];
                    IO<T>::unpack(load_vec<T>(buf, v), f);
#pragma unroll
                    for (int e = 0; e < 8; ++e) dn[i][e] += f[e];
                }
            }
            release_at(pos.abs());
            pos.next(Sg);
        }

        // pass 1 over x: row sums of g and g*xhat; parameter-gradient partials
        mbar_wait(smem_addr(&tail->full[pos.abs()]), pos.phase, abort, ERR_WAIT_FULL);
        const uint32_t sx = pos.abs();
        const unsigned char* xb = smem + (size_t)sx * a.stage_stride;
        pos.next(Sg);
        take_turn(0, j);
        float sg = 0.f, sgx = 0.f;
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const int v = c + i * C;
            if (v < hv) {
                float xv[8], gm[8], dgm[8];
                IO<T>::unpack(load_vec<T>(xb, v), xv);
                IO<T>::unpack(load_vec<T>(sgam, v), gm);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float xh = LN ? (xv[e] - mean) * rstd : xv[e] * rstd;
                    const float gg = dn[i][e] * gm[e];
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
        pass_turn(0);
        float2 tot = make_float2(warp_sum(sg), warp_sum(sgx));
        {
            float2* red = reinterpret_cast<float2*>(tail->red[parity][g]);
            if (lane == 0) red[c >> 5] = tot;
            asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "r"(C) : "memory");
            tot = warps_total2(red, C >> 5);
        }
        const float mg = tot.x / a.h_f, mgx = tot.y / a.h_f;

        const unsigned char* rb = nullptr;
        uint32_t sr = 0;
        if (a.drnext) {
            mbar_wait(smem_addr(&tail->full[pos.abs()]), pos.phase, abort, ERR_WAIT_FULL);
            sr = pos.abs();
            rb = smem + (size_t)sr * a.stage_stride;
            pos.next(Sg);
        }

        // pass 2: input gradient, residual gradient, dropout backward
        take_turn(1, j);
        unsigned char* dres =
            static_cast<unsigned char*>(a.dres) + (size_t)i_row * a.seg_bytes;   // shard
        unsigned char* dy =
            static_cast<unsigned char*>(a.dY) + (size_t)n * a.seg_bytes;       // gathered
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const int v = c + i * C;
            if (v < hv) {
                float xv[8], gm[8], dr[8], dz[8], rn[8];
                IO<T>::unpack(load_vec<T>(xb, v), xv);
                IO<T>::unpack(load_vec<T>(sgam, v), gm);
                if (rb) {
                    IO<T>::unpack(load_vec<T>(rb, v), rn);
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e) rn[e] = 0.f;
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float xh = LN ? (xv[e] - mean) * rstd : xv[e] * rstd;
                    const float gg = dn[i][e] * gm[e];
                    const float dx = LN ? rstd * (gg - mg - xh * mgx) : rstd * (gg - xh * mgx);
                    dr[e] = dx + rn[e];
                    dz[e] = ((kb[i] >> e) & 1u) ? dr[e] * a.scale : 0.f;
                }
                store_vec<T>(dres, v, IO<T>::pack(dr));
                if (a.dY) store_vec<T>(dy, v, IO<T>::pack(dz));
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
        pass_turn(1);
        release_at(sx);
        if (rb) release_at(sr);
    }

    // partial sums -> workspace: register accumulators give one slice per
    // group ([cta * G + g][q][h]); the shared set gives one slice per CTA
    // ([cta][q][h]), written by group 0 once every group has finished
    if (ACC_SMEM) {
        if (G > 1) asm volatile("bar.sync %0, %1;" ::"r"(1 + kMaxGroups), "r"(G * C) : "memory");
        if (g != 0) return;
    }
    float* ws = a.ws + (ACC_SMEM ? (size_t)blockIdx.x : (size_t)blockIdx.x * G + g) * 3 * a.h;
#pragma unroll
    for (int i = 0; i < V; ++i) {
        const int v = c + i * C;
        if (v < hv) {
            for (int q = 0; q < 3; ++q) {
                float4 lo, hi;
                if (ACC_SMEM) {
                    lo = accs[((size_t)q * 2 + 0) * hv + v];
                    hi = accs[((size_t)q * 2 + 1) * hv + v];
                } else {
                    const float* s_ = q == 0 ? ag[ACC_SMEM ? 0 : i]
                                             : (q == 1 ? ab[ACC_SMEM ? 0 : i]
                                                       : ac[ACC_SMEM ? 0 : i]);
                    lo = make_float4(s_[0], s_[1], s_[2], s_[3]);
                    hi = make_float4(s_[4], s_[5], s_[6], s_[7]);
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

    for (long long i_row = blockIdx.x; i_row < a.rows; i_row += gridDim.x) {
        const long long n = a.row0 + i_row;              // global row
        const long long base = n * (long long)h;         // upstream partials, dY
        const long long lbase = i_row * (long long)h;    // this call's shard
        const float rstd = a.rstd[i_row];
        const float mean = LN ? a.mean[i_row] : 0.f;
        float sg = 0.f, sgx = 0.f;
        for (int j = threadIdx.x; j < h; j += blockDim.x) {
            float d = 0.f;
            for (int k = 0; k < a.t; ++k) d = (k == 0) ? IO<T>::load1(a.dparts[k], base + j)
                                                       : d + IO<T>::load1(a.dparts[k], base + j);
            dns[j] = d;
            const float xv = IO<T>::load1(a.x, lbase + j);
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
            const float xv = IO<T>::load1(a.x, lbase + j);
            const float xh = LN ? (xv - mean) * rstd : xv * rstd;
            const float gg = d * IO<T>::load1(a.gamma, j);
            const float dx = LN ? rstd * (gg - mg - xh * mgx) : rstd * (gg - xh * mgx);
            const float dr = dx + (a.drnext ? IO<T>::load1(a.drnext, lbase + j) : 0.f);
            IO<T>::store1(a.dres, lbase + j, dr);
            uint32_t keep = 1u;
            if (a.mask) keep = (a.mask[(size_t)i_row * a.mask_row_bytes + (j >> 3)] >> (j & 7)) & 1u;
            const float dz = keep ? dr * a.scale : 0.f;
            if (a.dY) IO<T>::store1(a.dY, base + j, dz);
            if (a.want_dbias) ws[2 * h + j] += dz;
        }
        __syncthreads();   // dns is rewritten by the next row
    }
}

// dgamma / dbeta / dbias: fixed-order sum of the per-CTA (per-group)
// partials.  A block covers 32 consecutive columns of one quantity: lane =
// column, warp w sums partials w, w+8, w+16, ... in order, then warp 0 adds
// the 8 warp totals in order.  Deterministic for a given partial count.
__global__ void __launch_bounds__(256)
    k_colreduce(const float* __restrict__ ws, int nparts, int h, float* dgamma, float* dbeta,
                float* dbias)
{
    __shared__ float part[8][33];
    const int tiles = (h + 31) / 32;
    const int q = blockIdx.x / tiles;
    const int j = (blockIdx.x - q * tiles) * 32 + (threadIdx.x & 31);
    const int w = threadIdx.x >> 5;
    float* out = q == 0 ? dgamma : (q == 1 ? dbeta : dbias);
    if (!out) return;   // uniform over the block
    float s = 0.f;
    if (j < h) {
        const float* p = ws + (size_t)q * h + j;
        const size_t stride = (size_t)3 * h;
        int k = w;
        for (; k + 24 < nparts; k += 32) {
            const float v0 = p[(size_t)k * stride], v1 = p[(size_t)(k + 8) * stride];
            const float v2 = p[(size_t)(k + 16) * stride], v3 = p[(size_t)(k + 24) * stride];
            s += v0;
            s += v1;
            s += v2;
            s += v3;
        }
        for (; k < nparts; k += 8) s += p[(size_t)k * stride];
    }
    part[w][threadIdx.x & 31] = s;
    __syncthreads();
    if (w == 0 && j < h) {
        float t = 0.f;
        for (int i = 0; i < 8; ++i) t += part[i][threadIdx.x];
        out[j] = t;
    }
}

}  // namespace spk
