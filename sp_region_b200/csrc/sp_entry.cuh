// Entry into a tensor-parallel region on sm_100a: per-token norm of this
// rank's rows, then the all-gather ("SP: Partition Activations Alongside
// TP", section "Connect SP and TP across a layer": the norm runs on the
// sequence shard, and the gathered output feeds the column-parallel
// projections).
//
// k_norm_ag streams one row segment per token and has no partial sums to
// reduce, so it needs no staging ring: each thread loads its vectors of the
// row straight into registers (read-only, not kept in L1) and prefetches the
// same vectors of its group's next row while it normalises this one (the
// first row's loads are issued before gamma / beta are staged).  G consumer
// groups per CTA take every G-th row of the CTA; gamma / beta are copied to
// shared memory once.  The two row reductions (mean, then the centred second
// moment) are warp butterflies plus one value per warp through shared
// memory, double-buffered by row parity; the row is centred in place, so the
// output pass scales it directly.
#pragma once

#include "sp_device.cuh"
#include "sp_fwd.cuh"

namespace spk {

constexpr int kEntryThreads = 768;   // block bound: 85 registers per thread

struct EntryArgs {
    const void* x;           // [rows][h] this call's shard, by local row
    const void* gamma;
    const void* beta;        // NULL: no shift
    void* gathered[kMaxT];   // [N][h] replicas, by global row
    float* mean;             // [rows] or NULL
    float* rstd;             // [rows] or NULL
    long long rows;
    long long row0;          // global index of local row 0
    int hv;                  // h / 8
    int C;                   // threads per group (multiple of 32)
    int n_gathered;
    uint32_t seg_bytes;      // h * elem bytes
    uint32_t param_stride;   // shared-memory bytes per parameter copy
    float inv_h;
    float eps;
};

template <typename T>
__device__ __forceinline__ typename IO<T>::Vec ld_stream_vec(const void* base, long long v)
{
    typename IO<T>::Vec r;
    const uint4* p = static_cast<const uint4*>(base) + v * IO<T>::kWords;
#pragma unroll
    for (int k = 0; k < IO<T>::kWords; ++k)
        asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(r.u[k].x), "=r"(r.u[k].y), "=r"(r.u[k].z), "=r"(r.u[k].w)
                     : "l"(p + k));
    return r;
}

// EXACT: every thread owns V whole vectors (C * V == hv), no guards.
template <typename T, int V, bool LN, bool EXACT>
__global__ void __launch_bounds__(kEntryThreads, 1) k_norm_ag(const __grid_constant__ EntryArgs a)
{
    using Vec = typename IO<T>::Vec;
    extern __shared__ __align__(128) unsigned char smem[];
    const int hv = a.hv, C = a.C;
    const int G = blockDim.x / C;
    const int tid = threadIdx.x;
    const int g = tid / C, c = tid - g * C, lane = tid & 31;
    unsigned char* sg = smem;
    unsigned char* sb = smem + a.param_stride;
    float* red = reinterpret_cast<float*>(smem + 2 * a.param_stride);   // [2][G][2][32]
    const bool has_beta = LN && a.beta;
    auto valid = [&](int k) { return EXACT || c + k * C < hv; };
    const long long step = (long long)G * gridDim.x;
    long long i = blockIdx.x + (long long)g * gridDim.x;   // local row
    Vec nxt[V];
    auto fetch = [&](long long row) {
        const unsigned char* src = static_cast<const unsigned char*>(a.x) + row * a.seg_bytes;
#pragma unroll
        for (int k = 0; k < V; ++k)
            if (valid(k)) nxt[k] = ld_stream_vec<T>(src, c + k * C);
    };
    grid_dep_launch();
    grid_dep_wait();   // the previous kernel's outputs are visible
    if (i < a.rows) fetch(i);   // in flight while the parameters are staged
    for (int v = tid; v < hv; v += blockDim.x) {
        store_vec<T>(sg, v, load_vec<T>(a.gamma, v));
        if (has_beta) store_vec<T>(sb, v, load_vec<T>(a.beta, v));
    }
    __syncthreads();
    auto group_sum = [&](float x, float* slot) {
        x = warp_sum(x);
        if (lane == 0) slot[c >> 5] = x;
        asm volatile("bar.sync %0, %1;" ::"r"(1 + g), "r"(C) : "memory");
        return warps_total(slot, C >> 5);
    };
    for (int parity = 0; i < a.rows; i += step, parity ^= 1) {
        F2 acc[V][4];
#pragma unroll
        for (int k = 0; k < V; ++k)
            if (valid(k)) IO<T>::unpack2(nxt[k], acc[k]);
        if (i + step < a.rows) fetch(i + step);
        float* slots = red + (size_t)(parity * G + g) * 64;

        float mean = 0.f, rstd;
        if (LN) {
            F2 s2 = f2(0.f);
#pragma unroll
            for (int k = 0; k < V; ++k)
                if (valid(k))
#pragma unroll
                    for (int p = 0; p < 4; ++p) s2 = add2(s2, acc[k][p]);
            mean = group_sum(hsum(s2), slots) * a.inv_h;
            const F2 mean2 = f2(mean);
            F2 q2 = f2(0.f);
#pragma unroll
            for (int k = 0; k < V; ++k)
                if (valid(k))
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        acc[k][p] = sub2(acc[k][p], mean2);   // centred in place
                        q2 = fma2(acc[k][p], acc[k][p], q2);
                    }
            rstd = rsqrtf(group_sum(hsum(q2), slots + 32) * a.inv_h + a.eps);
        } else {
            F2 q2 = f2(0.f);
#pragma unroll
            for (int k = 0; k < V; ++k)
                if (valid(k))
#pragma unroll
                    for (int p = 0; p < 4; ++p) q2 = fma2(acc[k][p], acc[k][p], q2);
            rstd = rsqrtf(group_sum(hsum(q2), slots) * a.inv_h + a.eps);
        }

        const F2 rstd2 = f2(rstd);
        const size_t orow = (size_t)(a.row0 + i) * a.seg_bytes;   // gathered: global row
#pragma unroll
        for (int k = 0; k < V; ++k) {
            if (!valid(k)) continue;
            const int v = c + k * C;
            F2 gm[4], o[4];
            IO<T>::unpack2(load_vec<T>(sg, v), gm);
            if (has_beta) {
                F2 b[4];
                IO<T>::unpack2(load_vec<T>(sb, v), b);
#pragma unroll
                for (int p = 0; p < 4; ++p) o[p] = fma2(mul2(acc[k][p], rstd2), gm[p], b[p]);
            } else {
#pragma unroll
                for (int p = 0; p < 4; ++p) o[p] = mul2(mul2(acc[k][p], rstd2), gm[p]);
            }
            const Vec ov = IO<T>::pack2v(o);
            store_vec<T>(static_cast<unsigned char*>(a.gathered[0]) + orow, v, ov);
            for (int q = 1; q < a.n_gathered; ++q)
                store_vec<T>(static_cast<unsigned char*>(a.gathered[q]) + orow, v, ov);
        }
        if (c == 0) {
            if (LN && a.mean) a.mean[i] = mean;
            if (a.rstd) a.rstd[i] = rstd;
        }
    }
}

}  // namespace spk
