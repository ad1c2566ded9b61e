// All-gather along the sequence: t token shards -> n_out full [s,b,h]
// tensors ("SP: Partition Activations Alongside TP", section "Change layouts
// between SP and TP": the shards of the SP region combine into the same
// input X on every GPU).  On one GPU this is a copy of each shard into its
// row range of every output; each 16-byte vector is read once and written
// n_out times.
#pragma once

#include "sp_device.cuh"
#include "sp_fwd.cuh"

namespace spk {

struct GatherArgs {
    const void* shards[kMaxT];
    void* outs[kMaxT];
    long long shard_units;   // units per shard (16-byte vectors or elements)
    int t;
    int n_out;
    int unit_bytes;          // 16 (vector path), 4 or 2 (element path)
};

template <typename U>
__global__ void __launch_bounds__(512) k_all_gather(const __grid_constant__ GatherArgs a)
{
    grid_dep_launch();
    grid_dep_wait();
    const long long total = a.shard_units * a.t;
    const long long stride = (long long)gridDim.x * blockDim.x;
    constexpr int kUnroll = 4;
    long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    for (; i + (kUnroll - 1) * stride < total; i += kUnroll * stride) {
        U v[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const long long g = i + u * stride;
            const int r = (int)(g / a.shard_units);
            v[u] = static_cast<const U*>(a.shards[r])[g - (long long)r * a.shard_units];
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u)
            for (int q = 0; q < a.n_out; ++q) static_cast<U*>(a.outs[q])[i + u * stride] = v[u];
    }
    for (; i < total; i += stride) {
        const int r = (int)(i / a.shard_units);
        const U v = static_cast<const U*>(a.shards[r])[i - (long long)r * a.shard_units];
        for (int q = 0; q < a.n_out; ++q) static_cast<U*>(a.outs[q])[i] = v;
    }
}

// Diagnostic: one CTA waits on an mbarrier that nothing completes, with the
// given time limit, and reports whether the wait ran out (status 1) instead
// of hanging.  Exercises the same bounded wait as the streaming kernels.
__global__ void k_wait_selftest(unsigned long long limit_ns, int* status)
{
    grid_dep_launch();
    grid_dep_wait();
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort;
    if (threadIdx.x == 0) {
        mbar_init(smem_addr(&bar), 1);
        abort = 0;
        mbar_init_fence();
    }
    __syncthreads();
    const bool ok = mbar_wait(smem_addr(&bar), 0, &abort, ERR_SELFTEST, limit_ns);
    __syncthreads();
    if (threadIdx.x == 0) *status = ok ? 0 : 1;
}

}  // namespace spk
