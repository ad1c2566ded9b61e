// All-gather along the sequence: t token shards -> n_out full [s,b,h]
// tensors ("SP: Partition Activations Alongside TP", section "Change layouts
// between SP and TP": the shards of the SP region combine into the same
// input X on every GPU).  On one GPU this is a copy of each shard into its
// row range of every output: each shard is read once and written n_out
// times, by bulk copies through shared memory when every buffer is 16-byte
// aligned (k_all_gather_bulk), else element by element (k_all_gather).
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

// The aligned all-gather by bulk copies: each CTA's issuing thread loads a
// chunk of a shard into shared memory once and stores it to every output with
// one bulk copy each, so a vector crosses the SM once and the output writes
// leave as whole-chunk requests.  kAgSlots chunks are in flight: a slot is
// refilled once the stores of its previous chunk have read it.  shard_units
// counts 16-byte vectors; every address and size is a multiple of 16 bytes.
constexpr int kAgChunk = 32768;   // bytes per chunk
constexpr int kAgSlots = 6;

__device__ __forceinline__ void bulk_store(void* dst, uint32_t src, uint32_t bytes)
{
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
                 "r"(src), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit()
{
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// every committed group but the newest has finished reading shared memory
__device__ __forceinline__ void bulk_wait_read_all_but_one()
{
    asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}

// every committed group has completed (its writes are done)
__device__ __forceinline__ void bulk_wait_all()
{
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

__global__ void __launch_bounds__(32) k_all_gather_bulk(const __grid_constant__ GatherArgs a)
{
    extern __shared__ __align__(128) unsigned char agsm[];
    __shared__ __align__(8) uint64_t full[kAgSlots];
    __shared__ int abort_flag;
    grid_dep_launch();
    if (threadIdx.x != 0) return;   // one issuing thread per CTA
    for (int i = 0; i < kAgSlots; ++i) mbar_init(smem_addr(&full[i]), 1);
    abort_flag = 0;
    mbar_init_fence();
    grid_dep_wait();   // the shards written by the previous kernel are visible
    const long long shard_bytes = a.shard_units * 16;
    const long long cps = (shard_bytes + kAgChunk - 1) / kAgChunk;   // chunks per shard
    const long long total = cps * a.t;
    if ((long long)blockIdx.x >= total) return;
    const long long n_mine = (total - 1 - blockIdx.x) / gridDim.x + 1;
    const uint64_t pol = policy_evict_first();
    // chunk k of this CTA: its source, its offset in every output, its size
    auto chunk = [&](long long k, const unsigned char** src, long long* off, uint32_t* bytes) {
        const long long c = blockIdx.x + k * gridDim.x;
        const int r = (int)(c / cps);
        const long long o = (c - (long long)r * cps) * kAgChunk;
        const long long left = shard_bytes - o;
        *bytes = (uint32_t)(left < kAgChunk ? left : kAgChunk);
        *src = static_cast<const unsigned char*>(a.shards[r]) + o;
        *off = (long long)r * shard_bytes + o;
    };
    auto load = [&](long long k) {
        const int slot = (int)(k % kAgSlots);
        const unsigned char* src;
        long long off;
        uint32_t bytes;
        chunk(k, &src, &off, &bytes);
        const uint32_t bar = smem_addr(&full[slot]);
        mbar_arrive_expect_tx(bar, bytes);
        bulk_load(smem_addr(agsm + (size_t)slot * kAgChunk), src, bytes, bar, pol);
    };
    long long loaded = n_mine < kAgSlots ? n_mine : kAgSlots;
    for (long long k = 0; k < loaded; ++k) load(k);
    long long k = 0;
    for (; k < n_mine; ++k) {
        const int slot = (int)(k % kAgSlots);
        if (!mbar_wait(smem_addr(&full[slot]), (uint32_t)((k / kAgSlots) & 1), &abort_flag,
                       ERR_WAIT_FULL))
            break;
        const unsigned char* src;
        long long off;
        uint32_t bytes;
        chunk(k, &src, &off, &bytes);
        const uint32_t sa = smem_addr(agsm + (size_t)slot * kAgChunk);
        for (int q = 0; q < a.n_out; ++q)
            bulk_store(static_cast<unsigned char*>(a.outs[q]) + off, sa, bytes);
        bulk_commit();
        // the previous chunk's stores have read their slot: refill it
        if (k >= 1 && loaded < n_mine) {
            bulk_wait_read_all_but_one();
            load(loaded);
            ++loaded;
        }
    }
    if (k < n_mine) {
        // a wait ran out: the loads already issued land before the CTA's
        // shared memory goes away
        volatile int no_abort = 0;
        for (long long j = k; j < loaded; ++j)
            if (!mbar_wait(smem_addr(&full[j % kAgSlots]), (uint32_t)((j / kAgSlots) & 1),
                           &no_abort, ERR_DRAIN))
                break;
    }
    bulk_wait_all();   // every store has completed before the CTA exits
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
