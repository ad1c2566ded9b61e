// Device helpers shared by the sm_100a kernels of the SP boundary:
// mbarrier / bulk-copy wrappers with time-bounded waits, Philox4x32-10,
// I/O-dtype packing, and fp32 reductions in a fixed order.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace spk {

// ---------------------------------------------------------------------------
// Device-side error word.  A bounded wait that runs out records its code here
// (first error wins) and the kernel winds down instead of hanging; the host
// reads it with sp_device_error().  Each translation unit of the library is
// its own device module with its own word (static); SPK_ERROR_WORD_ACCESSOR
// defines the host function that reads and clears the word of the unit it
// is expanded in.
// ---------------------------------------------------------------------------
static __device__ unsigned int g_error;

#define SPK_ERROR_WORD_ACCESSOR(NAME)                                                \
    int NAME(unsigned* v, int clear)                                                 \
    {                                                                                \
        if (cudaMemcpyFromSymbol(v, g_error, sizeof(unsigned)) != cudaSuccess)       \
            return -1;                                                               \
        if (clear) {                                                                 \
            const unsigned zero = 0;                                                 \
            if (cudaMemcpyToSymbol(g_error, &zero, sizeof(zero)) != cudaSuccess)     \
                return -1;                                                           \
        }                                                                            \
        return 0;                                                                    \
    }

enum : unsigned {
    ERR_WAIT_FULL = 1,      // a consumer waited too long for a staged row
    ERR_WAIT_EMPTY = 2,     // the producer waited too long for a free stage
    ERR_DRAIN = 3,          // an aborted CTA could not drain its copies
    ERR_WAIT_PEER = 4,      // a CTA waited too long for its cluster peer's sums
    ERR_SELFTEST = 9,       // the diagnostic wait of sp_debug_wait_timeout
};

// Long enough that no legitimate wait on a B200 comes near it (a whole row
// stream of the largest workload takes microseconds), short enough that a
// lost copy surfaces as an error well inside any process timeout.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ unsigned long long globaltimer_ns()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void record_error(unsigned code)
{
    atomicCAS(&g_error, 0u, code);
}

// ---------------------------------------------------------------------------
// Programmatic dependent launch (PTX ISA: griddepcontrol).  The library
// launches every kernel so that the next kernel in the stream may be
// scheduled before this one has finished; its CTAs then wait in
// grid_dep_wait() until the kernels it depends on have completed and their
// memory is visible.  Every kernel calls grid_dep_wait() before its first
// global-memory access (read or write), so the early launch hides only the
// launch and set-up latency, never a data dependence.  grid_dep_launch()
// lets this kernel's own dependents be scheduled.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void grid_dep_wait()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ void grid_dep_launch()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------------------
// mbarrier and bulk copy (PTX ISA: mbarrier.*, cp.async.bulk)
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_addr(const void* p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void mbar_init_fence()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// A thread whose phase has not completed is suspended in hardware until the
// phase completes or about kSuspendHintNs pass, so waiting warps do not spin
// on the issue slots the working warps need.
constexpr uint32_t kSuspendHintNs = 20000;

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(kSuspendHintNs)
        : "memory");
    return ok != 0;
}

// Wait for the phase of `bar` with the given parity to complete.  Returns
// false, without waiting further, once *abort is set or the time limit runs
// out (which sets *abort and records `code`).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity,
                                          volatile int* abort, unsigned code,
                                          unsigned long long limit_ns = kWaitLimitNs)
{
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    for (;;) {
#pragma unroll 1
        for (int i = 0; i < 16; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (*abort) return false;
        if (globaltimer_ns() - t0 > limit_ns) {
            *abort = 1;
            record_error(code);
            return false;
        }
    }
}

// ---------------------------------------------------------------------------
// Thread-block clusters: a token row split across the CTAs of a cluster
// exchanges its per-row partial sums through distributed shared memory.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ uint32_t cluster_index()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
    return r;
}

__device__ __forceinline__ uint32_t cluster_count()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
    return r;
}

// Every thread of every CTA of the cluster (release / acquire at cluster
// scope): orders the barrier initialisation before any remote access, and
// keeps a CTA from exiting while a peer may still touch its shared memory.
__device__ __forceinline__ void cluster_sync_all()
{
    asm volatile(
        "barrier.cluster.arrive.release.aligned;\n\t"
        "barrier.cluster.wait.acquire.aligned;" ::
            : "memory");
}

// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t peer_addr(uint32_t local, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
    return r;
}

__device__ __forceinline__ void st_peer_f32x2(uint32_t addr, float x, float y)
{
    asm volatile("st.shared::cluster.v2.f32 [%0], {%1, %2};" ::"r"(addr), "f"(x), "f"(y)
                 : "memory");
}

// Arrive on an mbarrier in a peer CTA, releasing this thread's prior writes
// (the value just stored there) at cluster scope.
__device__ __forceinline__ void mbar_arrive_peer(uint32_t peer_bar)
{
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(peer_bar)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(kSuspendHintNs)
        : "memory");
    return ok != 0;
}

// Bounded wait with cluster-scope acquire (for values a peer CTA released).
__device__ __forceinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t parity,
                                                  volatile int* abort, unsigned code)
{
    if (mbar_try_wait_cluster(bar, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    for (;;) {
#pragma unroll 1
        for (int i = 0; i < 16; ++i)
            if (mbar_try_wait_cluster(bar, parity)) return true;
        if (*abort) return false;
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            *abort = 1;
            record_error(code);
            return false;
        }
    }
}

// One bulk copy global -> this CTA's shared memory, completing `bytes`
// transaction bytes on `bar`.  dst and src 16-byte aligned, bytes % 16 == 0.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar, uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1], %2, [%3], %4;" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar), "l"(policy)
        : "memory");
}

// L2 policy for data read exactly once.
__device__ __forceinline__ uint64_t policy_evict_first()
{
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// ---------------------------------------------------------------------------
// Tensor memory (PTX ISA: tcgen05.alloc / ld / st / wait / dealloc).  Each SM
// has 128 lanes x 512 columns of 32-bit cells; an address is
// (lane << 16) | column.  Warp w of a CTA may touch only lanes
// [32 * (w % 4), 32 * (w % 4) + 32), one lane per thread.  The kernels here
// use it as per-thread scratch that does not take shared memory or registers.
// ---------------------------------------------------------------------------
// one whole warp: allocate ncols columns (a power of 2 in [32, 512]) and
// write the base address to shared memory; waits while the SM's tensor
// memory is held by other CTAs
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(dst_smem), "r"(ncols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

// the warp that allocated, once no thread touches the columns any more
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

// order tensor-memory operations across a thread barrier
__device__ __forceinline__ void tmem_fence_before_sync()
{
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tmem_fence_after_sync()
{
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// this thread's earlier stores have landed (before the cells are read again)
__device__ __forceinline__ void tmem_wait_st()
{
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// 8 / 16 consecutive columns of this thread's lane.  The load and its wait
// are one statement, so no use of the registers can be scheduled before the
// data has arrived.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t r[8])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t r[16])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, "
        "%10, %11, %12, %13, %14, %15}, [%16];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t r[8])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]),
          "r"(r[6]), "r"(r[7])
        : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t r[16])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, "
        "%10, %11, %12, %13, %14, %15, %16};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]),
          "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]),
          "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

// ---------------------------------------------------------------------------
// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As
// Easy as 1, 2, 3", SC'11).  Each round multiplies counter words 0 and 2 by
// the two Philox constants; the new words are (hi1 ^ w1 ^ k0, lo1,
// hi0 ^ w3 ^ k1, lo0), and the key advances by the two Weyl constants.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint4 philox4x32_10(uint4 w, uint32_t k0, uint32_t k1)
{
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        // one widening multiply gives both halves of each 64-bit product
        const unsigned long long p0 = (unsigned long long)w.x * 0xD2511F53u;
        const unsigned long long p1 = (unsigned long long)w.z * 0xCD9E8D57u;
        w = make_uint4((uint32_t)(p1 >> 32) ^ w.y ^ k0, (uint32_t)p1,
                       (uint32_t)(p0 >> 32) ^ w.w ^ k1, (uint32_t)p0);
        k0 += 0x9E3779B9u;
        k1 += 0xBB67AE85u;
    }
    return w;
}

// The same rounds with the key schedule precomputed: ks[r] = (k0, k1) of
// round r, identical for every thread of a launch, so the rounds read it from
// the kernel's parameters instead of advancing it per call.
__device__ __forceinline__ uint4 philox4x32_10(uint4 w, const uint32_t (&ks)[10][2])
{
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        const unsigned long long p0 = (unsigned long long)w.x * 0xD2511F53u;
        const unsigned long long p1 = (unsigned long long)w.z * 0xCD9E8D57u;
        w = make_uint4((uint32_t)(p1 >> 32) ^ w.y ^ ks[r][0], (uint32_t)p1,
                       (uint32_t)(p0 >> 32) ^ w.w ^ ks[r][1], (uint32_t)p0);
    }
    return w;
}

// Keep bits of the 8 features [8v, 8v+8) of token row n (scheduled keys).
__device__ __forceinline__ uint32_t keep_bits8(uint32_t v, uint32_t n, uint32_t off_lo,
                                               uint32_t off_hi, const uint32_t (&ks)[10][2],
                                               uint32_t thr)
{
    const uint4 a = philox4x32_10(make_uint4(2u * v, n, off_lo, off_hi), ks);
    const uint4 b = philox4x32_10(make_uint4(2u * v + 1u, n, off_lo, off_hi), ks);
    return (uint32_t)(a.x >= thr) | (uint32_t)(a.y >= thr) << 1 |
           (uint32_t)(a.z >= thr) << 2 | (uint32_t)(a.w >= thr) << 3 |
           (uint32_t)(b.x >= thr) << 4 | (uint32_t)(b.y >= thr) << 5 |
           (uint32_t)(b.z >= thr) << 6 | (uint32_t)(b.w >= thr) << 7;
}

// Keep bits of the 8 features [8v, 8v+8) of token row n: counter
// (q, n, offset lo, offset hi) for q = 2v and 2v+1, word j & 3 of each;
// kept iff the word is >= thr.  Bit e of the result is feature 8v+e.
__device__ __forceinline__ uint32_t keep_bits8(uint32_t v, uint32_t n, uint32_t off_lo,
                                               uint32_t off_hi, uint32_t k0, uint32_t k1,
                                               uint32_t thr)
{
    const uint4 a = philox4x32_10(make_uint4(2u * v, n, off_lo, off_hi), k0, k1);
    const uint4 b = philox4x32_10(make_uint4(2u * v + 1u, n, off_lo, off_hi), k0, k1);
    return (uint32_t)(a.x >= thr) | (uint32_t)(a.y >= thr) << 1 |
           (uint32_t)(a.z >= thr) << 2 | (uint32_t)(a.w >= thr) << 3 |
           (uint32_t)(b.x >= thr) << 4 | (uint32_t)(b.y >= thr) << 5 |
           (uint32_t)(b.z >= thr) << 6 | (uint32_t)(b.w >= thr) << 7;
}

// Keep bit of one feature j of row n (general kernels).
__device__ __forceinline__ uint32_t keep_bit(uint32_t j, uint32_t n, uint32_t off_lo,
                                             uint32_t off_hi, uint32_t k0, uint32_t k1,
                                             uint32_t thr)
{
    const uint4 a = philox4x32_10(make_uint4(j >> 2, n, off_lo, off_hi), k0, k1);
    const uint32_t w = (j & 3) == 0 ? a.x : (j & 3) == 1 ? a.y : (j & 3) == 2 ? a.z : a.w;
    return w >= thr ? 1u : 0u;
}

// ---------------------------------------------------------------------------
// Two fp32 values in one 64-bit register.  sm_100a adds, subtracts,
// multiplies and fuses a multiply-add on both halves in one instruction (PTX
// add / sub / mul / fma .rn.f32x2); each half is rounded exactly as the scalar
// operation would round it, so pairing changes the instruction count, not
// the arithmetic.  .x is the lower feature of the pair.
// ---------------------------------------------------------------------------
struct F2 {
    unsigned long long r;
};

__device__ __forceinline__ F2 f2(float lo, float hi)
{
    F2 v;
    asm("mov.b64 %0, {%1, %2};" : "=l"(v.r) : "f"(lo), "f"(hi));
    return v;
}

__device__ __forceinline__ F2 f2(float x) { return f2(x, x); }

__device__ __forceinline__ float2 halves(F2 v)
{
    float2 o;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(o.x), "=f"(o.y) : "l"(v.r));
    return o;
}

__device__ __forceinline__ F2 add2(F2 a, F2 b)
{
    F2 d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d.r) : "l"(a.r), "l"(b.r));
    return d;
}

__device__ __forceinline__ F2 sub2(F2 a, F2 b)
{
    F2 d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d.r) : "l"(a.r), "l"(b.r));
    return d;
}

__device__ __forceinline__ F2 mul2(F2 a, F2 b)
{
    F2 d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d.r) : "l"(a.r), "l"(b.r));
    return d;
}

// a * b + c with one rounding per half
__device__ __forceinline__ F2 fma2(F2 a, F2 b, F2 c)
{
    F2 d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d.r) : "l"(a.r), "l"(b.r), "l"(c.r));
    return d;
}

// halves kept where bits b0 / b1 are set, else +0
__device__ __forceinline__ F2 keep2(F2 v, uint32_t b0, uint32_t b1)
{
    const float2 x = halves(v);
    return f2(b0 ? x.x : 0.f, b1 ? x.y : 0.f);
}

// sum of the two halves
__device__ __forceinline__ float hsum(F2 v)
{
    const float2 x = halves(v);
    return x.x + x.y;
}

// ---------------------------------------------------------------------------
// I/O dtype: 8 consecutive elements are one "vector" (16 B of bf16, 32 B of
// fp32).  Arithmetic is always fp32; stores round to nearest-even.  unpack2 /
// pack2v move a vector to and from four fp32 pairs.
// ---------------------------------------------------------------------------
template <typename T>
struct IO;

template <>
struct IO<__nv_bfloat16> {
    static constexpr int kBytes = 2;
    static constexpr int kWords = 1;   // uint4 per vector
    struct Vec {
        uint4 u[1];
    };

    __device__ static __forceinline__ void unpack(const Vec& v, float f[8])
    {
        const uint32_t w[4] = {v.u[0].x, v.u[0].y, v.u[0].z, v.u[0].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    }
    __device__ static __forceinline__ uint32_t pack2(float a, float b)
    {
        __nv_bfloat162 h = __floats2bfloat162_rn(a, b);   // .x (low half) = a
        return *reinterpret_cast<uint32_t*>(&h);
    }
    __device__ static __forceinline__ void unpack2(const Vec& v, F2 f[4])
    {
        const uint32_t w[4] = {v.u[0].x, v.u[0].y, v.u[0].z, v.u[0].w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
            f[i] = f2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u));
    }
    __device__ static __forceinline__ Vec pack2v(const F2 f[4])
    {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 x = halves(f[i]);
            w[i] = pack2(x.x, x.y);
        }
        Vec v;
        v.u[0] = make_uint4(w[0], w[1], w[2], w[3]);
        return v;
    }
    __device__ static __forceinline__ Vec pack(const float f[8])
    {
        Vec v;
        v.u[0] = make_uint4(pack2(f[0], f[1]), pack2(f[2], f[3]), pack2(f[4], f[5]),
                            pack2(f[6], f[7]));
        return v;
    }
    __device__ static __forceinline__ float load1(const void* p, long long i)
    {
        const uint16_t b = static_cast<const uint16_t*>(p)[i];
        return __uint_as_float(static_cast<uint32_t>(b) << 16);
    }
    __device__ static __forceinline__ void store1(void* p, long long i, float x)
    {
        static_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(x);
    }
    __device__ static __forceinline__ float round1(float x)
    {
        return __bfloat162float(__float2bfloat16_rn(x));
    }
};

template <>
struct IO<float> {
    static constexpr int kBytes = 4;
    static constexpr int kWords = 2;
    struct Vec {
        uint4 u[2];
    };

    __device__ static __forceinline__ void unpack(const Vec& v, float f[8])
    {
        f[0] = __uint_as_float(v.u[0].x);
        f[1] = __uint_as_float(v.u[0].y);
        f[2] = __uint_as_float(v.u[0].z);
        f[3] = __uint_as_float(v.u[0].w);
        f[4] = __uint_as_float(v.u[1].x);
        f[5] = __uint_as_float(v.u[1].y);
        f[6] = __uint_as_float(v.u[1].z);
        f[7] = __uint_as_float(v.u[1].w);
    }
    __device__ static __forceinline__ void unpack2(const Vec& v, F2 f[4])
    {
        f[0] = f2(__uint_as_float(v.u[0].x), __uint_as_float(v.u[0].y));
        f[1] = f2(__uint_as_float(v.u[0].z), __uint_as_float(v.u[0].w));
        f[2] = f2(__uint_as_float(v.u[1].x), __uint_as_float(v.u[1].y));
        f[3] = f2(__uint_as_float(v.u[1].z), __uint_as_float(v.u[1].w));
    }
    __device__ static __forceinline__ Vec pack2v(const F2 f[4])
    {
        float2 x[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) x[i] = halves(f[i]);
        Vec v;
        v.u[0] = make_uint4(__float_as_uint(x[0].x), __float_as_uint(x[0].y),
                            __float_as_uint(x[1].x), __float_as_uint(x[1].y));
        v.u[1] = make_uint4(__float_as_uint(x[2].x), __float_as_uint(x[2].y),
                            __float_as_uint(x[3].x), __float_as_uint(x[3].y));
        return v;
    }
    __device__ static __forceinline__ Vec pack(const float f[8])
    {
        Vec v;
        v.u[0] = make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]),
                            __float_as_uint(f[2]), __float_as_uint(f[3]));
        v.u[1] = make_uint4(__float_as_uint(f[4]), __float_as_uint(f[5]),
                            __float_as_uint(f[6]), __float_as_uint(f[7]));
        return v;
    }
    __device__ static __forceinline__ float load1(const void* p, long long i)
    {
        return static_cast<const float*>(p)[i];
    }
    __device__ static __forceinline__ void store1(void* p, long long i, float x)
    {
        static_cast<float*>(p)[i] = x;
    }
    __device__ static __forceinline__ float round1(float x) { return x; }
};

template <typename T>
__device__ __forceinline__ typename IO<T>::Vec load_vec(const void* base, long long v)
{
    typename IO<T>::Vec r;
    const uint4* p = static_cast<const uint4*>(base) + v * IO<T>::kWords;
#pragma unroll
    for (int i = 0; i < IO<T>::kWords; ++i) r.u[i] = p[i];
    return r;
}

template <typename T>
__device__ __forceinline__ void store_vec(void* base, long long v, const typename IO<T>::Vec& x)
{
    uint4* p = static_cast<uint4*>(base) + v * IO<T>::kWords;
#pragma unroll
    for (int i = 0; i < IO<T>::kWords; ++i) p[i] = x.u[i];
}

// ---------------------------------------------------------------------------
// fp32 sums, deterministic: butterfly within the warp, then every consumer
// thread adds the per-warp totals in warp order.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float warp_sum(float x)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xFFFFFFFFu, x, o);
    return x;
}

// Second level of a group reduction: lane l adds the total of warp l (warps
// have stored theirs in red[0 .. nwarps)); every lane of every warp ends with
// the same bits (an xor butterfly combines the same two partials on both
// sides of each exchange).
__device__ __forceinline__ float warps_total(const float* red, int nwarps)
{
    const int lane = threadIdx.x & 31;
    return warp_sum(lane < nwarps ? red[lane] : 0.f);
}

__device__ __forceinline__ float2 warps_total2(const float2* red, int nwarps)
{
    const int lane = threadIdx.x & 31;
    const float2 v = lane < nwarps ? red[lane] : make_float2(0.f, 0.f);
    return make_float2(warp_sum(v.x), warp_sum(v.y));
}

// Block-wide sum for the general kernels (all threads take part).
__device__ __forceinline__ float block_sum(float x, float* red)
{
    x = warp_sum(x);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    __syncthreads();   // red may still be read by a previous call
    if (lane == 0) red[warp] = x;
    __syncthreads();
    float s = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) s += red[w];
    return s;
}

}  // namespace spk
