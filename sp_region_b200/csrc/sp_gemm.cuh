// Tensor-parallel linears on sm_100a tensor cores (tcgen05), with the
// sequence-parallel collectives fused into them.
//
// "TP and SP explained with pictures", sections "Tensor parallelism, take
// two: split the inner dimension" and "Add Sequence parallelism": a
// row-parallel linear gives every rank a full-shape partial sum of its slice
// of the inner dimension, and with SP those partials are reduce-scattered
// into token shards; a column-parallel linear needs the full input, which SP
// all-gathers from the shards ("Chapter 6: TP and SP", sections 2 and 3).
//
// On one GPU the t ranks' slices of the inner dimension are consecutive
// column blocks of x and of the weight, so the reduce-scatter of the t
// partials IS the K loop of one GEMM: the tensor cores accumulate every
// rank's contribution into the same fp32 accumulator in tensor memory, rank
// by rank, and the partials never exist in HBM.  The epilogue then applies
// the SP region (bias, dropout, residual) to the reduced tile.  For the
// column-parallel linear the all-gather becomes the prologue: the A-operand
// tiles are loaded straight from the t shard buffers.
//
// k_tp_gemm: persistent, one CTA per SM; CTA c takes the 128 x BN output
// tiles c, c + gridDim.x, ... in a grouped order.  The library runs it for
// outputs narrower than 256 features; wider ones run on CTA pairs
// (k_tp_gemm2, sp_gemm2.cuh), 12 % faster on the C2 layer's linears.
//   warps 0 and 6 (one lane each)  TMA producers: warp 0 the A tile, warp 6
//                      the B tile of every stage (K-major, 128-byte swizzle,
//                      64 K-elements per stage) of an S-stage ring that runs on
//                      from one tile into the next.  Warp 0 arms each stage's
//                      full barrier for both copies.  The stage index and
//                      parity of every ring step are kept as counters: a 64-bit
//                      division per step on these threads and on the MMA
//                      thread cost 9-14 % of the throughput
//   warp 1 (one lane)  MMA issuer: tcgen05.mma kind::f16, M = 128, N = BN,
//                      K = 16, bf16 x bf16 -> fp32 in tensor memory, into one
//                      of two accumulator stages (2 x BN columns), so the
//                      epilogue of one tile overlaps the MMAs of the next;
//                      tcgen05.commit frees each ring stage and signals each
//                      finished accumulator
//   warps 2..5         epilogue: tcgen05.ld of the accumulator rows (warp w
//                      reads lanes 32 (w % 4) .. +32, one row per thread),
//                      then frees the accumulator stage
// Every wait is bounded in time; a wait that runs out records an error and
// the CTA drains what it issued, frees its tensor memory and returns.
#pragma once

#include <cuda.h>

#include "sp_device.cuh"
#include "sp_fwd.cuh"

namespace spk {

constexpr int kGemmBM = 128;           // rows per tile (tcgen05 M)
constexpr int kGemmBK = 64;            // K elements per stage: one 128-byte row
constexpr int kGemmThreads = 224;      // A producer, MMA, 4 epilogue warps, B producer
constexpr int kGemmMaxShards = 16;     // A tensor maps (sequence shards)
constexpr int kGemmGroup = 16;         // row tiles per group of the tile order

struct GemmArgs {
    // epilogue kind 0: row-parallel SP (bias, dropout, residual, mask)
    // epilogue kind 1: plain bf16 store
    long long M;              // output rows (tokens)
    int N;                    // output features
    int K;                    // inner dimension
    int stages;
    int rows_per_shard;       // A rows per tensor map (shards: M / nmaps)
    int nmaps;                // A tensor maps (1, or t shards)
    // epilogue
    void* out;                // kind 0: residual_out [M][N]; kind 1: out [M][N]
    const void* bias;         // [N] or NULL (kind 0)
    const void* residual;     // [M][N] (kind 0)
    uint8_t* mask;            // [M][mask_row_bytes] or NULL (kind 0)
    int mask_row_bytes;
    long long row0;           // global token row of output row 0 (Philox counter)
    float scale;              // 1 / (1 - p)
    uint32_t thr;
    uint32_t off_lo, off_hi;
    uint32_t keys[10][2];
    int dropout;
};

// Tensor maps (built on the host with cuTensorMapEncodeTiled): B = the
// weight [N][K]; A = the input rows, either one map of [M][K] or one map per
// sequence shard ([rows_per_shard][K] each).
struct GemmMaps {
    CUtensorMap b;
    CUtensorMap a[kGemmMaxShards];
};

// Shared memory of k_tp_gemm after the 1024-aligned stages: barriers.
struct GemmTail {
    uint64_t full[16];
    uint64_t empty[16];
    uint64_t acc_full[2];    // an accumulator stage is complete
    uint64_t acc_empty[2];   // the epilogue has read an accumulator stage
    uint64_t drain;          // every issued MMA has completed
    uint32_t tmem_base;
    int abort;
};

// ---------------------------------------------------------------------------
// tcgen05 / TMA wrappers (PTX ISA: tcgen05.mma, tcgen05.commit, tcgen05.ld,
// cp.async.bulk.tensor)
// ---------------------------------------------------------------------------

// Shared-memory matrix descriptor of a K-major tile with 128-byte swizzle:
// rows of 128 bytes, 8-row groups 1024 bytes apart (stride byte offset), the
// leading byte offset unused for this layout (1), descriptor version 1,
// swizzle mode 2.  The tile base must be 1024-byte aligned.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr)
{
    uint64_t d = (uint64_t)((saddr & 0x3FFFFu) >> 4);
    d |= (uint64_t)1 << 16;
    d |= (uint64_t)(1024 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

// Instruction descriptor, kind::f16: fp32 accumulator, bf16 A and B, both
// K-major, shape M x N.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on `bar` when every tcgen05.mma this thread issued so far has
// completed (and its shared-memory operands may be overwritten).
__device__ __forceinline__ void umma_commit(uint32_t bar)
{
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
        : "memory");
}

// 2-D tiled bulk tensor load into this CTA's shared memory; x (the inner
// coordinate, in elements) is always a multiple of 64, so x * 2 bytes is a
// multiple of 16 bytes.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            uint32_t bar, uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_last()
{
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// 32 consecutive accumulator columns of this thread's lane (one fp32 each).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t r[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
        "%28, %29, %30, %31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr)
        : "memory");
}

// ---------------------------------------------------------------------------
// The kernel.  BN: output features per tile (a multiple of 32, <= 256).
// EPI 0: row-parallel linear + SP epilogue; EPI 1: plain store.  Persistent:
// grid = min(tiles, SMs); CTA c takes tiles c, c + gridDim.x, ...  Dynamic
// shared memory: 1024 bytes of alignment slack, stages * (16 KB + BN * 128 B),
// then GemmTail.  A tile's rows lie in one A map (rows_per_shard is a
// multiple of 128, or the whole of M).
// ---------------------------------------------------------------------------
__device__ __forceinline__ void gemm_tile_coords(long long tile, int Mt, int Nt, int* tm, int* tn)
{
    // tile order: the CTAs that run at the same time cover a block of
    // kGemmGroup row tiles by a few column tiles, so the A and B slabs they
    // stream (in near lock-step along K) are read from HBM about once and
    // shared through L2
    const long long per_group = (long long)kGemmGroup * Nt;
    const int grp = (int)(tile / per_group);
    const int in_grp = (int)(tile - (long long)grp * per_group);
    const int rows_in_grp = min(kGemmGroup, Mt - grp * kGemmGroup);
    *tm = grp * kGemmGroup + in_grp % rows_in_grp;
    *tn = in_grp / rows_in_grp;
}

// After an abort: wait (bounded) for the last S of the `issued` stages a
// producer filled, so no copy lands in shared memory after the CTA is gone.
// A stage whose barrier was never armed (the other producer stopped first)
// runs out of its wait; by then that copy has long landed.
__device__ __forceinline__ void gemm_drain(GemmTail* tail, long long issued, int S)
{
    const long long first = issued > S ? issued - S : 0;
    for (long long i = first; i < issued; ++i) {
        volatile int no_abort = 0;
        if (!mbar_wait(smem_addr(&tail->full[i % S]), (uint32_t)((i / S) & 1), &no_abort,
                       ERR_DRAIN))
            break;
    }
}

template <int BN, int EPI>
__global__ void __launch_bounds__(kGemmThreads, 1)
    k_tp_gemm(const __grid_constant__ GemmArgs a, const __grid_constant__ GemmMaps maps)
{
    constexpr uint32_t kABytes = kGemmBM * kGemmBK * 2;   // 16 KB
    constexpr uint32_t kBBytes = BN * kGemmBK * 2;
    constexpr uint32_t kStage = kABytes + kBBytes;
    constexpr uint32_t kAccCols = BN <= 128 ? 128 : 256;   // one accumulator stage
    extern __shared__ __align__(1024) unsigned char gsm_raw[];
    // the stages need 1024-byte alignment (128-byte swizzle atoms)
    unsigned char* gsm = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(gsm_raw) + 1023) & ~(uintptr_t)1023);
    const int S = a.stages;
    GemmTail* tail = reinterpret_cast<GemmTail*>(gsm + (size_t)S * kStage);
    volatile int* abort = &tail->abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int Mt = (int)((a.M + kGemmBM - 1) / kGemmBM);
    const int Nt = (a.N + BN - 1) / BN;
    const long long T = (long long)Mt * Nt;
    const int KB = (a.K + kGemmBK - 1) / kGemmBK;
    const CUtensorMap* bmap = &maps.b;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(smem_addr(&tail->full[s]), 1);
            mbar_init(smem_addr(&tail->empty[s]), 1);
        }
        for (int q = 0; q < 2; ++q) {
            mbar_init(smem_addr(&tail->acc_full[q]), 1);
            mbar_init(smem_addr(&tail->acc_empty[q]), 4);   // the 4 epilogue warps
        }
        mbar_init(smem_addr(&tail->drain), 1);
        tail->abort = 0;
        mbar_init_fence();
    }
    if (warp == 1) {
        tmem_alloc(smem_addr(&tail->tmem_base), 2 * kAccCols);
        tmem_fence_before_sync();
    }
    if (warp == 0 && lane <= a.nmaps) {
        // the descriptors into the TMA unit's cache: lane 0 the weight's,
        // lane i the map of shard i - 1
        tma_prefetch_desc(lane == 0 ? bmap : &maps.a[lane - 1]);
    }
    __syncthreads();
    tmem_fence_after_sync();
    const uint32_t tbase = tail->tmem_base;
    grid_dep_launch();
    grid_dep_wait();   // inputs written by the previous kernel are visible

    if (warp == 0) {
        if (lane == 0) {
            // producer: A (x rows) is read by every column tile and B (weight
            // rows) by every row tile: keep both in L2
            const uint64_t pol = policy_evict_last();
            long long g = 0;   // k-steps issued over all tiles
            int s = 0;         // stage of step g: g % S
            uint32_t ph = 0;   // (g / S) & 1; counters, not divisions, on this path
            bool ok = true;
            for (long long tile = blockIdx.x; ok && tile < T; tile += gridDim.x) {
                int tm, tn;
                gemm_tile_coords(tile, Mt, Nt, &tm, &tn);
                const long long m0 = (long long)tm * kGemmBM;
                const int map_id = (int)(m0 / a.rows_per_shard);
                const int a_row = (int)(m0 - (long long)map_id * a.rows_per_shard);
                const CUtensorMap* amap = &maps.a[map_id];
                for (int kb = 0; kb < KB; ++kb, ++g) {
                    // the stage's previous fill (step g - S) has been consumed
                    if (g >= S && !mbar_wait(smem_addr(&tail->empty[s]), ph ^ 1u, abort,
                                             ERR_WAIT_EMPTY)) {
                        ok = false;
                        break;
                    }
                    // armed for both copies; the B producer's may land first
                    const uint32_t bar = smem_addr(&tail->full[s]);
                    mbar_arrive_expect_tx(bar, kStage);
                    tma_load_2d(smem_addr(gsm + (size_t)s * kStage), amap, kb * kGemmBK, a_row,
                                bar, pol);
                    if (++s == S) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            if (*abort) gemm_drain(tail, g, S);
        }
    } else if (warp == 6) {
        if (lane == 0) {
            // B producer: the weight tile of every stage, completing on the
            // full barrier warp 0 arms
            const uint64_t pol = policy_evict_last();
            long long g = 0;
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (long long tile = blockIdx.x; ok && tile < T; tile += gridDim.x) {
                int tm, tn;
                gemm_tile_coords(tile, Mt, Nt, &tm, &tn);
                for (int kb = 0; kb < KB; ++kb, ++g) {
                    if (g >= S && !mbar_wait(smem_addr(&tail->empty[s]), ph ^ 1u, abort,
                                             ERR_WAIT_EMPTY)) {
                        ok = false;
                        break;
                    }
                    tma_load_2d(smem_addr(gsm + (size_t)s * kStage) + kABytes, bmap, kb * kGemmBK,
                                tn * BN, smem_addr(&tail->full[s]), pol);
                    if (++s == S) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            if (*abort) gemm_drain(tail, g, S);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16(kGemmBM, BN);
            int s = 0;         // stage of the next k-step
            uint32_t ph = 0;   // parity of its fill
            bool ok = true;
            long long it = 0;
            for (long long tile = blockIdx.x; ok && tile < T; tile += gridDim.x, ++it) {
                const int as = (int)(it & 1);
                const uint32_t use = (uint32_t)(it >> 1);
                // the epilogue has read this accumulator stage's previous tile
                // (a fresh barrier passes parity 1 at once)
                if (!mbar_wait(smem_addr(&tail->acc_empty[as]), (use & 1u) ^ 1u, abort,
                               ERR_WAIT_EMPTY))
                    break;
                tmem_fence_after_sync();
                const uint32_t tacc = tbase + (uint32_t)as * kAccCols;
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait(smem_addr(&tail->full[s]), ph, abort, ERR_WAIT_FULL)) {
                        ok = false;
                        break;
                    }
                    tmem_fence_after_sync();
                    const uint32_t sa = smem_addr(gsm + (size_t)s * kStage);
                    const uint64_t ad = sw128_desc(sa), bd = sw128_desc(sa + kABytes);
#pragma unroll
                    for (int k = 0; k < kGemmBK / 16; ++k)
                        // +32 bytes of K per step: +2 in the start-address field
                        umma_bf16(tacc, ad + 2 * k, bd + 2 * k, idesc, (kb > 0 || k > 0) ? 1u : 0u);
                    umma_commit(smem_addr(&tail->empty[s]));   // stage s may be refilled
                    if (++s == S) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) break;
                umma_commit(smem_addr(&tail->acc_full[as]));   // the accumulator is complete
            }
            // every issued MMA has finished reading shared memory and writing
            // tensor memory
            umma_commit(smem_addr(&tail->drain));
            volatile int no_abort = 0;
            mbar_wait(smem_addr(&tail->drain), 0u, &no_abort, ERR_DRAIN);
        }
    } else {
        // epilogue warps 2..5: warp w owns accumulator lanes 32 (w % 4) ..
        const int q = warp & 3;
        long long it = 0;
        for (long long tile = blockIdx.x; tile < T; tile += gridDim.x, ++it) {
            int tm, tn;
            gemm_tile_coords(tile, Mt, Nt, &tm, &tn);
            const int as = (int)(it & 1);
            const uint32_t use = (uint32_t)(it >> 1);
            const long long m = (long long)tm * kGemmBM + 32 * q + lane;   // output row of this thread
            const int n0 = tn * BN;
            if (!mbar_wait(smem_addr(&tail->acc_full[as]), use & 1u, abort, ERR_WAIT_FULL)) break;
            tmem_fence_after_sync();
            const bool row_ok = m < a.M;
            const uint32_t trow = tbase + ((uint32_t)(32 * q) << 16) + (uint32_t)as * kAccCols;
#pragma unroll 1
            for (int c0 = 0; c0 < BN; c0 += 32) {
                if (n0 + c0 >= a.N) break;          // warp-uniform
                uint32_t r[32];
                tmem_ld32(trow + (uint32_t)c0, r);   // warp-wide, outside per-thread branches
                if (!row_ok) continue;
#pragma unroll
                for (int v8 = 0; v8 < 4; ++v8) {
                    const int col = n0 + c0 + 8 * v8;   // first feature of this 8-vector
                    if (col >= a.N) continue;           // N % 8 == 0: vectors are whole
                    F2 y[4];
#pragma unroll
                    for (int p = 0; p < 4; ++p)
                        y[p] = f2(__uint_as_float(r[8 * v8 + 2 * p]),
                                  __uint_as_float(r[8 * v8 + 2 * p + 1]));
                    if (EPI == 0) {
                        const long long n = a.row0 + m;   // global token row
                        if (a.bias) {
                            F2 b[4];
                            IO<__nv_bfloat16>::unpack2(load_vec<__nv_bfloat16>(a.bias, col / 8), b);
#pragma unroll
                            for (int p = 0; p < 4; ++p) y[p] = add2(y[p], b[p]);
                        }
                        uint32_t kb8 = 0xFFu;
                        if (a.dropout) {
                            kb8 = keep_bits8((uint32_t)(col / 8), (uint32_t)n, a.off_lo, a.off_hi,
                                             a.keys, a.thr);
                            const F2 sc2 = f2(a.scale);
#pragma unroll
                            for (int p = 0; p < 4; ++p)
                                y[p] = keep2(mul2(y[p], sc2), (kb8 >> (2 * p)) & 1u,
                                             (kb8 >> (2 * p + 1)) & 1u);
                        }
                        if (a.mask) a.mask[(size_t)m * a.mask_row_bytes + col / 8] = (uint8_t)kb8;
                        F2 rs[4];
                        const unsigned char* rrow =
                            static_cast<const unsigned char*>(a.residual) + (size_t)m * a.N * 2;
                        IO<__nv_bfloat16>::unpack2(load_vec<__nv_bfloat16>(rrow, col / 8), rs);
#pragma unroll
                        for (int p = 0; p < 4; ++p) y[p] = add2(rs[p], y[p]);
                    }
                    unsigned char* orow = static_cast<unsigned char*>(a.out) + (size_t)m * a.N * 2;
                    store_vec<__nv_bfloat16>(orow, col / 8, IO<__nv_bfloat16>::pack2v(y));
                }
                if (EPI == 0 && a.mask && n0 + c0 + 32 >= a.N) {
                    // the row's last features: zero the mask's padding bytes
                    for (int pb = a.N / 8; pb < a.mask_row_bytes; ++pb)
                        a.mask[(size_t)m * a.mask_row_bytes + pb] = 0;
                }
            }
            // this warp's reads of the stage are done: the MMA may refill it
            tmem_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_addr(&tail->acc_empty[as]));
        }
    }
    // every tensor-memory access is done before warp 1 frees the columns
    tmem_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tmem_fence_after_sync();
        tmem_dealloc(tbase, 2 * kAccCols);
    }
}

}  // namespace spk
