// Tensor-parallel linears on CTA pairs: the row-parallel linear with the
// sequence-parallel epilogue and the column-parallel linear with the
// all-gather prologue ("TP and SP explained with pictures", sections
// "Tensor parallelism, take two: split the inner dimension" and "Add Sequence
// parallelism"; "Chapter 6: TP and SP", sections 2 and 3), for outputs at
// least 256 features wide.  The single-CTA kernel k_tp_gemm covers narrower
// ones; both compute the same tile sums in the same order.
//
// k_tp_gemm2: persistent, one CTA pair (a 2-CTA cluster on one TPC) per
// 256 x 256 output tile at a time; cluster c takes tiles c, c + clusters, ...
// Each CTA stages its own 128 rows of A and its own 128 features of B (so a
// pair streams 64 KB per 64-deep K step for 8.4 MFLOP, a third less than two
// independent 128 x 256 tiles), and the leader CTA (rank 0) issues
// tcgen05.mma.cta_group::2, M = 256, N = 256, K = 16, which reads both CTAs'
// shared memory and leaves rows 0..127 of the fp32 accumulator in the
// leader's tensor memory and rows 128..255 in the peer's.  Two accumulator
// stages (2 x 256 of the 512 columns) let the epilogue of one tile overlap
// the MMAs of the next.
//   warp 0 (one lane, both CTAs)  TMA producer: A and B halves (K-major,
//                      128-byte swizzle) into an S-stage ring; every copy
//                      completes on the leader's "full" barrier, which the
//                      leader arms for both CTAs' bytes
//   warp 1 (one lane, leader)     MMA issuer; tcgen05.commit frees each stage
//                      in both CTAs and signals each accumulator stage to both
//   warps 2..5 (both CTAs)        epilogue: tcgen05.ld of this CTA's 128 rows
//                      (warp w reads lanes 32 (w % 4) .. +32, one row per
//                      thread), then an arrive on the leader's "accumulator
//                      empty" barrier
// The stage index and parity of every ring step are counters on the threads
// that walk the ring (no division per step).  Every wait is bounded in time;
// a wait that runs out records an error and the CTA drains what it issued
// before the pair frees its tensor memory.  Each CTA's copies write only its
// own shared memory.
#pragma once

#include "sp_gemm.cuh"

namespace spk {

constexpr int kGemm2BN = 256;           // output features per pair tile
constexpr int kGemm2HalfN = 128;        // B rows (features) each CTA stages
constexpr int kGemm2Threads = 192;      // producer, MMA, 4 epilogue warps
constexpr int kGemm2Group = 8;          // pair-row tiles per group of the tile order
constexpr int kGemm2MaxStages = 8;
constexpr uint32_t kGemm2TmemCols = 512;   // two accumulator stages of 256 columns

struct GemmTail2 {
    uint64_t full[kGemm2MaxStages];    // leader: both CTAs' halves of a stage landed
    uint64_t empty[kGemm2MaxStages];   // each CTA: the MMAs are done with its stage
    uint64_t acc_full[2];              // each CTA: an accumulator stage is complete
    uint64_t acc_empty[2];             // leader: both CTAs' epilogues have read it
    uint64_t drain;                    // leader: every issued MMA has completed
    long long issued;                  // k-steps this CTA's producer issued
    uint32_t tmem_base;
    int abort;
};

// The CTA-pair forms: one MMA over both CTAs' shared memory (issued by the
// leader), and the commit that tracks such MMAs; `bar` may be an mbarrier of
// either CTA (a shared::cluster address).
__device__ __forceinline__ void umma_bf16_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                               uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void umma_commit_pair(uint32_t bar)
{
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
        : "memory");
}

// Tensor memory shared by the CTA pair: both CTAs' warp 1 allocate (and
// later free) the same columns together.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(dst_smem), "r"(ncols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

// The same load issued by either CTA of a pair, completing its bytes on an
// mbarrier of either CTA (`bar`: a shared::cluster address; here always the
// leader's).  Each CTA writes only its own shared memory.
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, int x,
                                                 int y, uint32_t bar, uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx"
        "::bytes.L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void gemm2_tile_coords(long long tile, int Mt, int Nt, int* tm, int* tn)
{
    // tile order: the pairs that run at the same time cover a block of
    // kGemm2Group pair-row tiles by a few column tiles, so the A and B slabs
    // they stream (in near lock-step along K) are read from HBM about once
    // and shared through L2
    const long long per_group = (long long)kGemm2Group * Nt;
    const int grp = (int)(tile / per_group);
    const int in_grp = (int)(tile - (long long)grp * per_group);
    const int rows_in_grp = min(kGemm2Group, Mt - grp * kGemm2Group);
    *tm = grp * kGemm2Group + in_grp % rows_in_grp;
    *tn = in_grp / rows_in_grp;
}

template <int EPI>
__global__ void __launch_bounds__(kGemm2Threads, 1)
    k_tp_gemm2(const __grid_constant__ GemmArgs a, const __grid_constant__ GemmMaps maps)
{
    constexpr uint32_t kABytes = kGemmBM * kGemmBK * 2;      // 16 KB
    constexpr uint32_t kBBytes = kGemm2HalfN * kGemmBK * 2;   // 16 KB
    constexpr uint32_t kStage = kABytes + kBBytes;
    extern __shared__ __align__(1024) unsigned char gsm_raw[];
    // the stages need 1024-byte alignment (128-byte swizzle atoms); the
    // offset is the same in both CTAs, as the pair MMA requires
    unsigned char* gsm = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(gsm_raw) + 1023) & ~(uintptr_t)1023);
    const int S = a.stages;
    GemmTail2* tail = reinterpret_cast<GemmTail2*>(gsm + (size_t)S * kStage);
    volatile int* abort = &tail->abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();            // 0: the leader
    const long long cl = (long long)cluster_index(), ncl = (long long)cluster_count();
    const int Mt = (int)((a.M + 2 * kGemmBM - 1) / (2 * kGemmBM));
    const int Nt = (a.N + kGemm2BN - 1) / kGemm2BN;
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
            mbar_init(smem_addr(&tail->acc_empty[q]), 2 * 4);   // 4 epilogue warps per CTA
        }
        mbar_init(smem_addr(&tail->drain), 1);
        tail->abort = 0;
        mbar_init_fence();
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_addr(&tail->tmem_base), kGemm2TmemCols);
        tmem_fence_before_sync();
    }
    if (threadIdx.x == 0) tma_prefetch_desc(bmap);
    // barriers initialised in both CTAs before any remote arrive or copy
    cluster_sync_all();
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
            int s = 0;         // the stage of step g
            uint32_t ph = 0;   // the parity of its use
            bool ok = true;
            tail->issued = 0;
            for (long long tile = cl; ok && tile < T; tile += ncl) {
                int tm, tn;
                gemm2_tile_coords(tile, Mt, Nt, &tm, &tn);
                const long long m0 = (long long)tm * 2 * kGemmBM + (long long)rank * kGemmBM;
                int map_id = (int)(m0 / a.rows_per_shard);
                if (map_id >= a.nmaps) map_id = a.nmaps - 1;   // rows past M: zero fill
                const int a_row = (int)(m0 - (long long)map_id * a.rows_per_shard);
                const CUtensorMap* amap = &maps.a[map_id];
                const int b_row = tn * kGemm2BN + (int)rank * kGemm2HalfN;
                for (int kb = 0; kb < KB; ++kb, ++g) {
                    if (g >= S && !mbar_wait(smem_addr(&tail->empty[s]), ph ^ 1u, abort,
                                             ERR_WAIT_EMPTY)) {
                        ok = false;
                        break;
                    }
                    const uint32_t full_leader = peer_addr(smem_addr(&tail->full[s]), 0u);
                    if (rank == 0) mbar_arrive_expect_tx(smem_addr(&tail->full[s]), 2 * kStage);
                    const uint32_t sa = smem_addr(gsm + (size_t)s * kStage);
                    tma_load_2d_pair(sa, amap, kb * kGemmBK, a_row, full_leader, pol);
                    tma_load_2d_pair(sa + kABytes, bmap, kb * kGemmBK, b_row, full_leader, pol);
                    tail->issued = g + 1;
                    if (++s == S) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            constexpr uint32_t idesc = idesc_bf16(2 * kGemmBM, kGemm2BN);
            int s = 0;         // stage of the next k-step
            uint32_t ph = 0;   // parity of its fill
            bool ok = true;
            long long it = 0;
            for (long long tile = cl; ok && tile < T; tile += ncl, ++it) {
                const int as = (int)(it & 1);
                const uint32_t use = (uint32_t)(it >> 1);
                // both CTAs' epilogues have read this accumulator stage's
                // previous tile (a fresh barrier passes parity 1 at once)
                if (!mbar_wait_cluster(smem_addr(&tail->acc_empty[as]), (use & 1u) ^ 1u, abort,
                                       ERR_WAIT_EMPTY))
                    break;
                tmem_fence_after_sync();
                const uint32_t tacc = tbase + (uint32_t)(as * kGemm2BN);
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
                        umma_bf16_pair(tacc, ad + 2 * k, bd + 2 * k, idesc,
                                       (kb > 0 || k > 0) ? 1u : 0u);
                    // stage s may be refilled, in both CTAs
                    umma_commit_pair(smem_addr(&tail->empty[s]));
                    umma_commit_pair(peer_addr(smem_addr(&tail->empty[s]), 1u));
                    if (++s == S) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) break;
                // the accumulator stage is complete, in both CTAs
                umma_commit_pair(smem_addr(&tail->acc_full[as]));
                umma_commit_pair(peer_addr(smem_addr(&tail->acc_full[as]), 1u));
            }
            // every issued MMA has finished (with its reads of both CTAs'
            // shared memory and its writes to both CTAs' tensor memory)
            umma_commit_pair(smem_addr(&tail->drain));
            volatile int no_abort = 0;
            mbar_wait(smem_addr(&tail->drain), 0u, &no_abort, ERR_DRAIN);
        }
    } else {
        // epilogue warps 2..5: warp w owns accumulator lanes 32 (w % 4) ..
        const int q = warp & 3;
        const uint32_t acc_empty_leader0 = peer_addr(smem_addr(&tail->acc_empty[0]), 0u);
        const uint32_t acc_empty_leader1 = peer_addr(smem_addr(&tail->acc_empty[1]), 0u);
        long long it = 0;
        for (long long tile = cl; tile < T; tile += ncl, ++it) {
            int tm, tn;
            gemm2_tile_coords(tile, Mt, Nt, &tm, &tn);
            const int as = (int)(it & 1);
            const uint32_t use = (uint32_t)(it >> 1);
            const long long m = (long long)tm * 2 * kGemmBM + (long long)rank * kGemmBM + 32 * q + lane;
            const int n0 = tn * kGemm2BN;
            if (!mbar_wait(smem_addr(&tail->acc_full[as]), use & 1u, abort, ERR_WAIT_FULL)) break;
            tmem_fence_after_sync();
            const bool row_ok = m < a.M;
            const uint32_t trow = tbase + ((uint32_t)(32 * q) << 16) + (uint32_t)(as * kGemm2BN);
#pragma unroll 1
            for (int c0 = 0; c0 < kGemm2BN; c0 += 32) {
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
            // this warp's reads of the stage are done: tell the leader
            tmem_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive_peer(as ? acc_empty_leader1 : acc_empty_leader0);
        }
    }
    // neither CTA frees the pair's tensor memory or leaves while the other
    // (or the leader's MMAs) may still use its memory
    tmem_fence_before_sync();
    __syncwarp();
    cluster_sync_all();
    if (rank == 0 && threadIdx.x == 0) {
        // every copy either CTA issued completes on the leader's full
        // barriers: wait (bounded) for the last S of the longer stream; after
        // a normal run they have all completed already
        long long peer_issued;
        asm volatile("ld.shared::cluster.s64 %0, [%1];"
                     : "=l"(peer_issued)
                     : "r"(peer_addr(smem_addr(&tail->issued), 1u))
                     : "memory");
        const long long gmax = tail->issued > peer_issued ? tail->issued : peer_issued;
        for (long long i = gmax > S ? gmax - S : 0; i < gmax; ++i) {
            volatile int no_abort = 0;
            if (!mbar_wait(smem_addr(&tail->full[i % S]), (uint32_t)((i / S) & 1), &no_abort,
                           ERR_DRAIN))
                break;
        }
    }
    cluster_sync_all();
    if (warp == 1) {
        tmem_fence_after_sync();
        tmem_dealloc_pair(tbase, kGemm2TmemCols);
    }
}

}  // namespace spk
