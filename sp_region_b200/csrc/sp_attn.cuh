// Ring attention (context parallelism) on sm_100a tensor cores.
//
// "Sequence Parallelism math", section "Context parallelism and ring
// attention": Q, K and V are sharded along the sequence, rank r holding the
// contiguous block r of s/t tokens; at step i rank r attends its queries
// against K/V block (r - i) mod t and folds the result into an online
// softmax, so after t steps every query has seen every key and no rank ever
// holds more than an (s/t) x (s/t) tile of scores.
//
// On one GPU the t ranks' blocks are consecutive key ranges of one K/V
// tensor, and a CTA whose queries lie in rank r's block visits the key tiles
// in ring order: block r first, then r-1, r-2, ... (mod t), 128 keys per
// tile.
//
// k_ring_attn<QT>: one CTA per QT 128-query tiles of one head (QT = 2 when a
// rank's block holds an even number of tiles, so both tiles visit the key
// tiles in the same ring order and share every K / V tile); head dim 128.
//   warp 0 (one lane)  TMA producer: the Q tiles once, K and V tiles (2
//                      stages each)
//   warp 1 (one lane)  MMA issuer.  S_j = Q K_j^T (tcgen05 kind::f16, M = N =
//                      128) into a tensor-memory score buffer, and O += P_j V_j
//                      with P_j read from tensor memory (where the softmax
//                      wrote it over S_j) and V read as an MN-major operand.
//                      QT = 1: two score buffers by tile parity, in the order
//                      S0, S1, PV0, S2, PV1, ...  QT = 2: one score buffer per
//                      query tile, in the order S_A0, S_B0, PV_A0, S_A1, PV_B0,
//                      S_B1, ..., so the tensor cores run one query tile's PV
//                      and next scores while the other tile's softmax runs.
//                      The tensor cores run one CTA's MMAs in issue order, so
//                      S overwrites a buffer only after the PV that read the
//                      P there.
//   softmax warps      8 per query tile: each query row is shared by two warps
//                      of the same sub-partition (they read the same
//                      tensor-memory lanes), one taking score columns 0..63,
//                      the other 64..127.  The pair exchanges its halves'
//                      maxima once per tile; both keep the same running
//                      maximum, so their partial sums add up at the end.  The
//                      maximum used for the exponentials moves only when a
//                      row's true maximum exceeds it by more than 8 (log2
//                      units): the probabilities then stay below 2^8, and O is
//                      rescaled in tensor memory only on those tiles, so in
//                      most tiles the softmax never waits for the previous
//                      PV.  One exponential pair in 8 is a cubic on the FMA
//                      pipe, the rest the transcendental unit's.  P goes to
//                      tensor memory as bf16 pairs; at the end O / l to
//                      global memory and the log-sum-exp
// Tensor memory: QT = 1: S0/P0 [0, 128), S1/P1 [128, 256), O [256, 384);
// QT = 2: S/P of tile A [0, 128), of tile B [128, 256), O_A [256, 384), O_B
// [384, 512).
#pragma once

#include "sp_gemm.cuh"

namespace spk {

constexpr int kAttnBM = 128;        // queries per CTA
constexpr int kAttnBN = 128;        // keys per tile
constexpr int kAttnD = 128;         // head dimension
constexpr int kAttnSplit = 2;                      // softmax warps per query row
constexpr int kAttnCols = 128 / kAttnSplit;        // score columns per softmax warp
constexpr int kAttnSoftWarps = 4 * kAttnSplit;     // softmax warps per query tile
__host__ __device__ constexpr int attn_threads(int qt) { return 64 + qt * kAttnSoftWarps * 32; }
constexpr uint32_t kAttnTile = 128 * 128 * 2;   // one 128 x 128 bf16 tile (two 64-column chunks)

struct AttnArgs {
    long long s;              // sequence length
    int t;                    // ranks of the ring
    int tiles_per_block;      // (s / t) / 128
    float scale_log2;         // score scale * log2(e)
    void* out;                // [bh][s][128] bf16
    float* lse;               // [bh][s] natural-log sum of exp(scores), or NULL
    // work items (one CTA each): items [0, full_units) are whole units (QT
    // query tiles of one head, every ring step); each later unit is split into
    // `split` contiguous ranges of ring steps whose unnormalised results go to
    // part_o / part_ml for k_attn_merge
    int nx;                   // units per head: s / (QT * 128)
    int full_units;
    int split;
    float* part_o;            // [item - full_units][QT * 128][128] fp32: O
    float* part_ml;           // [item - full_units][QT * 128][2] fp32: maximum in use (log2), sum
};

struct AttnMaps {
    CUtensorMap q, k, v;      // [bh * s][128] bf16, boxes of 64 x 128
};

// Barriers and scratch after the tiles; arrays of 2 are indexed by the score
// buffer (tile parity for QT = 1, query tile for QT = 2).
template <int QT>
struct AttnTail {
    uint64_t q_full;
    uint64_t k_full[2], k_empty[2];
    uint64_t v_full[2], v_empty[2];
    uint64_t s_full[2];          // S in buffer
    uint64_t p_full[2];          // P in buffer (and O rescaled for its tile)
    uint64_t o_done[2];          // the PV that read buffer's P complete
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
    uint64_t pair[QT][4][2];     // per query tile, row quarter and tile parity: every slice's maximum posted
    uint64_t pair_fin[QT][4];    // per query tile and row quarter: every slice's sum posted
    float xmax[QT][2][kAttnSplit][kAttnBM];   // [query tile][tile parity][column slice][row]
    float xsum[QT][kAttnSplit][kAttnBM];      // [query tile][column slice][row]
};

// Shared-memory descriptor of an MN-major tile with 128-byte swizzle: 64
// MN-elements per 128-byte row, 8 K-rows per 1024-byte group (stride byte
// offset, between K groups) and mn_stride bytes between 64-element MN atoms
// (leading byte offset).
__device__ __forceinline__ uint64_t sw128_desc_mn(uint32_t saddr, uint32_t mn_stride)
{
    uint64_t d = (uint64_t)((saddr & 0x3FFFFu) >> 4);
    d |= (uint64_t)((mn_stride >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)(1024 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t r[32])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, "
        "%10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, "
        "%27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
        "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
        "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

// D (+)= A B with A (M x K, K-major) in tensor memory, B in shared memory.
__device__ __forceinline__ void umma_bf16_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc,
                                             uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
        "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// 2^x for both halves on the FMA pipe: x = n + f with n the nearest integer
// (the 1.5 * 2^23 rounding constant) and f in [-1/2, 1/2]; 2^f by a cubic
// fitted to it in relative error on that interval (at most 7.5e-5, far
// below the bf16 rounding P gets); 2^n added to the exponent field.  x is
// clamped at -125, where the result (2^-125) is negligible against the row
// sum, so the exponent field never underflows.
__device__ __forceinline__ F2 exp2_poly2(F2 x)
{
    const float2 xs = halves(x);
    const F2 xc = f2(fmaxf(xs.x, -125.0f), fmaxf(xs.y, -125.0f));
    const F2 sh = add2(xc, f2(12582912.0f));
    const F2 n = sub2(sh, f2(12582912.0f));
    const F2 fr = sub2(xc, n);
    F2 p = fma2(f2(0x1.c3f610p-5f), fr, f2(0x1.f0de1cp-3f));
    p = fma2(p, fr, f2(0x1.62f31ep-1f));
    p = fma2(p, fr, f2(0x1.fff692p-1f));
    const float2 ps = halves(p), ss = halves(sh);
    return f2(__int_as_float(__float_as_int(ps.x) + (__float_as_int(ss.x) << 23)),
              __int_as_float(__float_as_int(ps.y) + (__float_as_int(ss.y) << 23)));
}

// 2^x by the transcendental unit's approximation (PTX ex2.approx.ftz: at most
// 2 ulp; results below 2^-126 flush to zero).
__device__ __forceinline__ float ex2_approx(float x)
{
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ float max3f(float a, float b, float c)
{
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// The running maximum (log2 units) moves only when the tile's exceeds it by
// more than this, bounding the probabilities by 2^8.
constexpr float kAttnMaxSlack = 8.0f;

template <int QT>
__global__ void __launch_bounds__(attn_threads(QT), 1)
    k_ring_attn(const __grid_constant__ AttnArgs a, const __grid_constant__ AttnMaps maps)
{
    extern __shared__ __align__(1024) unsigned char asm_raw[];
    unsigned char* sm = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(asm_raw) + 1023) & ~(uintptr_t)1023);
    unsigned char* sq = sm;                                   // Q: QT tiles of 2 chunks
    unsigned char* sk = sm + QT * kAttnTile;                  // K: 2 stages
    unsigned char* sv = sm + (QT + 2) * kAttnTile;            // V: 2 stages
    AttnTail<QT>* tail = reinterpret_cast<AttnTail<QT>*>(sm + (QT + 4) * kAttnTile);
    volatile int* abort = &tail->abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int T = a.tiles_per_block;
    const int n_tiles = a.t * T;
    // this CTA's work item: a unit and the ring steps [j0, j0 + n_loc) of it;
    // slot >= 0: a piece of a split unit, whose result is partial
    int unit = (int)blockIdx.x, j0 = 0, n_loc = n_tiles, slot = -1;
    if (unit >= a.full_units) {
        slot = unit - a.full_units;
        const int pc = slot % a.split;
        unit = a.full_units + slot / a.split;
        j0 = (int)((long long)n_tiles * pc / a.split);
        n_loc = (int)((long long)n_tiles * (pc + 1) / a.split) - j0;
    }
    const long long q0 = (long long)(unit % a.nx) * (QT * kAttnBM);   // first query row
    const long long g = unit / a.nx;                                  // batch * head index
    const long long per = a.s / a.t;
    const int rank = (int)(q0 / per);                                 // the queries' rank
    // first key row of tile j: block (rank - j / T) mod t, its (j % T)-th tile
    auto kv_row = [&](int j) -> long long {
        const int blk = ((rank - j / T) % a.t + a.t) % a.t;
        return (long long)blk * per + (long long)(j % T) * kAttnBN;
    };
    // score buffer of query tile qt at key tile j, and the phase of its barriers
    auto sbuf = [](int qt, int j) -> int { return QT == 1 ? (j & 1) : qt; };
    auto sphase = [](int j) -> uint32_t { return QT == 1 ? (uint32_t)((j >> 1) & 1) : (uint32_t)(j & 1); };

    if (threadIdx.x == 0) {
        mbar_init(smem_addr(&tail->q_full), 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_addr(&tail->k_full[i]), 1);
            mbar_init(smem_addr(&tail->k_empty[i]), 1);
            mbar_init(smem_addr(&tail->v_full[i]), 1);
            mbar_init(smem_addr(&tail->v_empty[i]), 1);
            mbar_init(smem_addr(&tail->s_full[i]), 1);
            mbar_init(smem_addr(&tail->p_full[i]), kAttnSoftWarps);   // a query tile's softmax warps
            mbar_init(smem_addr(&tail->o_done[i]), 1);
        }
        mbar_init(smem_addr(&tail->drain), 1);
        for (int t = 0; t < QT; ++t)
            for (int qq = 0; qq < 4; ++qq) {   // every thread of the row's warps arrives
                mbar_init(smem_addr(&tail->pair[t][qq][0]), 32 * kAttnSplit);
                mbar_init(smem_addr(&tail->pair[t][qq][1]), 32 * kAttnSplit);
                mbar_init(smem_addr(&tail->pair_fin[t][qq]), 32 * kAttnSplit);
            }
        tail->abort = 0;
        mbar_init_fence();
    }
    if (warp == 1) {
        tmem_alloc(smem_addr(&tail->tmem_base), 512);
        tmem_fence_before_sync();
    }
    if (threadIdx.x == 0) {
        tma_prefetch_desc(&maps.q);
        tma_prefetch_desc(&maps.k);
        tma_prefetch_desc(&maps.v);
    }
    __syncthreads();
    tmem_fence_after_sync();
    const uint32_t tbase = tail->tmem_base;
    grid_dep_launch();
    grid_dep_wait();

    if (warp == 0) {
        if (lane == 0) {
            const uint64_t pol = policy_evict_last();
            const uint32_t qb = smem_addr(&tail->q_full);
            mbar_arrive_expect_tx(qb, QT * kAttnTile);
            for (int t = 0; t < QT; ++t) {
                const int qrow = (int)(g * a.s + q0 + t * kAttnBM);
                tma_load_2d(smem_addr(sq + (size_t)t * kAttnTile), &maps.q, 0, qrow, qb, pol);
                tma_load_2d(smem_addr(sq + (size_t)t * kAttnTile) + kAttnTile / 2, &maps.q, 64, qrow,
                            qb, pol);
            }
            int issued = 0;
            for (int j = 0; j < n_loc; ++j) {   // local step j: ring step j0 + j
                const int st = j & 1;
                const int krow = (int)(g * a.s + kv_row(j0 + j));
                if (j >= 2 && !mbar_wait(smem_addr(&tail->k_empty[st]),
                                         (uint32_t)(((j >> 1) - 1) & 1), abort, ERR_WAIT_EMPTY))
                    break;
                const uint32_t kb = smem_addr(&tail->k_full[st]);
                const uint32_t kd = smem_addr(sk + (size_t)st * kAttnTile);
                mbar_arrive_expect_tx(kb, kAttnTile);
                tma_load_2d(kd, &maps.k, 0, krow, kb, pol);
                tma_load_2d(kd + kAttnTile / 2, &maps.k, 64, krow, kb, pol);
                if (j >= 2 && !mbar_wait(smem_addr(&tail->v_empty[st]),
                                         (uint32_t)(((j >> 1) - 1) & 1), abort, ERR_WAIT_EMPTY)) {
                    ++issued;   // the K copies of this tile are in flight
                    break;
                }
                const uint32_t vb = smem_addr(&tail->v_full[st]);
                const uint32_t vd = smem_addr(sv + (size_t)st * kAttnTile);
                mbar_arrive_expect_tx(vb, kAttnTile);
                tma_load_2d(vd, &maps.v, 0, krow, vb, pol);
                tma_load_2d(vd + kAttnTile / 2, &maps.v, 64, krow, vb, pol);
                ++issued;
            }
            if (*abort) {
                // every issued copy lands before the CTA's memory goes away
                volatile int no_abort = 0;
                mbar_wait(smem_addr(&tail->q_full), 0u, &no_abort, ERR_DRAIN);
                const int first = issued > 2 ? issued - 2 : 0;
                for (int i = first; i < issued; ++i) {
                    mbar_wait(smem_addr(&tail->k_full[i & 1]), (uint32_t)((i >> 1) & 1),
                              &no_abort, ERR_DRAIN);
                    mbar_wait(smem_addr(&tail->v_full[i & 1]), (uint32_t)((i >> 1) & 1),
                              &no_abort, ERR_DRAIN);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16(kAttnBM, kAttnBN);
            constexpr uint32_t idesc_o = idesc_bf16(kAttnBM, kAttnD) | (1u << 16);  // B MN-major
            bool ok = mbar_wait(smem_addr(&tail->q_full), 0u, abort, ERR_WAIT_FULL);
            // S = Q_qt K_j^T into buffer sbuf(qt, j), after the PV that read
            // the P there; the K tile is freed after its last query tile
            auto issue_s = [&](int qt, int j) -> bool {
                const int b = sbuf(qt, j);
                if (qt == 0 && !mbar_wait(smem_addr(&tail->k_full[j & 1]), (uint32_t)((j >> 1) & 1),
                                          abort, ERR_WAIT_FULL))
                    return false;
                tmem_fence_after_sync();
                const uint32_t q_s = smem_addr(sq + (size_t)qt * kAttnTile);
                const uint32_t k_s = smem_addr(sk + (size_t)(j & 1) * kAttnTile);
#pragma unroll
                for (int kk = 0; kk < kAttnD / 16; ++kk) {
                    // 16 of the 128 head features: chunk kk / 4, 32 bytes each
                    const uint32_t off = (uint32_t)(kk >> 2) * (kAttnTile / 2) + (uint32_t)(kk & 3) * 32;
                    umma_bf16(tbase + (uint32_t)(b * kAttnBN), sw128_desc(q_s + off),
                              sw128_desc(k_s + off), idesc_s, kk > 0 ? 1u : 0u);
                }
                if (qt == QT - 1) umma_commit(smem_addr(&tail->k_empty[j & 1]));
                umma_commit(smem_addr(&tail->s_full[b]));
                return true;
            };
            // O_qt += P V_j, P from buffer sbuf(qt, j); the V tile is freed
            // after its last query tile
            auto issue_pv = [&](int qt, int j) -> bool {
                const int b = sbuf(qt, j);
                if (!mbar_wait(smem_addr(&tail->p_full[b]), sphase(j), abort, ERR_WAIT_FULL) ||
                    (qt == 0 && !mbar_wait(smem_addr(&tail->v_full[j & 1]),
                                           (uint32_t)((j >> 1) & 1), abort, ERR_WAIT_FULL)))
                    return false;
                tmem_fence_after_sync();
                const uint32_t v_s = smem_addr(sv + (size_t)(j & 1) * kAttnTile);
#pragma unroll
                for (int kk = 0; kk < kAttnBN / 16; ++kk) {
                    // keys 16 kk .. 16 kk + 15: P columns (two bf16 a column)
                    // at the start of the score columns of the slice that
                    // holds those keys, V rows 16 kk .. (two 8-row groups of
                    // 1024 bytes, MN-major)
                    const int slice = (16 * kk) / kAttnCols, kin = 16 * kk - slice * kAttnCols;
                    umma_bf16_ts(tbase + 256 + (uint32_t)(qt * kAttnD),
                                 tbase + (uint32_t)(b * kAttnBN + slice * kAttnCols + kin / 2),
                                 sw128_desc_mn(v_s + (uint32_t)kk * 2048, kAttnTile / 2), idesc_o,
                                 (j > 0 || kk > 0) ? 1u : 0u);
                }
                if (qt == QT - 1) umma_commit(smem_addr(&tail->v_empty[j & 1]));
                umma_commit(smem_addr(&tail->o_done[b]));
                return true;
            };
            if constexpr (QT == 1) {
                if (ok) ok = issue_s(0, 0);
                if (ok && n_loc > 1) ok = issue_s(0, 1);
                for (int j = 0; ok && j < n_loc; ++j) {
                    ok = issue_pv(0, j);
                    if (ok && j + 2 < n_loc) ok = issue_s(0, j + 2);
                }
            } else {
                if (ok) ok = issue_s(0, 0);
                if (ok) ok = issue_s(1, 0);
                for (int j = 0; ok && j < n_loc; ++j) {
                    ok = issue_pv(0, j);
                    if (ok && j + 1 < n_loc) ok = issue_s(0, j + 1);
                    if (ok) ok = issue_pv(1, j);
                    if (ok && j + 1 < n_loc) ok = issue_s(1, j + 1);
                }
            }
            // every issued MMA has finished before the CTA tears down
            umma_commit(smem_addr(&tail->drain));
            volatile int no_abort = 0;
            mbar_wait(smem_addr(&tail->drain), 0u, &no_abort, ERR_DRAIN);
        }
    } else {
        // softmax warps: query tile qt; row 32 (warp % 4) + lane of it; column
        // slice hf of the scores (and of O's columns); warps w, w + 4, ...
        // of a tile share rows
        const int sw = warp - 2;
        const int qt = sw / kAttnSoftWarps;
        const int q = warp & 3;
        const int hf = (sw % kAttnSoftWarps) >> 2;
        const int row = 32 * q + lane;
        const uint32_t tlane = (uint32_t)(32 * q) << 16;
        const uint32_t ocol = 256 + (uint32_t)(qt * kAttnD);
        // a bounded wait whose outcome is the same in every lane of the warp,
        // so the warp-collective tensor-memory accesses after it are uniform
        auto wait_all = [&](uint32_t bar, uint32_t parity) -> bool {
            const bool w = mbar_wait(bar, parity, abort, ERR_WAIT_FULL);
            return __all_sync(0xFFFFFFFFu, w) != 0;
        };
        float m = -INFINITY, l = 0.f;   // maximum in use (log2 units), this slice's sum
        bool ok = true;
        for (int j = 0; j < n_loc; ++j) {
            const int b = sbuf(qt, j);
            const int pb = j & 1;   // parity of the pair exchange
            if (!wait_all(smem_addr(&tail->s_full[b]), sphase(j))) {
                ok = false;
                break;
            }
            tmem_fence_after_sync();
            const uint32_t scol = tbase + tlane + (uint32_t)(b * kAttnBN + kAttnCols * hf);
            float mx;
            {
                // pass 1: the slice's maximum, 32 scores at a time, two
                // independent chains of three-input maxima
                float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
                for (int c = 0; c < kAttnCols / 32; ++c) {
                    uint32_t sc[32];
                    tmem_ld32(scol + 32 * c, sc);
#pragma unroll
                    for (int i = 0; i < 32; i += 4) {
                        m0 = max3f(m0, __uint_as_float(sc[i]), __uint_as_float(sc[i + 1]));
                        m1 = max3f(m1, __uint_as_float(sc[i + 2]), __uint_as_float(sc[i + 3]));
                    }
                }
                mx = fmaxf(m0, m1);
            }
            tail->xmax[qt][pb][hf][row] = mx;
            mbar_arrive(smem_addr(&tail->pair[qt][q][pb]));
            if (!wait_all(smem_addr(&tail->pair[qt][q][pb]), (uint32_t)((j >> 1) & 1))) {
                ok = false;
                break;
            }
#pragma unroll
            for (int h = 0; h < kAttnSplit; ++h) mx = fmaxf(mx, tail->xmax[qt][pb][h][row]);
            mx *= a.scale_log2;   // the row's maximum
            const bool bump = mx > m + kAttnMaxSlack;   // first tile: m = -inf
            const float alpha = bump ? ex2_approx(m - mx) : 1.0f;   // 0 at the first tile
            if (bump) m = mx;
            // pass 2: p = 2^(s * scale - m), the scaling as paired fused
            // multiply-adds, the sum in two pair lanes; P as bf16 pairs over
            // this warp's own score columns (32 scores read, then 16 columns
            // of P written behind them), so no other warp's scores are touched
            const F2 scale2 = f2(a.scale_log2), negm2 = f2(-m);
            F2 lsum2 = f2(0.f);
#pragma unroll
            for (int c = 0; c < kAttnCols / 32; ++c) {
                uint32_t sc[32], pk[16];
                tmem_ld32(scol + 32 * c, sc);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const F2 x2 = fma2(f2(__uint_as_float(sc[2 * i]), __uint_as_float(sc[2 * i + 1])),
                                       scale2, negm2);
                    F2 p2;
                    if ((i & 7) == 7) {
                        // one pair in 8 on the FMA pipe: the transcendental
                        // unit is the softmax's critical resource (16384
                        // exponentials a tile against the other query tile's
                        // MMAs); more than 1 in 8 costs more issue than it saves
                        p2 = exp2_poly2(x2);
                    } else {
                        const float2 x = halves(x2);
                        p2 = f2(ex2_approx(x.x), ex2_approx(x.y));
                    }
                    lsum2 = add2(lsum2, p2);
                    const float2 pp = halves(p2);
                    pk[i] = IO<__nv_bfloat16>::pack2(pp.x, pp.y);
                }
                tmem_st16(scol + 16 * c, pk);
            }
            l = l * alpha + hsum(lsum2);
            if (j > 0 && __any_sync(0xFFFFFFFFu, bump)) {
                // O of the previous tiles is complete: rescale this slice
                const int b_prev = sbuf(qt, j - 1);
                if (!wait_all(smem_addr(&tail->o_done[b_prev]), sphase(j - 1))) {
                    ok = false;
                    break;
                }
                tmem_fence_after_sync();
#pragma unroll 1
                for (int c = 0; c < kAttnCols / 32; ++c) {
                    uint32_t o[32];
                    const uint32_t oc = tbase + tlane + ocol + (uint32_t)(kAttnCols * hf + 32 * c);
                    tmem_ld32(oc, o);
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                    tmem_st32(oc, o);
                }
            }
            tmem_wait_st();
            tmem_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_addr(&tail->p_full[b]));
        }
        // the row's sum: every slice posts its own (a warp that left the loop
        // early makes the others' bounded wait run out, never hang)
        tail->xsum[qt][hf][row] = l;
        mbar_arrive(smem_addr(&tail->pair_fin[qt][q]));
        if (ok && !wait_all(smem_addr(&tail->pair_fin[qt][q]), 0u)) ok = false;
        float lt = tail->xsum[qt][0][row];   // the same order, so the same bits, in every warp
#pragma unroll
        for (int h = 1; h < kAttnSplit; ++h) lt += tail->xsum[qt][h][row];
        const int b_last = sbuf(qt, n_loc - 1);
        const bool o_ready = ok && wait_all(smem_addr(&tail->o_done[b_last]), sphase(n_loc - 1));
        if (o_ready && slot >= 0) {
            // a piece of a split unit: O as accumulated (scaled by 2^-m), m
            // and the row's sum, for k_attn_merge
            tmem_fence_after_sync();
            const size_t prow = (size_t)slot * (QT * kAttnBM) + (size_t)qt * kAttnBM + row;
            float* po = a.part_o + prow * kAttnD + kAttnCols * hf;
#pragma unroll 1
            for (int c = 0; c < kAttnCols / 32; ++c) {
                uint32_t o[32];
                tmem_ld32(tbase + tlane + ocol + (uint32_t)(kAttnCols * hf + 32 * c), o);
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    *reinterpret_cast<float4*>(po + 32 * c + 4 * u) =
                        make_float4(__uint_as_float(o[4 * u]), __uint_as_float(o[4 * u + 1]),
                                    __uint_as_float(o[4 * u + 2]), __uint_as_float(o[4 * u + 3]));
            }
            if (hf == 0) *reinterpret_cast<float2*>(a.part_ml + 2 * prow) = make_float2(m, lt);
        } else if (o_ready) {
            tmem_fence_after_sync();
            const float inv = 1.0f / lt;
            const long long qrow = q0 + (long long)qt * kAttnBM + row;
            unsigned char* orow = static_cast<unsigned char*>(a.out) +
                                  ((size_t)g * a.s + qrow) * (kAttnD * 2);
#pragma unroll 1
            for (int c = 0; c < kAttnCols / 32; ++c) {
                uint32_t o[32];
                tmem_ld32(tbase + tlane + ocol + (uint32_t)(kAttnCols * hf + 32 * c), o);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    F2 f[4];
#pragma unroll
                    for (int p = 0; p < 4; ++p)
                        f[p] = f2(__uint_as_float(o[8 * u + 2 * p]) * inv,
                                  __uint_as_float(o[8 * u + 2 * p + 1]) * inv);
                    store_vec<__nv_bfloat16>(orow, (kAttnCols / 8) * hf + 4 * c + u,
                                             IO<__nv_bfloat16>::pack2v(f));
                }
            }
            if (a.lse && hf == 0)
                a.lse[(size_t)g * a.s + qrow] = (m + log2f(lt)) * 0.69314718055994531f;
        }
    }
    tmem_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tmem_fence_after_sync();
        tmem_dealloc(tbase, 512);
    }
}

// The pieces of each split unit, combined in piece order: with m_i the
// maximum a piece's exponentials used (log2 units), l_i its row sum and O_i
// its accumulated output, M = max m_i, L = sum 2^(m_i - M) l_i and the row's
// output is sum 2^(m_i - M) O_i / L, its log-sum-exp (M + log2 L) ln 2.  One
// warp per query row; lane l owns head features 4l .. 4l + 3.
constexpr int kAttnMergeThreads = 256;

static __global__ void __launch_bounds__(kAttnMergeThreads)
    k_attn_merge(const __grid_constant__ AttnArgs a, int rows_per_unit, long long rows)
{
    grid_dep_launch();
    grid_dep_wait();   // every piece is written and visible
    const long long r = (long long)blockIdx.x * (kAttnMergeThreads / 32) + (threadIdx.x >> 5);
    if (r >= rows) return;   // uniform over the warp
    const int lane = threadIdx.x & 31;
    const long long u_t = r / rows_per_unit;   // split unit, counted from the first one
    const int rr = (int)(r - u_t * rows_per_unit);
    const long long unit = a.full_units + u_t;
    const long long g = unit / a.nx;
    const long long qrow = (unit % a.nx) * rows_per_unit + rr;
    const size_t prow0 = (size_t)u_t * a.split * rows_per_unit + rr;   // piece 0's row
    float M = -INFINITY;
    for (int pc = 0; pc < a.split; ++pc)
        M = fmaxf(M, a.part_ml[2 * (prow0 + (size_t)pc * rows_per_unit)]);
    float L = 0.f;
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int pc = 0; pc < a.split; ++pc) {
        const size_t prow = prow0 + (size_t)pc * rows_per_unit;
        const float2 ml = *reinterpret_cast<const float2*>(a.part_ml + 2 * prow);
        const float w = exp2f(ml.x - M);
        L += w * ml.y;
        const float4 x = *reinterpret_cast<const float4*>(a.part_o + prow * kAttnD + 4 * lane);
        o.x += w * x.x;
        o.y += w * x.y;
        o.z += w * x.z;
        o.w += w * x.w;
    }
    const float inv = 1.0f / L;
    const uint2 pk = make_uint2(IO<__nv_bfloat16>::pack2(o.x * inv, o.y * inv),
                                IO<__nv_bfloat16>::pack2(o.z * inv, o.w * inv));
    *reinterpret_cast<uint2*>(static_cast<unsigned char*>(a.out) +
                              ((size_t)g * a.s + qrow) * (kAttnD * 2) + 8 * lane) = pk;
    if (a.lse && lane == 0) a.lse[(size_t)g * a.s + qrow] = (M + log2f(L)) * 0.69314718055994531f;
}

}  // namespace spk
