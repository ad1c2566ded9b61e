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
// so the row never sits in registers.  The per-thread parameter-gradient
// partials (3 * 8V fp32) live in registers, in shared memory, or in tensor
// memory.  Tensor memory (256 KB per SM, outside both the register file and
// shared memory) is the default: it costs neither registers nor ring stages,
// and each thread keeps its own set, so the sums have a fixed order per
// consumer group.  With the shared-memory set, several consumer groups share
// one set and take turns in the CTA's row order (two turn barriers, one for
// each accumulating pass), so the sums stay bitwise deterministic while the
// groups' reduce-scatter phases overlap.
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
    void* dY[kMaxT];         // n_dY full [s,b,h] buffers, indexed by global row
    int n_dY;                // 0: no dY; t: every rank's copy (the all-gather)
    float* ws;               // [gridDim.x][3][h] per-CTA partial sums
    long long rows;          // token rows of this call (local index i)
    long long row0;          // global index of local row 0: n = row0 + i
    int h;
    int hv;
    int t;
    int stages;
    uint32_t seg_bytes;
    uint32_t res_seg_bytes;  // h * residual stream elem bytes (x, dR_next, dres)
    int res_f32;             // residual stream in fp32 (I/O dtype bf16)
    uint32_t stage_stride;
    int mask_row_bytes;
    uint32_t param_off;      // shared-memory offsets (fast kernel): gamma copy,
    uint32_t acc_off;        //   parameter-gradient accumulators (ACC_SMEM),
    uint32_t tail_off;       //   barriers / scratch
    float inv_h;             // 1 / h, rounded to fp32
    float scale;
    int want_dbeta;
    int want_dbias;
    uint32_t tmem_cols;      // tensor-memory columns allocated (ACC = 2)
    int fold;                // ACC = 2, G > 1: the groups' sums are added in the CTA
};

// ACC: where the per-CTA parameter-gradient partials live.  0: registers,
// one set per consumer group.  1: shared memory, one set per CTA that the
// groups update by turns.  2: tensor memory, one private set per thread:
// warp w uses the columns [(w / 4) * 24V, (w / 4 + 1) * 24V) of its lane
// quarter, 24 columns per vector i (dgamma, dbeta, dbias; 8 each).
// EXACT: the threads' vectors tile the row exactly (C * V == hv), so the
// per-vector bounds checks compile away.
template <typename T, int V, int G, int MAXT, bool LN, int ACC, bool EXACT = false>
__global__ void __launch_bounds__(MAXT, 1) k_bwd_tma(const __grid_constant__ BwdArgs a)
{
    constexpr bool ACC_SMEM = ACC == 1;
    constexpr bool ACC_TMEM = ACC == 2;
    constexpr bool ACC_REGS = ACC == 0;
    using Vec = typename IO<T>::Vec;
    extern __shared__ __align__(128) unsigned char smem[];
    RingTail* tail = reinterpret_cast<RingTail*>(smem + a.tail_off);
    // gamma copy and, for ACC_SMEM, the per-CTA accumulators [3][2][hv][4]
    // fp32; every slot is private to the thread that owns its vector
    unsigned char* sgam = smem + a.param_off;
    ulonglong2* accs = reinterpret_cast<ulonglong2*>(smem + a.acc_off);
    volatile int* abort = &tail->abort;

    const int C = (blockDim.x - 32) / G;
    const int tid = threadIdx.x;
    const int S = a.stages;
    const int nsrc = a.t + 1 + (a.drnext ? 1 : 0);   // dP_k..., x, [dR_next]

    if (ACC_TMEM && tid < 32) {
        tmem_alloc(smem_addr(&tail->tmem_base), a.tmem_cols);
        tmem_fence_before_sync();
    }
    init_ring(tail, S, C / 32);
    grid_dep_launch();
    grid_dep_wait();   // the previous kernel's outputs are visible

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
                                       (size_t)i * a.res_seg_bytes;
                            },
                            a.t, a.res_seg_bytes);
        return;
    }

    const int g = tid / C;
    const int c = tid - g * C;
    const int lane = tid & 31;
    const int bar_id = 1 + g;
    const int hv = a.hv;
    // fp32 pairs throughout (features 2p, 2p+1 of a vector in pair p)
    F2 ag[ACC_REGS ? V : 1][4], ab[ACC_REGS ? V : 1][4], ac[ACC_REGS ? V : 1][4];
    uint32_t tacc = 0;   // this thread's first tensor-memory accumulator
    if (ACC_TMEM) {
        tmem_fence_after_sync();
        const int w = tid >> 5;
        tacc = tail->tmem_base + ((uint32_t)(32 * (w & 3)) << 16) + (uint32_t)((w >> 2) * 24 * V);
        const uint32_t z[16] = {};
#pragma unroll
        for (int i = 0; i < V; ++i) {
            tmem_st16(tacc + 24 * i, z);
            tmem_st8(tacc + 24 * i + 16, z);
        }
    }
#pragma unroll
    for (int i = 0; i < V; ++i) {
        const int v = c + i * C;
        if (g == 0 && (EXACT || v < hv)) store_vec<T>(sgam, v, load_vec<T>(a.gamma, v));
        if (ACC_REGS) {
#pragma unroll
            for (int p = 0; p < 4; ++p) ag[i][p] = ab[i][p] = ac[i][p] = f2(0.f);
        } else if (ACC_SMEM && (EXACT || v < hv)) {
#pragma unroll
            for (int q = 0; q < 3; ++q) {
                accs[((size_t)q * 2 + 0) * hv + v] = make_ulonglong2(0ull, 0ull);
                accs[((size_t)q * 2 + 1) * hv + v] = make_ulonglong2(0ull, 0ull);
            }
        }
    }
    asm volatile("bar.sync %0, %1;" ::"r"(1 + kMaxGroups), "r"(G * C) : "memory");

    // accumulator q of vector v: pairs 0, 1 in the first 16 bytes, 2, 3 in
    // the second ([3][2][hv] slots of 16 bytes)
    auto acc_add = [&](int q, int v, const F2 d[4]) {
        ulonglong2* p0 = &accs[((size_t)q * 2 + 0) * hv + v];
        ulonglong2* p1 = &accs[((size_t)q * 2 + 1) * hv + v];
        ulonglong2 x0 = *p0, x1 = *p1;
        x0.x = add2(F2{x0.x}, d[0]).r;
        x0.y = add2(F2{x0.y}, d[1]).r;
        x1.x = add2(F2{x1.x}, d[2]).r;
        x1.y = add2(F2{x1.y}, d[3]).r;
        *p0 = x0;
        *p1 = x1;
    };
    // add d0 (and d1) to the 8 (16) tensor-memory cells at column offset col
    auto tmem_add8 = [&](uint32_t col, const F2 (&d0)[4]) {
        uint32_t r[8];
        tmem_ld8(tacc + col, r);
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const float2 x =
                halves(add2(f2(__uint_as_float(r[2 * p]), __uint_as_float(r[2 * p + 1])), d0[p]));
            r[2 * p] = __float_as_uint(x.x);
            r[2 * p + 1] = __float_as_uint(x.y);
        }
        tmem_st8(tacc + col, r);
    };
    auto tmem_add16 = [&](uint32_t col, const F2 (&d0)[4], const F2 (&d1)[4]) {
        uint32_t r[16];
        tmem_ld16(tacc + col, r);
#pragma unroll
        for (int p = 0; p < 8; ++p) {
            const float2 x = halves(add2(f2(__uint_as_float(r[2 * p]), __uint_as_float(r[2 * p + 1])),
                                         p < 4 ? d0[p] : d1[p - 4]));
            r[2 * p] = __float_as_uint(x.x);
            r[2 * p + 1] = __float_as_uint(x.y);
        }
        tmem_st16(tacc + col, r);
    };
    // a vector of a residual-stream tensor (x, dR_next) from shared memory
    auto load_res = [&](const unsigned char* buf, int v, F2 f[4]) {
        if (a.res_f32)
            IO<float>::unpack2(load_vec<float>(buf, v), f);
        else
            IO<T>::unpack2(load_vec<T>(buf, v), f);
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

    const F2 scale2 = f2(a.scale);
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
            kb[i] = (a.mask && (EXACT || v < hv)) ? a.mask[(size_t)i_row * a.mask_row_bytes + v] : 0xFFu;
        }

        // reduce-scatter of the upstream gradient partials, k ascending, from +0
        F2 dn[V][4];
#pragma unroll
        for (int i = 0; i < V; ++i)
#pragma unroll
            for (int p = 0; p < 4; ++p) dn[i][p] = f2(0.f);
        for (int k = 0; k < a.t; ++k) {
            mbar_wait(smem_addr(&tail->full[pos.abs()]), pos.phase, abort, ERR_WAIT_FULL);
            const unsigned char* buf = smem + (size_t)pos.abs() * a.stage_stride;
#pragma unroll
            for (int i = 0; i < V; ++i) {
                const int v = c + i * C;
                if (EXACT || v < hv) {
                    F2 f[4];
                    IO<T>::unpack2(load_vec<T>(buf, v), f);
#pragma unroll
                    for (int p = 0; p < 4; ++p) dn[i][p] = add2(dn[i][p], f[p]);
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
        const F2 mean2 = f2(mean), rstd2 = f2(rstd);
        auto xhat = [&](F2 xv) { return LN ? mul2(sub2(xv, mean2), rstd2) : mul2(xv, rstd2); };
        F2 sg2 = f2(0.f), sgx2 = f2(0.f);
        if (ACC_TMEM) {
            __syncwarp();
            tmem_wait_st();   // the previous row's updates have landed
        }
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const int v = c + i * C;
            F2 dgm[4] = {f2(0.f), f2(0.f), f2(0.f), f2(0.f)};
            if (EXACT || v < hv) {
                F2 xv[4], gm[4];
                load_res(xb, v, xv);
                IO<T>::unpack2(load_vec<T>(sgam, v), gm);
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    const F2 xh = xhat(xv[p]);
                    const F2 gg = mul2(dn[i][p], gm[p]);
                    sg2 = add2(sg2, gg);
                    sgx2 = fma2(gg, xh, sgx2);
                    dgm[p] = mul2(dn[i][p], xh);
                }
                if (ACC_SMEM) {
                    acc_add(0, v, dgm);
                    if (a.want_dbeta) acc_add(1, v, dn[i]);
                } else if (ACC_REGS) {
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        ag[ACC_REGS ? i : 0][p] = add2(ag[ACC_REGS ? i : 0][p], dgm[p]);
                        ab[ACC_REGS ? i : 0][p] = add2(ab[ACC_REGS ? i : 0][p], dn[i][p]);
                    }
                }
            }
            // warp-wide, outside the per-thread branch; vectors past the row
            // add zeros
            if (ACC_TMEM) {
                __syncwarp();
                if (a.want_dbeta)
                    tmem_add16(24 * i, dgm, dn[i]);
                else
                    tmem_add8(24 * i, dgm);
            }
        }
        pass_turn(0);
        float2 tot = make_float2(warp_sum(hsum(sg2)), warp_sum(hsum(sgx2)));
        {
            float2* red = reinterpret_cast<float2*>(tail->red[parity][g]);
            if (lane == 0) red[c >> 5] = tot;
            asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "r"(C) : "memory");
            tot = warps_total2(red, C >> 5);
        }
        const float mg = tot.x * a.inv_h, mgx = tot.y * a.inv_h;
        const F2 mg2 = f2(mg), nmgx2 = f2(-mgx);

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
            static_cast<unsigned char*>(a.dres) + (size_t)i_row * a.res_seg_bytes;   // shard
        const size_t dy_off = (size_t)n * a.seg_bytes;   // gathered: global row
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const int v = c + i * C;
            F2 dz[4] = {f2(0.f), f2(0.f), f2(0.f), f2(0.f)};
            if (EXACT || v < hv) {
                F2 xv[4], gm[4], dr[4];
                load_res(xb, v, xv);
                IO<T>::unpack2(load_vec<T>(sgam, v), gm);
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    const F2 xh = xhat(xv[p]);
                    const F2 gg = mul2(dn[i][p], gm[p]);
                    // rstd * (g - mean(g) - xhat * mean(g * xhat))
                    const F2 u = fma2(xh, nmgx2, LN ? sub2(gg, mg2) : gg);
                    dr[p] = mul2(rstd2, u);
                }
                if (rb) {
                    F2 rn[4];
                    load_res(rb, v, rn);
#pragma unroll
                    for (int p = 0; p < 4; ++p) dr[p] = add2(dr[p], rn[p]);
                }
#pragma unroll
                for (int p = 0; p < 4; ++p)
                    dz[p] = keep2(mul2(dr[p], scale2), (kb[i] >> (2 * p)) & 1u,
                                  (kb[i] >> (2 * p + 1)) & 1u);
                if (a.res_f32)
                    store_vec<float>(dres, v, IO<float>::pack2v(dr));
                else
                    store_vec<T>(dres, v, IO<T>::pack2v(dr));
                if (a.n_dY) {
                    // the all-gather of dY: this row into every rank's copy
                    const Vec dzv = IO<T>::pack2v(dz);
                    for (int q = 0; q < a.n_dY; ++q)
                        store_vec<T>(static_cast<unsigned char*>(a.dY[q]) + dy_off, v, dzv);
                }
                if (a.want_dbias) {
                    if (ACC_SMEM) {
                        acc_add(2, v, dz);
                    } else if (ACC_REGS) {
#pragma unroll
                        for (int p = 0; p < 4; ++p)
                            ac[ACC_REGS ? i : 0][p] = add2(ac[ACC_REGS ? i : 0][p], dz[p]);
                    }
                }
            }
            if (ACC_TMEM && a.want_dbias) {
                __syncwarp();
                tmem_add8(24 * i + 16, dz);
            }
        }
        pass_turn(1);
        release_at(sx);
        if (rb) release_at(sr);
    }

    // partial sums -> workspace: register accumulators give one slice per
    // group ([cta * G + g][q][h]); the shared set gives one slice per CTA
    // ([cta][q][h]), written by group 0 once every group has finished; the
    // tensor-memory sets give one per group, or one per CTA when folded
    if (ACC_SMEM) {
        if (G > 1) asm volatile("bar.sync %0, %1;" ::"r"(1 + kMaxGroups), "r"(G * C) : "memory");
        if (g != 0) return;
    }
    if (ACC_TMEM) {
        __syncwarp();
        tmem_wait_st();
    }
    // tensor-memory sums of a thread, vector i: 24 words (dgamma, dbeta, dbias)
    auto tmem_sums = [&](int i, uint32_t tr[24]) {   // warp-wide
        __syncwarp();
        tmem_ld16(tacc + 24 * i, tr);
        tmem_ld8(tacc + 24 * i + 16, tr + 16);
    };
    auto pair_of = [](const uint32_t* r) {   // 4 words -> two fp32 pairs
        return make_ulonglong2(f2(__uint_as_float(r[0]), __uint_as_float(r[1])).r,
                               f2(__uint_as_float(r[2]), __uint_as_float(r[3])).r);
    };
    if (ACC_TMEM && G > 1 && a.fold) {
        // One slice per CTA: once every row is consumed the ring is idle;
        // groups 1..G-1 stage their sums there ([g-1][q][2][hv] of 16
        // bytes) and group 0 adds them to its own in group order.
        ulonglong2* stg = reinterpret_cast<ulonglong2*>(smem);
        asm volatile("bar.sync %0, %1;" ::"r"(1 + kMaxGroups), "r"(G * C) : "memory");
        if (g > 0) {
#pragma unroll
            for (int i = 0; i < V; ++i) {
                const int v = c + i * C;
                uint32_t tr[24];
                tmem_sums(i, tr);
                if (EXACT || v < hv)
                    for (int q = 0; q < 3; ++q) {
                        ulonglong2* d = stg + ((size_t)(g - 1) * 3 + q) * 2 * hv;
                        d[v] = pair_of(tr + 8 * q);
                        d[hv + v] = pair_of(tr + 8 * q + 4);
                    }
            }
        }
        asm volatile("bar.sync %0, %1;" ::"r"(1 + kMaxGroups), "r"(G * C) : "memory");
        if (g == 0) {
            float* wsc = a.ws + (size_t)blockIdx.x * 3 * a.h;
#pragma unroll
            for (int i = 0; i < V; ++i) {
                const int v = c + i * C;
                uint32_t tr[24];
                tmem_sums(i, tr);
                if (EXACT || v < hv)
                    for (int q = 0; q < 3; ++q) {
                        ulonglong2 lo = pair_of(tr + 8 * q), hi = pair_of(tr + 8 * q + 4);
                        for (int gg = 1; gg < G; ++gg) {
                            const ulonglong2* d = stg + ((size_t)(gg - 1) * 3 + q) * 2 * hv;
                            const ulonglong2 x = d[v], y = d[hv + v];
                            lo = make_ulonglong2(add2(F2{lo.x}, F2{x.x}).r, add2(F2{lo.y}, F2{x.y}).r);
                            hi = make_ulonglong2(add2(F2{hi.x}, F2{y.x}).r, add2(F2{hi.y}, F2{y.y}).r);
                        }
                        ulonglong2* dst =
                            reinterpret_cast<ulonglong2*>(wsc + (size_t)q * a.h + 8 * (size_t)v);
                        dst[0] = lo;
                        dst[1] = hi;
                    }
            }
        }
    } else {
        float* ws = a.ws + (ACC_SMEM ? (size_t)blockIdx.x : (size_t)blockIdx.x * G + g) * 3 * a.h;
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const int v = c + i * C;
            uint32_t tr[24];
            if (ACC_TMEM) tmem_sums(i, tr);
            if (EXACT || v < hv) {
                for (int q = 0; q < 3; ++q) {
                    ulonglong2 lo, hi;
                    if (ACC_SMEM) {
                        lo = accs[((size_t)q * 2 + 0) * hv + v];
                        hi = accs[((size_t)q * 2 + 1) * hv + v];
                    } else if (ACC_TMEM) {
                        lo = pair_of(tr + 8 * q);
                        hi = pair_of(tr + 8 * q + 4);
                    } else {
                        const F2* s_ = q == 0 ? ag[ACC_REGS ? i : 0]
                                              : (q == 1 ? ab[ACC_REGS ? i : 0]
                                                        : ac[ACC_REGS ? i : 0]);
                        lo = make_ulonglong2(s_[0].r, s_[1].r);
                        hi = make_ulonglong2(s_[2].r, s_[3].r);
                    }
                    ulonglong2* dst = reinterpret_cast<ulonglong2*>(ws + (size_t)q * a.h + 8 * (size_t)v);
                    dst[0] = lo;
                    dst[1] = hi;
                }
            }
        }
    }
    if (ACC_TMEM) {
        // every consumer thread is done with its columns before warp 0,
        // which allocated them, gives them back
        tmem_fence_before_sync();
        asm volatile("bar.sync %0, %1;" ::"r"(1 + kMaxGroups), "r"(G * C) : "memory");
        if (tid < 32) {
            tmem_fence_after_sync();
            tmem_dealloc(tail->tmem_base, a.tmem_cols);
        }
    }
}

// General backward: any h.  One CTA per row (grid stride over at most one CTA
// per SM); the reduced dn row lives in shared memory, the CTA's
// parameter-gradient partials in its own workspace slice (zeroed first, owned
// column by column by one thread each).
template <typename T, bool LN>
__global__ void __launch_bounds__(1024) k_bwd_general(const __grid_constant__ BwdArgs a)
{
    grid_dep_launch();
    grid_dep_wait();
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
            const float xv = a.res_f32 ? IO<float>::load1(a.x, lbase + j)
                                       : IO<T>::load1(a.x, lbase + j);
            const float xh = LN ? (xv - mean) * rstd : xv * rstd;
            const float gg = d * IO<T>::load1(a.gamma, j);
            sg += gg;
            sgx += gg * xh;
            ws[j] += d * xh;
            if (a.want_dbeta) ws[h + j] += d;
        }
        const float mg = block_sum(sg, red) * a.inv_h;
        const float mgx = block_sum(sgx, red) * a.inv_h;
        for (int j = threadIdx.x; j < h; j += blockDim.x) {
            const float d = dns[j];
            const float xv = a.res_f32 ? IO<float>::load1(a.x, lbase + j)
                                       : IO<T>::load1(a.x, lbase + j);
            const float xh = LN ? (xv - mean) * rstd : xv * rstd;
            const float gg = d * IO<T>::load1(a.gamma, j);
            const float dx = LN ? rstd * (gg - mg - xh * mgx) : rstd * (gg - xh * mgx);
            float dr = dx;
            if (a.res_f32) {
                if (a.drnext) dr += IO<float>::load1(a.drnext, lbase + j);
                IO<float>::store1(a.dres, lbase + j, dr);
            } else {
                if (a.drnext) dr += IO<T>::load1(a.drnext, lbase + j);
                IO<T>::store1(a.dres, lbase + j, dr);
            }
            uint32_t keep = 1u;
            if (a.mask) keep = (a.mask[(size_t)i_row * a.mask_row_bytes + (j >> 3)] >> (j & 7)) & 1u;
            const float dz = keep ? dr * a.scale : 0.f;
            for (int q = 0; q < a.n_dY; ++q) IO<T>::store1(a.dY[q], base + j, dz);
            if (a.want_dbias) ws[2 * h + j] += dz;
        }
        __syncthreads();   // dns is rewritten by the next row
    }
}

// dgamma / dbeta / dbias: fixed-order sum of the nparts workspace slices
// ([nparts][3][h] fp32).  A block covers 32 consecutive columns of one
// quantity with kColreduceWarps warps: lane = column; warp w sums slices w,
// w + W, w + 2W, ... in ascending order, loading up to 16 of them at once so
// that their latencies overlap; then warp 0 adds the W warp totals in warp
// order.  Deterministic for a given slice count.
// (static: one copy per translation unit that launches it)
constexpr int kColreduceWarps = 16;

static __global__ void __launch_bounds__(kColreduceWarps * 32)
    k_colreduce(const float* __restrict__ ws, int nparts, int h, float* dgamma, float* dbeta,
                float* dbias)
{
    constexpr int W = kColreduceWarps;
    constexpr int kBatch = 16;
    __shared__ float part[W][33];
    const int tiles = (h + 31) / 32;
    const int q = blockIdx.x / tiles;
    const int lane = threadIdx.x & 31;
    const int j = (blockIdx.x - q * tiles) * 32 + lane;
    const int w = threadIdx.x >> 5;
    float* out = q == 0 ? dgamma : (q == 1 ? dbeta : dbias);
    grid_dep_launch();
    if (!out) return;   // uniform over the block
    grid_dep_wait();    // the backward's slices are complete and visible
    float s = 0.f;
    if (j < h) {
        const float* p = ws + (size_t)q * h + j;
        const size_t stride = (size_t)3 * h;
        for (int k0 = w; k0 < nparts; k0 += kBatch * W) {
            float v[kBatch];
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                const int k = k0 + u * W;
                v[u] = k < nparts ? __ldcg(p + (size_t)k * stride) : 0.f;
            }
#pragma unroll
            for (int u = 0; u < kBatch; ++u)
                if (k0 + u * W < nparts) s += v[u];
        }
    }
    part[w][lane] = s;
    __syncthreads();
    if (w == 0 && j < h) {
        float t = 0.f;
#pragma unroll
        for (int i = 0; i < W; ++i) t += part[i][lane];
        out[j] = t;
    }
}

}  // namespace spk
