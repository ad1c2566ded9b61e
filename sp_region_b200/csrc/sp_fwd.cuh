// Forward of the SP boundary on sm_100a.
//
// Per token row n (rank r = n / (N/t) owns it), as the Megatron SP pages
// describe the exit of a tensor-parallel region ("Sequence Parallelism
// math", sections "The collective substitution" and "The move"; "SP:
// Partition Activations Alongside TP", sections "Normalize and add residuals
// by token" and "Connect SP and TP across a layer"):
//   reduce-scatter of the t partial sums -> + bias -> inverted dropout ->
//   + residual (stored in the residual stream's dtype) -> LayerNorm / RMSNorm -> written to
//   every gathered replica (the all-gather).
//
// k_fwd_tma: persistent, one CTA per SM.  The last warp is a producer: one
// lane streams whole row segments (partial k of row n, then the residual row)
// from HBM into a ring of shared-memory stages with cp.async.bulk, each stage
// completing on its own "full" mbarrier.  The other warps are consumers: each
// thread owns V vectors of 8 features of the row, accumulates the t partials
// from shared memory in fp32 registers, applies bias / dropout / residual,
// and runs the two-pass mean / variance with fixed-order reductions.  The
// ring keeps the next rows' segments in flight while a row is normalised.
#pragma once

#include "sp_device.cuh"

namespace spk {

constexpr int kMaxT = 64;
constexpr int kFwdMaxConsumers = 512;

struct FwdArgs {
    const void* parts[kMaxT];
    void* gathered[kMaxT];
    const void* bias;
    const void* residual;
    const void* gamma;
    const void* beta;
    void* residual_out;
    uint8_t* mask;          // bytes: [rows][mask_row_bytes]
    float* mean;
    float* rstd;
    long long rows;         // token rows of this call (local index i)
    long long row0;         // global index of local row 0: n = row0 + i
    int h;
    int hv;                 // h / 8 (fast kernel)
    int t;
    int n_gathered;
    int stages;
    uint32_t seg_bytes;     // h * elem bytes
    uint32_t res_seg_bytes; // h * residual stream elem bytes (residual, residual_out)
    int res_f32;            // residual stream in fp32 (I/O dtype bf16)
    uint32_t stage_stride;  // largest segment rounded up to 128
    int mask_row_bytes;     // 4 * ceil(h / 32)
    uint32_t param_off;     // shared-memory offsets (fast kernel): parameters,
    uint32_t param_stride;  //   one slot of param_stride bytes each,
    uint32_t tail_off;      //   then the barriers / scratch
    float eps;
    float inv_h;            // 1 / h, rounded to fp32
    float scale;            // 1 / (1 - p)
    uint32_t thr;           // floor(p * 2^32)
    uint32_t seed_lo, seed_hi, off_lo, off_hi;
    uint32_t keys[10][2];   // Philox key (k0, k1) of each round, from the seed
    int dropout;            // p > 0
};

// Shared-memory tail after the ring: barriers, per-group reduction scratch,
// abort flag.
constexpr int kMaxGroups = 6;
// Reduction scratch: two buffers per group, used alternately by row parity
// (or by the two reductions of one LayerNorm row), so a warp that runs ahead
// to the next row never overwrites totals a slower warp is still reading.
struct RingTail {
    uint64_t full[64];
    uint64_t empty[64];
    uint64_t turn[2][kMaxGroups];   // backward: shared-accumulator turns
    uint64_t xbar[2][kMaxGroups][2];   // cluster split: the peer's sums landed
    float2 xslot[2][kMaxGroups][2];    // cluster split: the peer's sums
    float red[2][kMaxGroups][64];
    int abort;
    uint32_t tmem_base;   // backward, tensor-memory accumulators: allocated base
};

// Position in a sub-ring of Sg stages starting at stage `base`: the i-th
// segment a consumer group receives lives in stage base + i % Sg and completes
// phase i / Sg of that stage's barriers.  Each group consumes its own sub-ring
// strictly in order, so a group never waits on a stage more than one phase
// ahead of it (mbarrier parity waits only tell adjacent phases apart).
struct RingPos {
    uint32_t base, stage, phase;
    __device__ __forceinline__ RingPos(uint32_t base_, uint32_t i, uint32_t Sg)
        : base(base_), stage(i % Sg), phase((i / Sg) & 1u) {}
    __device__ __forceinline__ uint32_t abs() const { return base + stage; }
    __device__ __forceinline__ void next(uint32_t Sg)
    {
        if (++stage == Sg) {
            stage = 0;
            phase ^= 1u;
        }
    }
};

// The producer lane: streams every segment of this CTA's rows, in row order.
// Row j of the CTA belongs to consumer group j % G and goes to that group's
// sub-ring (stages [g*Sg, (g+1)*Sg)).  nsrc sources per row; src(k, i) gives
// the address of source k's segment for local row i.  Sources k >= k_split
// (the residual stream's tensors) move seg2 bytes from slice_off2 instead.
template <int G, typename SrcFn>
__device__ __forceinline__ void ring_produce(unsigned char* smem, RingTail* tail,
                                             volatile int* abort, long long rows,
                                             int nsrc, uint32_t seg_bytes,
                                             uint32_t stage_stride, int S, SrcFn src,
                                             int k_split, uint32_t seg2,
                                             long long first = -1, long long stride = 0,
                                             uint32_t slice_off = 0, uint32_t slice_off2 = 0)
{
    // rows first, first + stride, ... (default: this CTA's blockIdx rows);
    // each copy moves seg_bytes starting slice_off bytes into the segment
    if (first < 0) {
        first = blockIdx.x;
        stride = gridDim.x;
    }
    const uint64_t pol = policy_evict_first();
    const int Sg = S / G;
    uint32_t stage[G], phase[G];
    long long issued[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        stage[g] = 0;
        phase[g] = 1;   // a fresh "empty" barrier counts as released
        issued[g] = 0;
    }
    bool ok = true;
    for (long long jj = 0; ok; ++jj) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const long long i = first + (jj * G + g) * stride;
            if (!ok || i >= rows) {
                ok = false;
                break;
            }
            for (int k = 0; k < nsrc; ++k) {
                const uint32_t st = (uint32_t)(g * Sg) + stage[g];
                if (!mbar_wait(smem_addr(&tail->empty[st]), phase[g], abort, ERR_WAIT_EMPTY)) {
                    ok = false;
                    break;
                }
                const bool second = k >= k_split;
                const uint32_t nb = second ? seg2 : seg_bytes;
                const void* p = static_cast<const unsigned char*>(src(k, i)) +
                                (second ? slice_off2 : slice_off);
                const uint32_t bar = smem_addr(&tail->full[st]);
                mbar_arrive_expect_tx(bar, nb);
                bulk_load(smem_addr(smem + (size_t)st * stage_stride), p, nb, bar, pol);
                ++issued[g];
                if (++stage[g] == (uint32_t)Sg) {
                    stage[g] = 0;
                    phase[g] ^= 1;
                }
            }
        }
    }
    if (*abort) {
        // wind down: let every copy already issued land before the CTA exits
        // (its shared memory must not be released under a copy)
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const long long first = issued[g] > Sg ? issued[g] - Sg : 0;
            for (long long i = first; i < issued[g]; ++i) {
                volatile int no_abort = 0;
                if (!mbar_wait(smem_addr(&tail->full[g * Sg + i % Sg]), (uint32_t)((i / Sg) & 1),
                               &no_abort, ERR_DRAIN))
                    break;
            }
        }
    }
}

__device__ __forceinline__ void init_ring(RingTail* tail, int S, int warps_per_group)
{
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(smem_addr(&tail->full[s]), 1);
            mbar_init(smem_addr(&tail->empty[s]), warps_per_group);
        }
        for (int g = 0; g < kMaxGroups; ++g) {
            mbar_init(smem_addr(&tail->turn[0][g]), warps_per_group);
            mbar_init(smem_addr(&tail->turn[1][g]), warps_per_group);
            for (int q = 0; q < 4; ++q) mbar_init(smem_addr(&tail->xbar[q >> 1][g][q & 1]), 1);
        }
        tail->abort = 0;
        mbar_init_fence();
    }
    __syncthreads();
}

// Fast-kernel instantiations are k_*_tma<T, V, G, MAXT, ...>: G consumer
// groups of C threads (C <= (MAXT - 32) / G), each thread owning V vectors of
// 8 features of a row, plus one producer warp; MAXT bounds the block size and
// so sets the register budget.
// CS = 1: one CTA per token row.  CS = 2: each token row is split across the
// two CTAs of a thread-block cluster (CTA rank r owns vectors
// [r*hv/2, (r+1)*hv/2) of every row); the row's partial sums for mean and
// variance are exchanged through distributed shared memory and added in rank
// order, so both CTAs normalise with the same bits.
// EXACT: the threads' vectors tile the row slice exactly (C * V == hv / CS),
// so the per-vector bounds checks compile away.
template <typename T, int V, int G, int MAXT, bool LN, int CS = 1, bool EXACT = false>
__global__ void __launch_bounds__(MAXT, 1) k_fwd_tma(const __grid_constant__ FwdArgs a)
{
    using Vec = typename IO<T>::Vec;
    extern __shared__ __align__(128) unsigned char smem[];
    RingTail* tail = reinterpret_cast<RingTail*>(smem + a.tail_off);
    volatile int* abort = &tail->abort;
    unsigned char* sg = smem + a.param_off;   // gamma, beta, bias copies (this slice)
    unsigned char* sb = sg + a.param_stride;
    unsigned char* sc = sb + a.param_stride;

    const int C = (blockDim.x - 32) / G;      // consumer threads per group
    const int tid = threadIdx.x;
    const int S = a.stages;                   // G sub-rings of S / G stages
    const int nsrc = a.t + 1;                 // t partials, then the residual
    const uint32_t rank = CS > 1 ? cluster_rank() : 0u;
    const long long cid = CS > 1 ? (long long)cluster_index() : (long long)blockIdx.x;
    const long long ncl = CS > 1 ? (long long)cluster_count() : (long long)gridDim.x;
    const int hvc = a.hv / CS;                // vectors of this CTA's slice
    const int vg0 = (int)rank * hvc;          // first global vector of the slice
    const uint32_t slice_bytes = a.seg_bytes / CS;
    const uint32_t res_slice_bytes = a.res_seg_bytes / CS;
    // the fp32 residual stream is compiled out of the plans with the most
    // live registers per thread (the host does not pick them for it)
    constexpr bool kResF32 = !(V >= 4 && MAXT <= 544);
    const bool res_f32 = kResF32 && a.res_f32;

    init_ring(tail, S, C / 32);
    if (CS > 1) cluster_sync_all();   // the peer's barriers exist before any remote arrive
    grid_dep_launch();
    grid_dep_wait();                  // the previous kernel's outputs are visible

    if (tid >= G * C) {
        if (tid == G * C)
            ring_produce<G>(smem, tail, abort, a.rows, nsrc, slice_bytes, a.stage_stride, S,
                            [&](int k, long long i) -> const void* {
                                // partial sums are indexed by global row, the
                                // residual shard by local row
                                return k < a.t ? static_cast<const unsigned char*>(a.parts[k]) +
                                                     (size_t)(a.row0 + i) * a.seg_bytes
                                               : static_cast<const unsigned char*>(a.residual) +
                                                     (size_t)i * a.res_seg_bytes;
                            },
                            a.t, res_slice_bytes, cid, ncl, rank * slice_bytes,
                            rank * res_slice_bytes);
    } else {
        // consumers: group g handles every G-th row of this CTA (cluster);
        // thread c of a group owns slice vectors v = c + i*C (8 features each)
        const int g = tid / C;
        const int c = tid - g * C;
        const int lane = tid & 31;
        const int bar_id = 1 + g;
        if (g == 0) {
#pragma unroll
            for (int i = 0; i < V; ++i) {
                const int v = c + i * C;
                if (EXACT || v < hvc) {
                    store_vec<T>(sg, v, load_vec<T>(a.gamma, vg0 + v));
                    if (a.beta) store_vec<T>(sb, v, load_vec<T>(a.beta, vg0 + v));
                    if (a.bias) store_vec<T>(sc, v, load_vec<T>(a.bias, vg0 + v));
                }
            }
        }
        // every group reads the copies group 0 wrote
        asm volatile("bar.sync %0, %1;" ::"r"(1 + kMaxGroups), "r"(G * C) : "memory");

        int parity = 0, rcount = 0;
        // sum over the row: this group's warps, then (CS = 2) the peer CTA
        auto row_sum = [&](float x, float* red, int idx) {
            x = warp_sum(x);
            if (lane == 0) red[c >> 5] = x;
            asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "r"(C) : "memory");
            const float local = warps_total(red, C >> 5);
            if (CS == 1) return local;
            const uint32_t slot = smem_addr(&tail->xslot[parity][g][idx]);
            const uint32_t xb = smem_addr(&tail->xbar[parity][g][idx]);
            if (c == 0) {
                st_peer_f32x2(peer_addr(slot, rank ^ 1u), local, 0.f);
                mbar_arrive_peer(peer_addr(xb, rank ^ 1u));
            }
            mbar_wait_cluster(xb, (uint32_t)((rcount >> 1) & 1), abort, ERR_WAIT_PEER);
            const float other = tail->xslot[parity][g][idx].x;
            return rank == 0 ? local + other : other + local;
        };

        const uint32_t Sg = (uint32_t)(S / G);
        RingPos pos((uint32_t)g * Sg, 0, Sg);
        auto release = [&]() {
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_addr(&tail->empty[pos.abs()]));
            pos.next(Sg);
        };
        const F2 scale2 = f2(a.scale);
        for (long long j = g;; j += G, parity ^= 1, ++rcount) {
            const long long i_row = cid + j * ncl;              // local row
            if (i_row >= a.rows) break;
            const long long n = a.row0 + i_row;                  // global row

            // reduce-scatter: sum of the t partial rows, k ascending, from +0;
            // fp32 pairs throughout (features 2p, 2p+1 of a vector in pair p).
            // With no partial sums, bias, dropout or stored sum (the entry into
            // a TP region) the row is the input itself, already in the I/O dtype.
            F2 acc[V][4];
            const bool direct = a.t == 0 && !a.bias && !a.dropout && !a.residual_out;
            if (!direct) {
#pragma unroll
                for (int i = 0; i < V; ++i)
#pragma unroll
                    for (int p = 0; p < 4; ++p) acc[i][p] = f2(0.f);
            }
            for (int k = 0; k < a.t; ++k) {
                mbar_wait(smem_addr(&tail->full[pos.abs()]), pos.phase, abort, ERR_WAIT_FULL);
                const unsigned char* buf = smem + (size_t)pos.abs() * a.stage_stride;
#pragma unroll
                for (int i = 0; i < V; ++i) {
                    const int v = c + i * C;
                    if (EXACT || v < hvc) {
                        F2 f[4];
                        IO<T>::unpack2(load_vec<T>(buf, v), f);
#pragma unroll
                        for (int p = 0; p < 4; ++p) acc[i][p] = add2(acc[i][p], f[p]);
                    }
                }
                release();
            }

            // bias once, then inverted dropout with the packed keep bits
            uint8_t* mrow = a.mask ? a.mask + (size_t)i_row * a.mask_row_bytes : nullptr;
#pragma unroll
            for (int i = 0; i < V; ++i) {
                const int v = c + i * C;
                if (EXACT || v < hvc) {
                    if (a.bias) {
                        F2 f[4];
                        IO<T>::unpack2(load_vec<T>(sc, v), f);
#pragma unroll
                        for (int p = 0; p < 4; ++p) acc[i][p] = add2(acc[i][p], f[p]);
                    }
                    uint32_t kb = 0xFFu;
                    if (a.dropout) {
                        kb = keep_bits8((uint32_t)(vg0 + v), (uint32_t)n, a.off_lo, a.off_hi,
                                        a.keys, a.thr);
#pragma unroll
                        for (int p = 0; p < 4; ++p)
                            acc[i][p] = keep2(mul2(acc[i][p], scale2), (kb >> (2 * p)) & 1u,
                                              (kb >> (2 * p + 1)) & 1u);
                    }
                    if (mrow) mrow[vg0 + v] = (uint8_t)kb;
                }
            }
            if (mrow && c == 0 && rank == 0)
                for (int pbyte = a.hv; pbyte < a.mask_row_bytes; ++pbyte) mrow[pbyte] = 0;

            // residual add; the sum is stored in the residual stream's dtype
            // and the norm reads the stored (rounded) value
            mbar_wait(smem_addr(&tail->full[pos.abs()]), pos.phase, abort, ERR_WAIT_FULL);
            if (direct) {
                const unsigned char* buf = smem + (size_t)pos.abs() * a.stage_stride;
#pragma unroll
                for (int i = 0; i < V; ++i)
                    if (EXACT || c + i * C < hvc) {
                        if (res_f32)
                            IO<float>::unpack2(load_vec<float>(buf, c + i * C), acc[i]);
                        else
                            IO<T>::unpack2(load_vec<T>(buf, c + i * C), acc[i]);
                    }
            } else if (res_f32) {
                // fp32 residual stream: the sum is exact in its storage format
                const unsigned char* buf = smem + (size_t)pos.abs() * a.stage_stride;
                unsigned char* rout =
                    static_cast<unsigned char*>(a.residual_out) + (size_t)i_row * a.res_seg_bytes;
#pragma unroll
                for (int i = 0; i < V; ++i) {
                    const int v = c + i * C;
                    if (EXACT || v < hvc) {
                        F2 f[4];
                        IO<float>::unpack2(load_vec<float>(buf, v), f);
#pragma unroll
                        for (int p = 0; p < 4; ++p) acc[i][p] = add2(f[p], acc[i][p]);
                        if (a.residual_out)
                            store_vec<float>(rout, vg0 + v, IO<float>::pack2v(acc[i]));
                    }
                }
            } else {
                const unsigned char* buf = smem + (size_t)pos.abs() * a.stage_stride;
                unsigned char* rout =
                    static_cast<unsigned char*>(a.residual_out) + (size_t)i_row * a.res_seg_bytes;
#pragma unroll
                for (int i = 0; i < V; ++i) {
                    const int v = c + i * C;
                    if (EXACT || v < hvc) {
                        F2 f[4];
                        IO<T>::unpack2(load_vec<T>(buf, v), f);
#pragma unroll
                        for (int p = 0; p < 4; ++p) f[p] = add2(f[p], acc[i][p]);
                        const Vec r = IO<T>::pack2v(f);
                        if (a.residual_out) store_vec<T>(rout, vg0 + v, r);
                        IO<T>::unpack2(r, acc[i]);
                    }
                }
            }
            release();

            // per-token norm, two passes over the row held in registers (the
            // two reductions use the group's two scratch buffers)
            float mean = 0.f, rstd;
            if (LN) {
                F2 s2 = f2(0.f);
#pragma unroll
                for (int i = 0; i < V; ++i)
                    if (EXACT || c + i * C < hvc)
#pragma unroll
                        for (int p = 0; p < 4; ++p) s2 = add2(s2, acc[i][p]);
                mean = row_sum(hsum(s2), tail->red[0][g], 0) * a.inv_h;
                const F2 mean2 = f2(mean);
                F2 q2 = f2(0.f);
#pragma unroll
                for (int i = 0; i < V; ++i)
                    if (EXACT || c + i * C < hvc)
#pragma unroll
                        for (int p = 0; p < 4; ++p) {
                            const F2 d = sub2(acc[i][p], mean2);
                            q2 = fma2(d, d, q2);
                        }
                const float var = row_sum(hsum(q2), tail->red[1][g], 1) * a.inv_h;
                rstd = rsqrtf(var + a.eps);
            } else {
                F2 q2 = f2(0.f);
#pragma unroll
                for (int i = 0; i < V; ++i)
                    if (EXACT || c + i * C < hvc)
#pragma unroll
                        for (int p = 0; p < 4; ++p) q2 = fma2(acc[i][p], acc[i][p], q2);
                const float ms = row_sum(hsum(q2), tail->red[parity][g], 0) * a.inv_h;
                rstd = rsqrtf(ms + a.eps);
            }

            const F2 mean2 = f2(mean), rstd2 = f2(rstd);
#pragma unroll
            for (int i = 0; i < V; ++i) {
                const int v = c + i * C;
                if (EXACT || v < hvc) {
                    F2 gm[4], o[4];
                    IO<T>::unpack2(load_vec<T>(sg, v), gm);
                    if (LN && a.beta) {
                        F2 b[4];
                        IO<T>::unpack2(load_vec<T>(sb, v), b);
#pragma unroll
                        for (int p = 0; p < 4; ++p)
                            o[p] = fma2(mul2(sub2(acc[i][p], mean2), rstd2), gm[p], b[p]);
                    } else {
#pragma unroll
                        for (int p = 0; p < 4; ++p)
                            o[p] = mul2(mul2(LN ? sub2(acc[i][p], mean2) : acc[i][p], rstd2),
                                        gm[p]);
                    }
                    const Vec ov = IO<T>::pack2v(o);
                    for (int q = 0; q < a.n_gathered; ++q)
                        store_vec<T>(static_cast<unsigned char*>(a.gathered[q]) +
                                         (size_t)n * a.seg_bytes,
                                     vg0 + v, ov);
                }
            }
            if (c == 0 && rank == 0) {
                if (LN && a.mean) a.mean[i_row] = mean;
                if (a.rstd) a.rstd[i_row] = rstd;
            }
        }
    }
    if (CS > 1) {
        __syncwarp();
        cluster_sync_all();   // no CTA leaves while its peer may still write here
    }
}

// General forward: any h, element-aligned pointers.  One CTA per row (grid
// stride); the row's residual sum is kept in shared memory as fp32.
template <typename T, bool LN>
__global__ void __launch_bounds__(256) k_fwd_general(const __grid_constant__ FwdArgs a)
{
    grid_dep_launch();
    grid_dep_wait();
    extern __shared__ __align__(128) unsigned char smem[];
    float* xs = reinterpret_cast<float*>(smem);
    uint32_t* mw = reinterpret_cast<uint32_t*>(xs + a.h);
    const int W = a.mask_row_bytes / 4;
    __shared__ float red[32];
    const int h = a.h;

    for (long long i_row = blockIdx.x; i_row < a.rows; i_row += gridDim.x) {
        const long long n = a.row0 + i_row;      // global row
        for (int w = threadIdx.x; w < W; w += blockDim.x) mw[w] = 0u;
        __syncthreads();
        const long long base = n * (long long)h;         // partials, gathered
        const long long lbase = i_row * (long long)h;    // this call's shard
        for (int j = threadIdx.x; j < h; j += blockDim.x) {
            float y = 0.f;
            for (int k = 0; k < a.t; ++k) y = (k == 0) ? IO<T>::load1(a.parts[k], base + j)
                                                       : y + IO<T>::load1(a.parts[k], base + j);
            if (a.bias) y += IO<T>::load1(a.bias, j);
            uint32_t keep = 1u;
            if (a.dropout) {
                keep = keep_bit((uint32_t)j, (uint32_t)n, a.off_lo, a.off_hi, a.seed_lo,
                                a.seed_hi, a.thr);
                y = keep ? y * a.scale : 0.f;
            }
            if (keep) atomicOr(&mw[j >> 5], 1u << (j & 31));
            float r;
            if (a.res_f32) {   // fp32 residual stream: the sum is its own rounding
                r = IO<float>::load1(a.residual, lbase + j) + y;
                if (a.residual_out) IO<float>::store1(a.residual_out, lbase + j, r);
            } else {
                r = IO<T>::round1(IO<T>::load1(a.residual, lbase + j) + y);
                if (a.residual_out) IO<T>::store1(a.residual_out, lbase + j, r);
            }
            xs[j] = r;
        }
        __syncthreads();
        if (a.mask) {
            uint32_t* mrow =
                reinterpret_cast<uint32_t*>(a.mask + (size_t)i_row * a.mask_row_bytes);
            for (int w = threadIdx.x; w < W; w += blockDim.x) mrow[w] = mw[w];
        }
        float mean = 0.f, rstd;
        if (LN) {
            float s = 0.f;
            for (int j = threadIdx.x; j < h; j += blockDim.x) s += xs[j];
            mean = block_sum(s, red) * a.inv_h;
            float q = 0.f;
            for (int j = threadIdx.x; j < h; j += blockDim.x) {
                const float d = xs[j] - mean;
                q += d * d;
            }
            rstd = rsqrtf(block_sum(q, red) * a.inv_h + a.eps);
        } else {
            float q = 0.f;
            for (int j = threadIdx.x; j < h; j += blockDim.x) q += xs[j] * xs[j];
            rstd = rsqrtf(block_sum(q, red) * a.inv_h + a.eps);
        }
        for (int j = threadIdx.x; j < h; j += blockDim.x) {
            const float g = IO<T>::load1(a.gamma, j);
            float o;
            if (LN) {
                const float b = a.beta ? IO<T>::load1(a.beta, j) : 0.f;
                o = (xs[j] - mean) * rstd * g + b;
            } else {
                o = xs[j] * rstd * g;
            }
            for (int q = 0; q < a.n_gathered; ++q) IO<T>::store1(a.gathered[q], base + j, o);
        }
        if (threadIdx.x == 0) {
            if (LN && a.mean) a.mean[i_row] = mean;
            if (a.rstd) a.rstd[i_row] = rstd;
        }
        __syncthreads();   // xs / mw are reused by the next row
    }
}

}  // namespace spk
