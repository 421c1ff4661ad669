// kla_forward_stream.cuh -- channel-owning streaming scan of the KLA filter
// (sm_100a).
//
// Every channel (b, h, n) is an independent scalar filter (the review's
// diagonal model).  Here one CTA owns a tile of 32 consecutive channels of a
// batch row for the WHOLE sequence, so the carry between chunks never leaves
// the SM:
//
//   producer warp   streams the tile's chunks (L tokens x 32 channels of a, p,
//                   phi, b) into a ring of NS shared-memory stages with TMA
//                   bulk-tensor loads (mbarriers full[s] / empty[s]);
//   W chunk warps   warp w takes chunks w, w + W, w + 2W, ...  Lane = channel.
//                   A warp copies its chunk into registers and releases the
//                   stage at once (so nearly the whole ring is in flight),
//                   then (1) folds the L tokens into the chunk's 3x3
//                   homogeneous aggregate (no dependency on any other chunk),
//                   (2) waits for the state leaving the previous chunk (a
//                   shared-memory slot written by the previous warp, mbarrier
//                   carry[slot]), applies its aggregate to it and hands the
//                   result to the next warp -- the only serial link, a few
//                   hundred cycles per chunk -- and (3) runs the plain
//                   per-token recursion from the entering state.  Outputs go
//                   through a per-warp, double-buffered shared-memory box of
//                   G tokens x 32 channels x 4 outputs and leave with TMA
//                   bulk-tensor stores issued by the warp's lane 0 (which
//                   also clip ragged edges), so the chunk warps do no global
//                   address arithmetic.
//
// A lane owns VEC consecutive channels (CW = 32 VEC per tile): with VEC = 2
// (bf16 inputs: 64-channel tiles, 16-token chunks, the same registers per
// thread) every lane runs two independent recursion chains side by side, and
// one 32-bit shared load brings a token's two bf16 values of an input; its
// output box is the whole chunk (G = L), single-buffered: the next chunk's
// first pass runs while the bulk stores read it out.
//
// Within a tile no global flags, fences or look-back: the W warps overlap
// their passes while the producer keeps HBM busy.  Chunk aggregates are formed
// and applied exactly as in kla_forward_kernel (one thread's run = the whole
// chunk here).  A CTA with more than one work unit processes them one after
// another, taking them by ticket when they are long enough for a faster SM
// to gain by taking more.  When tiles do not divide evenly over the SMs, each
// tile's sequence is cut into a few runs taken by ticket, run-major, so that a run
// after the first finds the state published by the previous run (one bounded
// global wait per run; deadlock-free because a run only waits on a run with a
// smaller ticket).  Every wait is bounded by the wait limit (a timeout
// records KLA_ERR_TIMEOUT and the CTA carries on, so nothing can hang).
#pragma once

#include "kla_forward.cuh"

namespace kla {

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(smem_u32(bar)) : "memory");
}

// Wait until at most N committed bulk store groups are still reading shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_group_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" :: "n"(N) : "memory");
}

// Wait until every committed bulk store group has completed (writes done).
__device__ __forceinline__ void bulk_wait_group_all() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

struct StreamParams {
    const float *lam0, *eta0;      // [B, H, N] prior
    // lambda, eta, mu, var [B, T, H, N] (mu / var may be null); the kernels
    // store through the tensor maps.  The field stays: the long fp32 workload
    // measured 4-5% faster, on three boxes, with the parameter block laid
    // out with it than without.
    float *out[4];
    int64_t T, HN;
    int64_t ntiles;                // B * ceil(HN / CW)
    int nct;                       // tiles of CW channels per batch row
    int nchunks;                   // ceil(T / L)
    int write_mu, write_var;       // outputs 2 / 3 requested
    uint64_t wait_ns;
    // Work units.  parts == 1: unit = tile, taken by ticket or (ticket null)
    // round-robin, CTA c taking tiles c, c + grid, ...  parts > 1: each
    // tile's chunks are cut into `parts` consecutive runs of decreasing length
    // (guided_start); unit u = part * ntiles + tile is taken by ticket (part
    // major), and a run after the first enters with the state the previous
    // run of the same tile published in part_state (flag part_flags).
    // chunks_per_part (equal runs) is no longer read by these kernels; the
    // field stays because this kernel's speed follows its register
    // allocation, which follows the parameter block's layout.
    int parts, chunks_per_part;
    int64_t nunits;                // ntiles * parts
    unsigned *ticket;              // unit counter (zeroed per call); null: round-robin units
    unsigned *part_flags;          // [ntiles][parts - 1], zeroed per call
    float *part_state;             // [ntiles][parts - 1][2][CW]
    int64_t stall_chunk;           // test hook: this chunk's carry waits on a flag nothing sets (-1: off)
};

// What a producer tells its chunk warps about the chunk in a stage: the work
// unit's tile coordinates and run bounds, computed once per unit (used by
// the convolutional-form kernel).
struct StreamChunk {
    int64_t tile;                  // bb * nct + ct
    int chunk;                     // -1: no more work
    int part, bb, ct;
    int first, last;               // chunks of the run
};

// Output buffers per chunk warp: 2 (double-buffered output groups) or 1 (a
// group waits for the bulk stores of the previous one to have read it).
#ifndef KLA_STREAM_NBUF
#define KLA_STREAM_NBUF 2
#endif
#ifndef KLA_STREAM2_NBUF
#define KLA_STREAM2_NBUF 1
#endif

template <typename Tin, int L, int W, int NS, int G, int VEC = 1>
struct StreamTile {
    // Chunk j sits in stage j % NS and is handled by warp j % W.  With
    // NS >= W a warp waiting for stage s is always waiting for the stage's
    // next phase (its previous chunk is no older than the stage's previous
    // chunk, through the carry chain), so the parity of the mbarrier wait is
    // unambiguous.  With NS < W a warp could pass a wait one phase early.
    static_assert(NS >= W, "the stage ring must be at least as deep as the number of chunk warps");
    static_assert(L % G == 0, "output groups must tile the chunk");
    static_assert(VEC == 1 || VEC == 2, "one or two channels per lane");
    static constexpr int CW = 32 * VEC;                              // channels per tile
    static constexpr int THREADS = 32 * (W + 1);                     // producer + W chunk warps
    static constexpr int STAGE_BYTES = 4 * L * CW * (int)sizeof(Tin);
    static constexpr int OUTBOX_BYTES = G * CW * 4;                 // one output, one group
    static constexpr int OUTBUF_BYTES = 4 * OUTBOX_BYTES;           // four outputs
    static constexpr int NBUF = VEC == 1 ? KLA_STREAM_NBUF : KLA_STREAM2_NBUF;
    static_assert(NBUF == 1 || NBUF == 2, "one or two output buffers per warp");
    static constexpr int OUT_OFF = NS * STAGE_BYTES;                 // [W][NBUF][4][G][CW] fp32
    static constexpr int CARRY_OFF = OUT_OFF + W * NBUF * OUTBUF_BYTES; // [W][2][CW] fp32
    static constexpr int META_OFF = CARRY_OFF + W * 2 * CW * 4;      // per stage: unit (int64), chunk (int64)
    static constexpr int BAR_OFF = align_up(META_OFF + NS * 16, 128); // full, empty, carry
    static constexpr int SMEM = align_up(BAR_OFF + (2 * NS + W) * 8, 128);
};

__device__ __forceinline__ void mbar_wait_or_flag(uint64_t *bar, unsigned parity, uint64_t limit_ns) {
    if (!mbar_wait_bounded(bar, parity, limit_ns)) {
        atomicOr(&g_error_word, DEV_ERR_TIMEOUT);
        (void)mbar_wait_bounded(bar, parity, limit_ns);
    }
}

// The VEC consecutive values of a lane in one row of a stage (CW = 32 VEC
// values of one input and token), widened to fp32.
template <typename Tin, int VEC> struct RowVec;
template <typename Tin> struct RowVec<Tin, 1> {
    static __device__ __forceinline__ void load(const Tin *row, int lane, float (&v)[1]) { v[0] = to_f32(row[lane]); }
};
template <> struct RowVec<float, 2> {
    static __device__ __forceinline__ void load(const float *row, int lane, float (&v)[2]) {
        const float2 x = reinterpret_cast<const float2 *>(row)[lane];
        v[0] = x.x; v[1] = x.y;
    }
};
template <> struct RowVec<__nv_bfloat16, 2> {
    static __device__ __forceinline__ void load(const __nv_bfloat16 *row, int lane, float (&v)[2]) {
        const unsigned u = reinterpret_cast<const unsigned *>(row)[lane];  // channel 2 lane in the low half
        v[0] = __uint_as_float(u << 16);
        v[1] = __uint_as_float(u & 0xffff0000u);
    }
};

// VEC consecutive floats into shared memory.
__device__ __forceinline__ void sts_vec(float *dst, const float (&v)[1]) { *dst = v[0]; }
__device__ __forceinline__ void sts_vec(float *dst, const float (&v)[2]) {
    *reinterpret_cast<float2 *>(dst) = make_float2(v[0], v[1]);
}

// Start chunk of run r of P over n chunks, run lengths in the ratio
// P : P-1 : ... : 1: the tickets taken last are the shortest runs, so the
// CTAs finish closer together (1-5% faster than equal runs on LM-layer and
// run-split fp32 shapes).  n >= P (P + 1) / 2 keeps every run non-empty (the
// host cuts runs only for n >= 8 P).
__device__ __forceinline__ int guided_start(int r, int P, int n) {
    const int k = P - r;
    return n - (int)(((int64_t)n * (k * (k + 1) / 2)) / (P * (P + 1) / 2));
}

template <typename Tin, int L, int W, int NS, int G>
__global__ void __launch_bounds__(32 * (W + 1), 1)
kla_forward_stream_kernel(const StreamParams prm, const __grid_constant__ FwdMaps maps) {
    using Cfg = StreamTile<Tin, L, W, NS, G>;
    constexpr int LC = L * 32;
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + Cfg::BAR_OFF);
    uint64_t *empty = full + NS;
    uint64_t *carry_bar = empty + NS;
    float *slots = reinterpret_cast<float *>(smem + Cfg::CARRY_OFF);
    int64_t *meta_unit = reinterpret_cast<int64_t *>(smem + Cfg::META_OFF);  // -1: no more work
    int64_t *meta_chunk = meta_unit + NS;

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int s = 0; s < W; ++s) mbar_init(&carry_bar[s], 1);
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane != 0) return;
        int next = 0, round = 0;  // next stage to fill; completed passes over the ring
        auto claim = [&]() -> int {
            const int s = next;
            if (round > 0) mbar_wait_or_flag(&empty[s], (unsigned)((round - 1) & 1), prm.wait_ns);
            if (++next == NS) {
                next = 0;
                ++round;
            }
            return s;
        };
        auto load = [&](int64_t unit, int chunk, int bb, int ct) {
            const int s = claim();
            meta_unit[s] = unit;
            meta_chunk[s] = chunk;
            Tin *stage = reinterpret_cast<Tin *>(smem + s * Cfg::STAGE_BYTES);
            mbar_arrive_expect_tx(&full[s], (unsigned)Cfg::STAGE_BYTES);
#pragma unroll
            for (int q = 0; q < 4; ++q)
                tma_load_3d(stage + q * LC, &maps.in[q], ct * 32, chunk * L, bb, &full[s]);
        };
        // one unit: the tile's run u / ntiles, in time order (its tile
        // coordinates computed once per unit, not per chunk)
        auto unit_chunks = [&](int64_t u) {
            const int64_t tile = u % prm.ntiles;
            const int part = (int)(u / prm.ntiles);
            const int bb = (int)(tile / prm.nct);
            const int ct = (int)(tile - (int64_t)bb * prm.nct);
            const int first = guided_start(part, prm.parts, prm.nchunks);
            const int last = guided_start(part + 1, prm.parts, prm.nchunks) - 1;
#pragma unroll 1
            for (int c = first; c <= last; ++c) load(u, c, bb, ct);
        };
        if (prm.ticket == nullptr) {
#pragma unroll 1
            for (int64_t u = blockIdx.x; u < prm.nunits; u += gridDim.x) unit_chunks(u);
        } else {
#pragma unroll 1
            for (;;) {
                const int64_t u = (int64_t)atomicAdd(prm.ticket, 1u);
                if (u >= prm.nunits) break;
                unit_chunks(u);
            }
        }
        // one end marker for each chunk warp
#pragma unroll 1
        for (int k = 0; k < W; ++k) {
            const int s = claim();
            meta_unit[s] = -1;
            mbar_arrive(&full[s]);
        }
        return;
    }

    // ------------------------------------------------------------ chunk warps
    const int w = warp - 1;
    float *outbuf0 = reinterpret_cast<float *>(smem + Cfg::OUT_OFF + w * Cfg::NBUF * Cfg::OUTBUF_BYTES);
    int group_seq = 0;  // output groups this warp has committed (bulk groups are per thread: lane 0)
#pragma unroll 1
    for (int64_t j = w;; j += W) {
        const int s = (int)(j % NS);
        mbar_wait_or_flag(&full[s], (unsigned)((j / NS) & 1), prm.wait_ns);
        const int64_t unit = meta_unit[s];
        if (unit < 0) break;
        const int64_t chunk = meta_chunk[s];
        const int64_t tile = unit % prm.ntiles;
        const int64_t part = unit / prm.ntiles;
        const int64_t bb = tile / prm.nct;
        const int64_t ct = tile - bb * prm.nct;
        const int64_t t0 = chunk * L;
        const int t_valid = (int)(prm.T - t0 < (int64_t)L ? prm.T - t0 : (int64_t)L);
        const int64_t ch = ct * 32 + lane;
        const bool cvalid = ch < prm.HN;
        const Tin *stage = reinterpret_cast<const Tin *>(smem + s * Cfg::STAGE_BYTES);
        const int64_t first = guided_start((int)part, prm.parts, prm.nchunks);  // first chunk of this unit
        const int64_t last = guided_start((int)part + 1, prm.parts, prm.nchunks) - 1;

        // State entering chunk j -- from the previous chunk's warp, from the
        // prior at a tile's first chunk, or from the previous run of the tile
        // at a later run's first chunk -- and the state leaving it, handed to
        // the next warp (and published for the next run at a run's end).
        auto chunk_carry = [&](const Agg &g, float &lam, float &eta) {
            if (j > 0) {
                const int ps = (int)((j - 1) % W);
                mbar_wait_or_flag(&carry_bar[ps], (unsigned)(((j - 1) / W) & 1), prm.wait_ns);
                lam = slots[ps * 64 + lane];
                eta = slots[ps * 64 + 32 + lane];
            }
            if (chunk == prm.stall_chunk &&
                !warp_wait_flags(lane == 0 ? &g_never_set_word : nullptr, prm.wait_ns)) {
                lam = __int_as_float(0x7fc00000);  // ran out of time: poison what follows
                eta = lam;
                if (lane == 0) atomicOr(&g_error_word, DEV_ERR_TIMEOUT);
            } else if (chunk == 0) {
                lam = cvalid ? prm.lam0[bb * prm.HN + ch] : 1.f;
                eta = cvalid ? prm.eta0[bb * prm.HN + ch] : 0.f;
            } else if (chunk == first) {
                const int64_t slot = tile * (prm.parts - 1) + (part - 1);
                if (warp_wait_flags(lane == 0 ? prm.part_flags + slot : nullptr, prm.wait_ns)) {
                    lam = __ldcg(prm.part_state + slot * 64 + lane);
                    eta = __ldcg(prm.part_state + slot * 64 + 32 + lane);
                } else {
                    lam = __int_as_float(0x7fc00000);
                    eta = lam;
                    if (lane == 0) atomicOr(&g_error_word, DEV_ERR_TIMEOUT);
                }
            }
            float lo = lam, eo = eta;
            agg_apply(g, lo, eo);
            const int ms = (int)(j % W);
            slots[ms * 64 + lane] = lo;
            slots[ms * 64 + 32 + lane] = eo;
            __syncwarp();
            if (lane == 0) mbar_arrive(&carry_bar[ms]);
            if (chunk == last && part + 1 < prm.parts) {
                const int64_t slot = tile * (prm.parts - 1) + part;
                prm.part_state[slot * 64 + lane] = lo;
                prm.part_state[slot * 64 + 32 + lane] = eo;
                __threadfence();
                __syncwarp();
                if (lane == 0) st_release_gpu(prm.part_flags + slot, 1u);
            }
        };

        // Output group q of this chunk (tokens q*G .. q*G+G-1): claim a free
        // half of the warp's double buffer (the store that last read it must
        // be done), fill it, and send it out with TMA bulk-tensor stores.
        auto group_begin = [&]() -> float * {
            float *buf = outbuf0 + (group_seq & (Cfg::NBUF - 1)) * (Cfg::OUTBUF_BYTES / 4);
            if (group_seq >= Cfg::NBUF) {
                if (lane == 0) bulk_wait_group_read<Cfg::NBUF - 1>();
                __syncwarp();
            }
            return buf;
        };
        auto group_end = [&](float *buf, int q) {
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                const int ty = (int)(t0 + q * G);
                const int x = (int)(ct * 32);
                tma_store_3d(&maps.out[0], buf, x, ty, (int)bb);
                tma_store_3d(&maps.out[1], buf + G * 32, x, ty, (int)bb);
                if (prm.write_mu) tma_store_3d(&maps.out[2], buf + 2 * G * 32, x, ty, (int)bb);
                if (prm.write_var) tma_store_3d(&maps.out[3], buf + 3 * G * 32, x, ty, (int)bb);
                bulk_commit_group();
            }
            ++group_seq;
        };
        auto put = [&](float *buf, int u, const TokenOut &o) {
            buf[u * 32 + lane] = o.lam;
            buf[G * 32 + u * 32 + lane] = o.eta;
            buf[2 * G * 32 + u * 32 + lane] = o.mu;
            buf[3 * G * 32 + u * 32 + lane] = o.var;
        };

        if (t_valid == L) {
            // Full chunk: read it from shared memory once into registers,
            // release the stage to the producer right away, then run both
            // passes from registers.
            float xa[L], xp[L], xf[L], xb[L];
#pragma unroll
            for (int t = 0; t < L; ++t) {
                const int i = t * 32 + lane;
                xa[t] = to_f32(stage[i]);
                xp[t] = to_f32(stage[LC + i]);
                xf[t] = to_f32(stage[2 * LC + i]);
                xb[t] = to_f32(stage[3 * LC + i]);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            // (1) the chunk's aggregate (renormalised every second token)
            Agg g = agg_identity();
#pragma unroll
            for (int t = 0; t < L; ++t) {
                agg_push_token(g, xa[t], xp[t], xf[t], xb[t]);
                if (renorm_after(t)) agg_renorm(g);
            }
            agg_renorm(g);
            // (2) carry
            float lam, eta;
            chunk_carry(g, lam, eta);
            // (3) per-token recursion from the entering state
#pragma unroll
            for (int q = 0; q < L / G; ++q) {
                float *buf = group_begin();
#pragma unroll
                for (int u = 0; u < G; ++u) {
                    const int t = q * G + u;
                    put(buf, u, filter_token(lam, eta, xa[t], xp[t], xf[t], xb[t]));
                }
                group_end(buf, q);
            }
        } else {
            // Ragged last chunk: straight from shared memory, released at the
            // end; rows past T are clipped by the TMA stores.
            Agg g = agg_identity();
#pragma unroll 2
            for (int t = 0; t < t_valid; ++t) {
                const int i = t * 32 + lane;
                agg_push_token(g, to_f32(stage[i]), to_f32(stage[LC + i]), to_f32(stage[2 * LC + i]),
                               to_f32(stage[3 * LC + i]));
                if (renorm_after(t)) agg_renorm(g);
            }
            agg_renorm(g);
            float lam, eta;
            chunk_carry(g, lam, eta);
            const int ngroups = (t_valid + G - 1) / G;
#pragma unroll 1
            for (int q = 0; q < ngroups; ++q) {
                float *buf = group_begin();
#pragma unroll
                for (int u = 0; u < G; ++u) {
                    const int t = q * G + u;
                    if (t < t_valid) {
                        const int i = t * 32 + lane;
                        put(buf, u, filter_token(lam, eta, to_f32(stage[i]), to_f32(stage[LC + i]),
                                                 to_f32(stage[2 * LC + i]), to_f32(stage[3 * LC + i])));
                    }
                }
                group_end(buf, q);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }
    }
    // every bulk store of this warp must be complete before the CTA exits
    if (lane == 0) bulk_wait_group_all();
    __syncwarp();
}

// The same scan with VEC channels per lane (used with VEC = 2 for bf16
// inputs: 64-channel tiles, two independent recursion chains per lane).  The
// one-channel kernel above is kept separate: compiled from this template with
// VEC = 1 it measured 5% slower on the long fp32 workload.

template <typename Tin, int L, int W, int NS, int G, int VEC>
__global__ void __launch_bounds__(32 * (W + 1), 1)
kla_forward_stream_vec_kernel(const StreamParams prm, const __grid_constant__ FwdMaps maps) {
    using Cfg = StreamTile<Tin, L, W, NS, G, VEC>;
    constexpr int CW = Cfg::CW;
    constexpr int LC = L * CW;
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + Cfg::BAR_OFF);
    uint64_t *empty = full + NS;
    uint64_t *carry_bar = empty + NS;
    float *slots = reinterpret_cast<float *>(smem + Cfg::CARRY_OFF);
    int64_t *meta_unit = reinterpret_cast<int64_t *>(smem + Cfg::META_OFF);  // -1: no more work
    int64_t *meta_chunk = meta_unit + NS;

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int s = 0; s < W; ++s) mbar_init(&carry_bar[s], 1);
        fence_mbar_init();
    }
    __syncthreads();
    grid_dependency_wait();  // a workspace clear launched before this kernel is done

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane != 0) return;
        int next = 0, round = 0;  // next stage to fill; completed passes over the ring
        auto claim = [&]() -> int {
            const int s = next;
            if (round > 0) mbar_wait_or_flag(&empty[s], (unsigned)((round - 1) & 1), prm.wait_ns);
            if (++next == NS) {
                next = 0;
                ++round;
            }
            return s;
        };
        auto load = [&](int64_t unit, int chunk, int bb, int ct) {
            const int s = claim();
            meta_unit[s] = unit;
            meta_chunk[s] = chunk;
            Tin *stage = reinterpret_cast<Tin *>(smem + s * Cfg::STAGE_BYTES);
            mbar_arrive_expect_tx(&full[s], (unsigned)Cfg::STAGE_BYTES);
#pragma unroll
            for (int q = 0; q < 4; ++q)
                tma_load_3d(stage + q * LC, &maps.in[q], ct * CW, chunk * L, bb, &full[s]);
        };
        // one unit: the tile's run u / ntiles, in time order (its tile
        // coordinates computed once per unit, not per chunk)
        auto unit_chunks = [&](int64_t u) {
            const int64_t tile = u % prm.ntiles;
            const int part = (int)(u / prm.ntiles);
            const int bb = (int)(tile / prm.nct);
            const int ct = (int)(tile - (int64_t)bb * prm.nct);
            const int first = guided_start(part, prm.parts, prm.nchunks);
            const int last = guided_start(part + 1, prm.parts, prm.nchunks) - 1;
#pragma unroll 1
            for (int c = first; c <= last; ++c) load(u, c, bb, ct);
        };
        if (prm.ticket == nullptr) {
#pragma unroll 1
            for (int64_t u = blockIdx.x; u < prm.nunits; u += gridDim.x) unit_chunks(u);
        } else {
#pragma unroll 1
            for (;;) {
                const int64_t u = (int64_t)atomicAdd(prm.ticket, 1u);
                if (u >= prm.nunits) break;
                unit_chunks(u);
            }
        }
        // one end marker for each chunk warp
#pragma unroll 1
        for (int k = 0; k < W; ++k) {
            const int s = claim();
            meta_unit[s] = -1;
            mbar_arrive(&full[s]);
        }
        return;
    }

    // ------------------------------------------------------------ chunk warps
    const int w = warp - 1;
    float *outbuf0 = reinterpret_cast<float *>(smem + Cfg::OUT_OFF + w * Cfg::NBUF * Cfg::OUTBUF_BYTES);
    int group_seq = 0;  // output groups this warp has committed (bulk groups are per thread: lane 0)
    const int lc = lane * VEC;  // this lane's first channel within a tile
#pragma unroll 1
    for (int64_t j = w;; j += W) {
        const int s = (int)(j % NS);
        mbar_wait_or_flag(&full[s], (unsigned)((j / NS) & 1), prm.wait_ns);
        const int64_t unit = meta_unit[s];
        if (unit < 0) break;
        const int64_t chunk = meta_chunk[s];
        const int64_t tile = unit % prm.ntiles;
        const int64_t part = unit / prm.ntiles;
        const int64_t bb = tile / prm.nct;
        const int64_t ct = tile - bb * prm.nct;
        const int64_t t0 = chunk * L;
        const int t_valid = (int)(prm.T - t0 < (int64_t)L ? prm.T - t0 : (int64_t)L);
        const int64_t ch = ct * CW + lc;  // the lane's channels ch .. ch + VEC - 1
        const Tin *stage = reinterpret_cast<const Tin *>(smem + s * Cfg::STAGE_BYTES);
        const int64_t first = guided_start((int)part, prm.parts, prm.nchunks);  // first chunk of this unit
        const int64_t last = guided_start((int)part + 1, prm.parts, prm.nchunks) - 1;

        // State entering chunk j -- from the previous chunk's warp, from the
        // prior at a tile's first chunk, or from the previous run of the tile
        // at a later run's first chunk -- and the state leaving it, handed to
        // the next warp (and published for the next run at a run's end).
        auto chunk_carry = [&](const Agg (&g)[VEC], float (&lam)[VEC], float (&eta)[VEC]) {
            if (j > 0) {
                const int ps = (int)((j - 1) % W);
                mbar_wait_or_flag(&carry_bar[ps], (unsigned)(((j - 1) / W) & 1), prm.wait_ns);
#pragma unroll
                for (int v = 0; v < VEC; ++v) {
                    lam[v] = slots[ps * 2 * CW + lc + v];
                    eta[v] = slots[ps * 2 * CW + CW + lc + v];
                }
            }
            if (chunk == prm.stall_chunk &&
                !warp_wait_flags(lane == 0 ? &g_never_set_word : nullptr, prm.wait_ns)) {
#pragma unroll
                for (int v = 0; v < VEC; ++v) {
                    lam[v] = __int_as_float(0x7fc00000);  // ran out of time: poison what follows
                    eta[v] = lam[v];
                }
                if (lane == 0) atomicOr(&g_error_word, DEV_ERR_TIMEOUT);
            } else if (chunk == 0) {
#pragma unroll
                for (int v = 0; v < VEC; ++v) {
                    const bool cvalid = ch + v < prm.HN;
                    lam[v] = cvalid ? prm.lam0[bb * prm.HN + ch + v] : 1.f;
                    eta[v] = cvalid ? prm.eta0[bb * prm.HN + ch + v] : 0.f;
                }
            } else if (chunk == first) {
                const int64_t slot = tile * (prm.parts - 1) + (part - 1);
                if (warp_wait_flags(lane == 0 ? prm.part_flags + slot : nullptr, prm.wait_ns)) {
#pragma unroll
                    for (int v = 0; v < VEC; ++v) {
                        lam[v] = __ldcg(prm.part_state + slot * 2 * CW + lc + v);
                        eta[v] = __ldcg(prm.part_state + slot * 2 * CW + CW + lc + v);
                    }
                } else {
#pragma unroll
                    for (int v = 0; v < VEC; ++v) {
                        lam[v] = __int_as_float(0x7fc00000);
                        eta[v] = lam[v];
                    }
                    if (lane == 0) atomicOr(&g_error_word, DEV_ERR_TIMEOUT);
                }
            }
            float lo[VEC], eo[VEC];
#pragma unroll
            for (int v = 0; v < VEC; ++v) {
                lo[v] = lam[v];
                eo[v] = eta[v];
                agg_apply(g[v], lo[v], eo[v]);
            }
            const int ms = (int)(j % W);
            sts_vec(slots + ms * 2 * CW + lc, lo);
            sts_vec(slots + ms * 2 * CW + CW + lc, eo);
            __syncwarp();
            if (lane == 0) mbar_arrive(&carry_bar[ms]);
            if (chunk == last && part + 1 < prm.parts) {
                const int64_t slot = tile * (prm.parts - 1) + part;
#pragma unroll
                for (int v = 0; v < VEC; ++v) {
                    prm.part_state[slot * 2 * CW + lc + v] = lo[v];
                    prm.part_state[slot * 2 * CW + CW + lc + v] = eo[v];
                }
                __threadfence();
                __syncwarp();
                if (lane == 0) st_release_gpu(prm.part_flags + slot, 1u);
            }
        };

        // Output group q of this chunk (tokens q*G .. q*G+G-1): claim a free
        // half of the warp's double buffer (the store that last read it must
        // be done), fill it, and send it out with TMA bulk-tensor stores.
        auto group_begin = [&]() -> float * {
            float *buf = outbuf0 + (group_seq & (Cfg::NBUF - 1)) * (Cfg::OUTBUF_BYTES / 4);
            if (group_seq >= Cfg::NBUF) {
                if (lane == 0) bulk_wait_group_read<Cfg::NBUF - 1>();
                __syncwarp();
            }
            return buf;
        };
        auto group_end = [&](float *buf, int q) {
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                const int ty = (int)(t0 + q * G);
                const int x = (int)(ct * CW);
                tma_store_3d(&maps.out[0], buf, x, ty, (int)bb);
                tma_store_3d(&maps.out[1], buf + G * CW, x, ty, (int)bb);
                if (prm.write_mu) tma_store_3d(&maps.out[2], buf + 2 * G * CW, x, ty, (int)bb);
                if (prm.write_var) tma_store_3d(&maps.out[3], buf + 3 * G * CW, x, ty, (int)bb);
                bulk_commit_group();
            }
            ++group_seq;
        };
        // token u of the group: the four outputs of the lane's VEC channels
        auto run_token = [&](float *buf, int u, float (&lam)[VEC], float (&eta)[VEC], const float (&a)[VEC],
                             const float (&p)[VEC], const float (&f)[VEC], const float (&b)[VEC]) {
            float ol[VEC], oe[VEC], om[VEC], ov[VEC];
#pragma unroll
            for (int v = 0; v < VEC; ++v) {
                const TokenOut o = filter_token(lam[v], eta[v], a[v], p[v], f[v], b[v]);
                ol[v] = o.lam; oe[v] = o.eta; om[v] = o.mu; ov[v] = o.var;
            }
            sts_vec(buf + u * CW + lc, ol);
            sts_vec(buf + G * CW + u * CW + lc, oe);
            sts_vec(buf + 2 * G * CW + u * CW + lc, om);
            sts_vec(buf + 3 * G * CW + u * CW + lc, ov);
        };

        if (t_valid == L) {
            // Full chunk: read it from shared memory once into registers,
            // release the stage to the producer right away, then run both
            // passes from registers.
            float xa[L][VEC], xp[L][VEC], xf[L][VEC], xb[L][VEC];
#pragma unroll
            for (int t = 0; t < L; ++t) {
                RowVec<Tin, VEC>::load(stage + t * CW, lane, xa[t]);
                RowVec<Tin, VEC>::load(stage + LC + t * CW, lane, xp[t]);
                RowVec<Tin, VEC>::load(stage + 2 * LC + t * CW, lane, xf[t]);
                RowVec<Tin, VEC>::load(stage + 3 * LC + t * CW, lane, xb[t]);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            // (1) the chunk's aggregates (renormalised every second token)
            Agg g[VEC];
#pragma unroll
            for (int v = 0; v < VEC; ++v) g[v] = agg_identity();
#pragma unroll
            for (int t = 0; t < L; ++t) {
#pragma unroll
                for (int v = 0; v < VEC; ++v) {
                    agg_push_token(g[v], xa[t][v], xp[t][v], xf[t][v], xb[t][v]);
                    if (renorm_after(t)) agg_renorm(g[v]);
                }
            }
#pragma unroll
            for (int v = 0; v < VEC; ++v) agg_renorm(g[v]);
            // (2) carry
            float lam[VEC], eta[VEC];
            chunk_carry(g, lam, eta);
            // (3) per-token recursion from the entering state
#pragma unroll
            for (int q = 0; q < L / G; ++q) {
                float *buf = group_begin();
#pragma unroll
                for (int u = 0; u < G; ++u) {
                    const int t = q * G + u;
                    run_token(buf, u, lam, eta, xa[t], xp[t], xf[t], xb[t]);
                }
                group_end(buf, q);
            }
        } else {
            // Ragged last chunk: straight from shared memory, released at the
            // end; rows past T are clipped by the TMA stores.
            Agg g[VEC];
#pragma unroll
            for (int v = 0; v < VEC; ++v) g[v] = agg_identity();
#pragma unroll 2
            for (int t = 0; t < t_valid; ++t) {
                float a[VEC], p[VEC], f[VEC], b[VEC];
                RowVec<Tin, VEC>::load(stage + t * CW, lane, a);
                RowVec<Tin, VEC>::load(stage + LC + t * CW, lane, p);
                RowVec<Tin, VEC>::load(stage + 2 * LC + t * CW, lane, f);
                RowVec<Tin, VEC>::load(stage + 3 * LC + t * CW, lane, b);
#pragma unroll
                for (int v = 0; v < VEC; ++v) {
                    agg_push_token(g[v], a[v], p[v], f[v], b[v]);
                    if (renorm_after(t)) agg_renorm(g[v]);
                }
            }
#pragma unroll
            for (int v = 0; v < VEC; ++v) agg_renorm(g[v]);
            float lam[VEC], eta[VEC];
            chunk_carry(g, lam, eta);
            const int ngroups = (t_valid + G - 1) / G;
#pragma unroll 1
            for (int q = 0; q < ngroups; ++q) {
                float *buf = group_begin();
#pragma unroll
                for (int u = 0; u < G; ++u) {
                    const int t = q * G + u;
                    if (t < t_valid) {
                        float a[VEC], p[VEC], f[VEC], b[VEC];
                        RowVec<Tin, VEC>::load(stage + t * CW, lane, a);
                        RowVec<Tin, VEC>::load(stage + LC + t * CW, lane, p);
                        RowVec<Tin, VEC>::load(stage + 2 * LC + t * CW, lane, f);
                        RowVec<Tin, VEC>::load(stage + 3 * LC + t * CW, lane, b);
                        run_token(buf, u, lam, eta, a, p, f, b);
                    }
                }
                group_end(buf, q);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }
    }
    // every bulk store of this warp must be complete before the CTA exits
    if (lane == 0) bulk_wait_group_all();
    __syncwarp();
}

}  // namespace kla
