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
//                   then (1) folds the L tokens into the
//                   chunk's 3x3 homogeneous aggregate (no dependency on any
//                   other chunk), (2) waits for the state leaving the previous
//                   chunk (a shared-memory slot written by the previous warp,
//                   mbarrier carry[slot]), applies its aggregate to it and
//                   hands the result to the next warp -- the only serial link,
//                   a few hundred cycles per chunk -- and (3) runs the plain
//                   per-token recursion from the entering state, storing
//                   lambda, eta, mu, var straight to global memory.
//
// No global flags, fences or look-back: the W warps overlap their passes
// while the producer keeps HBM busy.  Chunk aggregates are formed and applied
// exactly as in kla_forward_kernel (one thread's run = the whole chunk here).
// A CTA with more than one tile processes them one after another.  Every
// mbarrier wait is bounded by the wait limit (a timeout records
// KLA_ERR_TIMEOUT and the CTA carries on, so nothing can hang).
#pragma once

#include "kla_forward.cuh"

namespace kla {

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(smem_u32(bar)) : "memory");
}

struct StreamParams {
    const float *lam0, *eta0;      // [B, H, N] prior
    float *out[4];                 // lambda, eta, mu, var ; mu / var may be null
    int64_t T, HN;
    int64_t ntiles;                // B * ceil(HN / 32)
    int nct;                       // 32-channel tiles per batch row
    int nchunks;                   // ceil(T / L)
    uint64_t wait_ns;
};

template <typename Tin, int L, int W, int NS>
struct StreamTile {
    // Chunk j sits in stage j % NS and is handled by warp j % W.  With
    // NS >= W a warp waiting for stage s is always waiting for the stage's
    // next phase (its previous chunk is no older than the stage's previous
    // chunk, through the carry chain), so the parity of the mbarrier wait is
    // unambiguous.  With NS < W a warp could pass a wait one phase early.
    static_assert(NS >= W, "the stage ring must be at least as deep as the number of chunk warps");
    static constexpr int CW = 32;
    static constexpr int THREADS = 32 * (W + 1);
    static constexpr int STAGE_BYTES = 4 * L * CW * (int)sizeof(Tin);
    static constexpr int CARRY_OFF = NS * STAGE_BYTES;                       // [W][2][32] fp32
    static constexpr int BAR_OFF = align_up(CARRY_OFF + W * 2 * CW * 4, 128);  // full, empty, carry
    static constexpr int SMEM = align_up(BAR_OFF + (2 * NS + W) * 8, 128);
};

__device__ __forceinline__ void mbar_wait_or_flag(uint64_t *bar, unsigned parity, uint64_t limit_ns) {
    if (!mbar_wait_bounded(bar, parity, limit_ns)) {
        atomicOr(&g_error_word, DEV_ERR_TIMEOUT);
        (void)mbar_wait_bounded(bar, parity, limit_ns);
    }
}

template <typename Tin, int L, int W, int NS>
__global__ void __launch_bounds__(32 * (W + 1), 1)
kla_forward_stream_kernel(const StreamParams prm, const __grid_constant__ FwdMaps maps) {
    using Cfg = StreamTile<Tin, L, W, NS>;
    constexpr int LC = L * 32;
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + Cfg::BAR_OFF);
    uint64_t *empty = full + NS;
    uint64_t *carry_bar = empty + NS;
    float *slots = reinterpret_cast<float *>(smem + Cfg::CARRY_OFF);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    // tiles of this CTA: blockIdx.x, blockIdx.x + gridDim.x, ...
    const int64_t my_tiles = prm.ntiles > blockIdx.x
                                 ? (prm.ntiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    const int64_t my_chunks = my_tiles * prm.nchunks;

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
#pragma unroll 1
        for (int64_t j = 0; j < my_chunks; ++j) {
            const int s = (int)(j % NS);
            if (j >= NS) mbar_wait_or_flag(&empty[s], (unsigned)((j / NS - 1) & 1), prm.wait_ns);
            const int64_t tile = blockIdx.x + (j / prm.nchunks) * gridDim.x;
            const int64_t chunk = j % prm.nchunks;
            const int bb = (int)(tile / prm.nct);
            const int ct = (int)(tile - (int64_t)bb * prm.nct);
            Tin *stage = reinterpret_cast<Tin *>(smem + s * Cfg::STAGE_BYTES);
            mbar_arrive_expect_tx(&full[s], (unsigned)Cfg::STAGE_BYTES);
#pragma unroll
            for (int q = 0; q < 4; ++q)
                tma_load_3d(stage + q * LC, &maps.in[q], ct * 32, (int)(chunk * L), bb, &full[s]);
        }
        return;
    }

    // ------------------------------------------------------------ chunk warps
    const int w = warp - 1;
#pragma unroll 1
    for (int64_t j = w; j < my_chunks; j += W) {
        const int s = (int)(j % NS);
        mbar_wait_or_flag(&full[s], (unsigned)((j / NS) & 1), prm.wait_ns);
        const int64_t tile = blockIdx.x + (j / prm.nchunks) * gridDim.x;
        const int64_t chunk = j % prm.nchunks;
        const int64_t bb = tile / prm.nct;
        const int64_t ct = tile - bb * prm.nct;
        const int64_t t0 = chunk * L;
        const int t_valid = (int)(prm.T - t0 < (int64_t)L ? prm.T - t0 : (int64_t)L);
        const int64_t ch = ct * 32 + lane;
        const bool cvalid = ch < prm.HN;
        const Tin *stage = reinterpret_cast<const Tin *>(smem + s * Cfg::STAGE_BYTES);

        // State entering chunk j (from the previous chunk's warp, or the prior
        // at a tile's first chunk); hands the state leaving it to the next warp.
        auto chunk_carry = [&](int64_t jj, int64_t ck, const Agg &g, float &lam, float &eta) {
            if (jj > 0) {
                const int ps = (int)((jj - 1) % W);
                mbar_wait_or_flag(&carry_bar[ps], (unsigned)(((jj - 1) / W) & 1), prm.wait_ns);
                lam = slots[ps * 64 + lane];
                eta = slots[ps * 64 + 32 + lane];
            }
            if (ck == 0) {
                lam = cvalid ? prm.lam0[bb * prm.HN + ch] : 1.f;
                eta = cvalid ? prm.eta0[bb * prm.HN + ch] : 0.f;
            }
            float lo = lam, eo = eta;
            agg_apply(g, lo, eo);
            const int ms = (int)(jj % W);
            slots[ms * 64 + lane] = lo;
            slots[ms * 64 + 32 + lane] = eo;
            __syncwarp();
            if (lane == 0) mbar_arrive(&carry_bar[ms]);
        };
        const int64_t gi = (bb * prm.T + t0) * prm.HN + ch;
        float *o0 = prm.out[0] + gi, *o1 = prm.out[1] + gi;
        float *o2 = prm.out[2] != nullptr ? prm.out[2] + gi : nullptr;
        float *o3 = prm.out[3] != nullptr ? prm.out[3] + gi : nullptr;
        const int64_t HN = prm.HN;
        auto emit = [&](int t, const TokenOut &o) {
            if (cvalid) {
                __stcs(o0 + t * HN, o.lam);
                __stcs(o1 + t * HN, o.eta);
                if (o2 != nullptr) __stcs(o2 + t * HN, o.mu);
                if (o3 != nullptr) __stcs(o3 + t * HN, o.var);
            }
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
                if (t & 1) agg_renorm(g);
            }
            agg_renorm(g);
            // (2) carry
            float lam, eta;
            chunk_carry(j, chunk, g, lam, eta);
            // (3) per-token recursion from the entering state
#pragma unroll
            for (int t = 0; t < L; ++t) {
                const TokenOut o = filter_token(lam, eta, xa[t], xp[t], xf[t], xb[t]);
                emit(t, o);
            }
        } else {
            // Ragged last chunk: straight from shared memory, released at the end.
            Agg g = agg_identity();
#pragma unroll 2
            for (int t = 0; t < t_valid; ++t) {
                const int i = t * 32 + lane;
                agg_push_token(g, to_f32(stage[i]), to_f32(stage[LC + i]), to_f32(stage[2 * LC + i]),
                               to_f32(stage[3 * LC + i]));
                if (t & 1) agg_renorm(g);
            }
            agg_renorm(g);
            float lam, eta;
            chunk_carry(j, chunk, g, lam, eta);
#pragma unroll 2
            for (int t = 0; t < t_valid; ++t) {
                const int i = t * 32 + lane;
                const TokenOut o = filter_token(lam, eta, to_f32(stage[i]), to_f32(stage[LC + i]),
                                                to_f32(stage[2 * LC + i]), to_f32(stage[3 * LC + i]));
                emit(t, o);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }
    }
}

}  // namespace kla
