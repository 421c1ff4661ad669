// kla_forward.cuh -- single-pass chunked scan of the KLA filter (sm_100a).
//
// Work decomposition.  Every channel (b, h, n) runs an independent scalar
// filter over T tokens (the review's diagonal model: "every feature channel
// runs an independent scalar Kalman filter").  A CTA owns one TILE: CW
// consecutive channels of one batch row times L consecutive tokens (one
// "chunk").  Thread (c, r) of the CTA owns channel c and the r-th run of S =
// L / R tokens of the chunk.
//
//   1. load     the tile's a, p, phi, b into shared memory (TMA bulk-tensor
//               boxes when the layout allows it, plain coalesced loads
//               otherwise);
//   2. reduce   each thread folds its S tokens into a 3x3 homogeneous
//               aggregate (see Agg in kla_device.cuh);
//   3. carry    the first row of threads composes the R aggregates into the
//               chunk aggregate.  Every D-th chunk is a checkpoint: it
//               publishes the state leaving it; every other chunk publishes
//               its aggregate.  The state entering chunk c is the aggregates
//               of chunks c-1 ... j+1 applied, in that fixed order, to the
//               state leaving the last checkpoint j < c.  The serial chain is
//               one hop per D chunks, and the result does not depend on
//               timing (bitwise reproducible);
//   4. filter   each thread enters its run with the state given by the carry
//               and the aggregates of the runs before it, then runs the plain
//               per-token recursion over its S tokens (exact up to fp32
//               rounding, nothing approximated) and writes lambda, eta, mu,
//               var into shared memory;
//   5. store    the tile's outputs go back with TMA bulk-tensor stores.
//
// Every input and output byte crosses HBM once; the carries add at most 28
// bytes per channel per chunk (written once, read from L2).  Chunks are taken in ticket order from a global
// counter, so a CTA only ever waits on CTAs that started before it, and
// every wait is bounded (a timeout writes NaN and records an error).
#pragma once

#include "kla_device.cuh"

namespace kla {

struct FwdMaps {
    CUtensorMap in[4];   // a, p, phi, b       : dims {HN, T, B}, box {CW, L, 1}
    CUtensorMap out[4];  // lambda, eta, mu, var (fp32), same geometry
};

struct FwdParams {
    const void *in[4];             // a, p, phi, b (used by the plain-load path)
    const float *lam0, *eta0;      // [B, H, N] prior
    float *out[4];                 // lambda, eta, mu, var ; mu / var may be null
    int64_t T, HN;
    int64_t tiles_per_chunk;       // B * nct
    int nct;                       // channel tiles per batch row
    int nchunks;                   // chunks per sequence
    unsigned *ticket;              // global ticket counter (zeroed per call)
    unsigned *flags;               // [tiles][CW / 32] : 0 empty, 1 aggregate, 2 carried state
    int64_t ckpt;                  // checkpoint interval D in chunks (1 <= D <= 32)
    float *agg_ws;                 // [tiles][7][CW]
    float *incl_ws;                // [tiles][2][CW] (checkpoint chunks only)
    uint64_t wait_ns;              // bound of every wait
    int64_t stall_chunk;           // test hook: chunk whose look-back waits on never_set (-1: off)
};

constexpr int align_up(int x, int a) { return (x + a - 1) / a * a; }

template <typename Tin, int L, int CW, int R>
struct FwdTile {
    static_assert(CW % 32 == 0, "channel tile must be whole warps");
    static_assert(L % R == 0, "rows must split the chunk evenly");
    static constexpr int THREADS = CW * R;
    static constexpr int S = L / R;          // tokens per thread
    static constexpr int NW = CW / 32;       // look-back warps (one flag each)
    static constexpr bool SEPARATE_OUT = sizeof(Tin) != sizeof(float);
    static constexpr int IN_BYTES = 4 * L * CW * (int)sizeof(Tin);
    static constexpr int OUT_OFF = SEPARATE_OUT ? align_up(IN_BYTES, 128) : 0;
    static constexpr int OUT_BYTES = 4 * L * CW * 4;
    static constexpr int AGG_OFF = align_up(SEPARATE_OUT ? OUT_OFF + OUT_BYTES : IN_BYTES, 128);
    static constexpr int AGG_BYTES = R * 7 * CW * 4;
    static constexpr int CARRY_OFF = AGG_OFF + AGG_BYTES;
    static constexpr int CARRY_BYTES = 2 * CW * 4;
    static constexpr int BAR_OFF = align_up(CARRY_OFF + CARRY_BYTES, 128);
    static constexpr int SMEM = BAR_OFF + 128;
};

__device__ __forceinline__ void agg_store_smem(float *base, int stride, const Agg &g) {
    base[0 * stride] = g.m11; base[1 * stride] = g.m12; base[2 * stride] = g.m21;
    base[3 * stride] = g.m22; base[4 * stride] = g.g1; base[5 * stride] = g.g2;
    base[6 * stride] = g.A;
}

__device__ __forceinline__ Agg agg_load_smem(const float *base, int stride) {
    Agg g;
    g.m11 = base[0 * stride]; g.m12 = base[1 * stride]; g.m21 = base[2 * stride];
    g.m22 = base[3 * stride]; g.g1 = base[4 * stride]; g.g2 = base[5 * stride];
    g.A = base[6 * stride];
    return g;
}

__device__ __forceinline__ Agg agg_load_l2(const float *base, int stride) {
    Agg g;
    g.m11 = __ldcg(base + 0 * stride); g.m12 = __ldcg(base + 1 * stride);
    g.m21 = __ldcg(base + 2 * stride); g.m22 = __ldcg(base + 3 * stride);
    g.g1 = __ldcg(base + 4 * stride); g.g2 = __ldcg(base + 5 * stride);
    g.A = __ldcg(base + 6 * stride);
    return g;
}

#ifndef KLA_MIN_BLOCKS
#define KLA_MIN_BLOCKS 3
#endif

template <typename Tin, int L, int CW, int R, bool TMA>
__global__ void __launch_bounds__(CW * R, KLA_MIN_BLOCKS)
kla_forward_kernel(const FwdParams prm, const __grid_constant__ FwdMaps maps) {
    using Cfg = FwdTile<Tin, L, CW, R>;
    constexpr int S = Cfg::S;
    constexpr int LC = L * CW;
    extern __shared__ __align__(128) unsigned char smem[];
    Tin *s_in = reinterpret_cast<Tin *>(smem);                               // [4][L][CW]
    float *s_out = reinterpret_cast<float *>(smem + Cfg::OUT_OFF);            // [4][L][CW]
    float *s_agg = reinterpret_cast<float *>(smem + Cfg::AGG_OFF);            // [R][7][CW]
    float *s_carry = reinterpret_cast<float *>(smem + Cfg::CARRY_OFF);        // [2][CW]
    uint64_t *s_bar = reinterpret_cast<uint64_t *>(smem + Cfg::BAR_OFF);
    unsigned *s_ticket = reinterpret_cast<unsigned *>(smem + Cfg::BAR_OFF + 8);

    const int tid = threadIdx.x;
    const int c = tid % CW;
    const int r = tid / CW;

    // ---- 1. ticket and load ------------------------------------------------
    grid_dependency_wait();  // the workspace clear before this kernel is done
    if (tid == 0) {
        const unsigned ticket = atomicAdd(prm.ticket, 1u);
        *s_ticket = ticket;
        if constexpr (TMA) {
            const int64_t tile = ticket;
            const int64_t chunk = tile / prm.tiles_per_chunk;
            const int64_t rem = tile - chunk * prm.tiles_per_chunk;
            const int bb = (int)(rem / prm.nct);
            const int ct = (int)(rem - (int64_t)bb * prm.nct);
            mbar_init(s_bar, 1);
            fence_mbar_init();
            mbar_arrive_expect_tx(s_bar, (unsigned)Cfg::IN_BYTES);
#pragma unroll
            for (int k = 0; k < 4; ++k)
                tma_load_3d(s_in + k * LC, &maps.in[k], ct * CW, (int)(chunk * L), bb, s_bar);
        }
    }
    __syncthreads();
    const int64_t tile = *s_ticket;
    const int64_t chunk = tile / prm.tiles_per_chunk;
    const int64_t rem = tile - chunk * prm.tiles_per_chunk;
    const int64_t bb = rem / prm.nct;
    const int64_t ct = rem - bb * prm.nct;
    const int64_t t0 = chunk * L;
    const int64_t c0 = ct * CW;
    const int t_valid = (int)(prm.T - t0 < (int64_t)L ? prm.T - t0 : (int64_t)L);

    bool load_failed = false;
    if constexpr (TMA) {
        const bool ok = mbar_wait_bounded(s_bar, 0, prm.wait_ns);
        load_failed = __syncthreads_or(!ok) != 0;
        if (load_failed) {
            if (tid == 0) atomicOr(&g_error_word, DEV_ERR_TIMEOUT);
            (void)mbar_wait_bounded(s_bar, 0, prm.wait_ns);  // let the copy land before exit
        }
    } else {
        const int c_valid = (int)(prm.HN - c0 < (int64_t)CW ? prm.HN - c0 : (int64_t)CW);
        for (int i = tid; i < LC; i += Cfg::THREADS) {
            const int t = i / CW, cc = i - (i / CW) * CW;
            const bool ok = t < t_valid && cc < c_valid;
            const int64_t g = ((bb * prm.T + t0 + t) * prm.HN) + c0 + cc;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const Tin *src = static_cast<const Tin *>(prm.in[k]);
                s_in[k * LC + i] = ok ? src[g] : Tin(0.f);
            }
        }
        __syncthreads();
    }

    // ---- 2. per-thread aggregate of S tokens -------------------------------
    {
        Agg g = agg_identity();
#pragma unroll
        for (int s = 0; s < S; ++s) {
            const int t = r * S + s;
            if (t < t_valid) {
                const int i = t * CW + c;
                agg_push_token(g, to_f32(s_in[i]), to_f32(s_in[LC + i]),
                               to_f32(s_in[2 * LC + i]), to_f32(s_in[3 * LC + i]));
                if (s & 1) agg_renorm(g);
            }
        }
        agg_renorm(g);
        agg_store_smem(s_agg + r * 7 * CW + c, CW, g);
    }
    __syncthreads();

    // ---- 3. chunk carry (first row of threads) -----------------------------
    if (r == 0) {
        const int lane = tid & 31;
        const int w = tid >> 5;
        const int64_t ch = c0 + c;
        const bool valid = ch < prm.HN;
        const bool publish = chunk + 1 < prm.nchunks;  // the last chunk has no reader
        Agg tot = agg_load_smem(s_agg + c, CW);
#pragma unroll
        for (int rr = 1; rr < R; ++rr) {
            tot = agg_compose(agg_load_smem(s_agg + rr * 7 * CW + c, CW), tot);
            agg_renorm(tot);
        }
        unsigned *my_flag = prm.flags + tile * Cfg::NW + w;
        const int64_t D = prm.ckpt;
        const bool is_ckpt = (chunk % D) == 0;
        float lam_in, eta_in;
        if (load_failed) {
            lam_in = __int_as_float(0x7fc00000);
            eta_in = lam_in;
        } else if (chunk == 0) {
            lam_in = valid ? prm.lam0[bb * prm.HN + ch] : 1.f;
            eta_in = valid ? prm.eta0[bb * prm.HN + ch] : 0.f;
        } else {
            if (publish && !is_ckpt) {  // aggregate for the chunks up to the next checkpoint
                agg_store_smem(prm.agg_ws + tile * 7 * CW + c, CW, tot);
                __threadfence();
                __syncwarp();
                if (lane == 0) st_release_gpu(my_flag, 1u);
            }
            // Carry = (aggregates of chunks chunk-1 ... j+1) applied to the
            // carried state of the checkpoint chunk j, in that fixed order.
            const int64_t j = ((chunk - 1) / D) * D;
            const int nd = (int)(chunk - j);  // chunks to read, <= D <= 32
            const unsigned *f = lane < nd ? prm.flags + (tile - (int64_t)(lane + 1) * prm.tiles_per_chunk) * Cfg::NW + w
                                          : nullptr;
            if (chunk == prm.stall_chunk) f = lane == 0 ? &g_never_set_word : nullptr;
            if (!warp_wait_flags(f, prm.wait_ns)) {  // ran out of time: poison this chunk
                lam_in = __int_as_float(0x7fc00000);
                eta_in = lam_in;
                if (lane == 0) atomicOr(&g_error_word, DEV_ERR_TIMEOUT);
            } else {
                Agg acc = agg_identity();
                for (int i = 0; i + 1 < nd; ++i) {
                    const int64_t jt = tile - (int64_t)(i + 1) * prm.tiles_per_chunk;
                    const Agg g = agg_load_l2(prm.agg_ws + jt * 7 * CW + c, CW);
                    acc = i == 0 ? g : agg_compose(acc, g);
                    agg_renorm(acc);
                }
                const int64_t jt = tile - (int64_t)nd * prm.tiles_per_chunk;
                lam_in = __ldcg(prm.incl_ws + jt * 2 * CW + c);
                eta_in = __ldcg(prm.incl_ws + jt * 2 * CW + CW + c);
                if (nd > 1) agg_apply(acc, lam_in, eta_in);
            }
        }
        if (publish && is_ckpt) {  // carried state out of a checkpoint chunk
            float li = lam_in, ei = eta_in;
            agg_apply(tot, li, ei);
            prm.incl_ws[tile * 2 * CW + c] = li;
            prm.incl_ws[tile * 2 * CW + CW + c] = ei;
            __threadfence();
            __syncwarp();
            if (lane == 0) st_release_gpu(my_flag, 2u);
        }
        s_carry[c] = lam_in;
        s_carry[CW + c] = eta_in;
    }
    __syncthreads();
    if (load_failed) return;  // outputs of this tile stay unwritten; successors see NaN

    // ---- 4. per-token filter over this thread's run ------------------------
    {
        float lam = s_carry[c];
        float eta = s_carry[CW + c];
        if (r > 0) {
            Agg e = agg_load_smem(s_agg + c, CW);
            for (int rr = 1; rr < r; ++rr) {
                e = agg_compose(agg_load_smem(s_agg + rr * 7 * CW + c, CW), e);
                agg_renorm(e);
            }
            agg_apply(e, lam, eta);
        }
#pragma unroll
        for (int s = 0; s < S; ++s) {
            const int t = r * S + s;
            if (t < t_valid) {
                const int i = t * CW + c;
                const float a = to_f32(s_in[i]);
                const float p = to_f32(s_in[LC + i]);
                const float phi = to_f32(s_in[2 * LC + i]);
                const float b = to_f32(s_in[3 * LC + i]);
                const TokenOut o = filter_token(lam, eta, a, p, phi, b);
                s_out[i] = o.lam;
                s_out[LC + i] = o.eta;
                s_out[2 * LC + i] = o.mu;
                s_out[3 * LC + i] = o.var;
            }
        }
    }

    // ---- 5. store -----------------------------------------------------------
    if constexpr (TMA) {
        fence_proxy_async_smem();
        __syncthreads();
        if (tid == 0) {
#pragma unroll
            for (int k = 0; k < 4; ++k)
                if (prm.out[k] != nullptr)
                    tma_store_3d(&maps.out[k], s_out + k * LC, (int)c0, (int)t0, (int)bb);
            bulk_commit_group();
            bulk_wait_group_read_all();
        }
    } else {
        __syncthreads();
        const int c_valid = (int)(prm.HN - c0 < (int64_t)CW ? prm.HN - c0 : (int64_t)CW);
        for (int i = tid; i < LC; i += Cfg::THREADS) {
            const int t = i / CW, cc = i - (i / CW) * CW;
            if (t < t_valid && cc < c_valid) {
                const int64_t g = ((bb * prm.T + t0 + t) * prm.HN) + c0 + cc;
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    if (prm.out[k] != nullptr) prm.out[k][g] = s_out[k * LC + i];
            }
        }
    }
}

// Zero the ticket counter and the ready flags of a workspace.
// Zeroes a workspace's counters and flags.  The scan kernel that follows it
// may be launched as its programmatic dependent: it becomes resident and sets
// up while this kernel runs, and waits for it before touching the workspace.
__global__ void kla_clear_kernel(uint4 *p, int64_t n16) {
    allow_dependent_launch();
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n16;
         i += (int64_t)gridDim.x * blockDim.x)
        p[i] = make_uint4(0u, 0u, 0u, 0u);
}

// Test hook: a bounded wait on a flag nothing sets.
__global__ void kla_unset_flag_wait_kernel(uint64_t wait_ns) {
    const bool ok = warp_wait_flags(threadIdx.x == 0 ? &g_never_set_word : nullptr, wait_ns);
    if (!ok && threadIdx.x == 0) atomicOr(&g_error_word, DEV_ERR_TIMEOUT);
}

}  // namespace kla
