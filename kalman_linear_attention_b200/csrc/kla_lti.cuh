// kla_lti.cuh -- the convolutional form of the KLA filter for deterministic
// time-invariant channels (sm_100a).
//
// KLA review, Theorem 3: for a deterministic linear time-invariant system the
// filter is a convolution.  With no process noise (p = 0) and a decay a that
// is constant in time, the precision map of the review's M_t = [[1, a^2 phi],
// [0, a^2]] is affine, lambda_t = a^-2 lambda_{t-1} + phi_t, and the gate is
// f = 1 / a, so (rows 0-based)
//
//   lambda_t = kappa_{t+1} lambda_0 + sum_{s<=t} kappa_{t-s} phi_s,   kappa_m = a^(-2m)
//   eta_t    = nu_{t+1}    eta_0    + sum_{s<=t} nu_{t-s}    b_s,     nu_m    = a^(-m)
//
// causal convolutions of the evidence with geometric kernels.  Blockwise, a
// convolution splits exactly into local convolutions plus the tail of
// everything before, which the geometric kernel carries as ONE number per
// sequence (kappa_{m+n} = kappa_m kappa_n).  So per chunk of L tokens:
//
//   1. local convolutions over sub-blocks of S tokens (an S x S lower-
//      triangular Toeplitz product, S(S-1)/2 multiply-adds per sub-block and
//      output, independent of everything else);
//   2. the chunk's exit with zero entry, by Horner over its sub-blocks;
//   3. the carry: exit = kappa_L entry + (2), kept in fp64 from chunk to
//      chunk, so that a constant decay, whose powers repeat the same
//      rounding in every chunk, does not drift over long sequences;
//   4. the final pass: each sub-block enters with the state leaving the
//      previous one (x_i = local_i + kappa_{i-i0+1} state), and
//      mu = eta / lambda, var = 1 / lambda are emitted.
//
// Only phi and b are read per token (a is per channel, p is zero): 8 bytes
// (fp32 inputs) or 4 (bf16) plus 16 written, against the general scan's 16
// (or 8) read + 16 written.  The kernel is the general streaming scan's
// structure with two input streams: a CTA owns 32 channels of a batch row for
// the whole sequence; a producer warp streams chunks into a ring of shared-
// memory stages with TMA; chunk warps take chunks round-robin, compute (1)
// and (2) without waiting, take the entering state from the previous chunk's
// warp (mbarrier), hand on the exit, and run (4) straight from registers to
// global memory: one coalesced 128-byte streaming store per output and token
// (measured faster here than output boxes stored with TMA).  Rows past T
// arrive as zeros (TMA fill) and are not stored.  Tiles
// that do not spread evenly over the SMs are cut into runs taken by ticket,
// as in the general streaming scan (and, as there, more tiles than SMs, each
// long enough, are taken whole by ticket); run boundaries hand on fp64
// states.  The
// producer passes each chunk's tile coordinates in the stage's metadata.
#pragma once

#include "kla_forward_stream.cuh"

namespace kla {

struct LtiParams {
    const float *a;                // [B, H, N] time-invariant decay
    const float *lam0, *eta0;      // [B, H, N] prior
    float *out[4];                 // lambda, eta, mu, var [B, T, H, N]; mu / var may be null
    int64_t T, HN;
    int64_t ntiles;                // B * ceil(HN / 32)
    int nct;                       // 32-channel tiles per batch row
    int nchunks;
    int write_mu, write_var;
    uint64_t wait_ns;
    int parts, chunks_per_part;
    int64_t nunits;
    unsigned *ticket;              // unit counter (zeroed per call); null: round-robin units
    unsigned *part_flags;          // [ntiles][parts - 1]
    double *part_state;            // [ntiles][parts - 1][2][32]
};

struct LtiMaps {
    CUtensorMap in[2];             // phi, b: {HN, T, B}, box {32, L, 1}
};

template <typename Tin, int L, int W, int NS>
struct LtiTile {
    static_assert(NS >= W, "the stage ring must be at least as deep as the number of chunk warps");
    static constexpr int THREADS = 32 * (W + 1);
    static constexpr int STAGE_BYTES = 2 * L * 32 * (int)sizeof(Tin);
    static constexpr int CARRY_OFF = NS * STAGE_BYTES;                 // [W][2][32] fp64
    static constexpr int META_OFF = CARRY_OFF + W * 2 * 32 * 8;        // per stage: StreamChunk
    static constexpr int BAR_OFF = align_up(META_OFF + NS * (int)sizeof(StreamChunk), 128);
    static constexpr int SMEM = align_up(BAR_OFF + (2 * NS + W) * 8, 128);
};

// Kernel powers of one channel: kappa_m = a^(-2m), nu_m = a^(-m) for
// m = 1..S in fp32, and the chunk multipliers kappa_L, nu_L in fp64, all
// from fp64 products of the correctly rounded 1/a.
template <int S, int L>
struct LtiPowers {
    float k[S + 1], n[S + 1];
    double kL, nL;
};

template <int S, int L>
__device__ __forceinline__ void lti_powers(double a, LtiPowers<S, L> &w) {
    const double r = 1.0 / a;
    double nu = 1.0;
    w.k[0] = 1.f;
    w.n[0] = 1.f;
#pragma unroll
    for (int m = 1; m <= S; ++m) {
        nu *= r;
        w.n[m] = (float)nu;
        w.k[m] = (float)(nu * nu);
    }
    double nL = 1.0, base = r;  // r^L by squaring
#pragma unroll
    for (int e = L; e > 0; e >>= 1) {
        if (e & 1) nL *= base;
        base *= base;
    }
    w.nL = nL;
    w.kL = nL * nL;
}

template <typename Tin, int L, int S, int W, int NS>
__global__ void __launch_bounds__(32 * (W + 1), 1)
kla_lti_stream_kernel(const LtiParams prm, const __grid_constant__ LtiMaps maps) {
    static_assert(L % S == 0, "sub-blocks tile the chunk");
    using Cfg = LtiTile<Tin, L, W, NS>;
    constexpr int LC = L * 32;
    constexpr int NSB = L / S;
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + Cfg::BAR_OFF);
    uint64_t *empty = full + NS;
    uint64_t *carry_bar = empty + NS;
    double *slots = reinterpret_cast<double *>(smem + Cfg::CARRY_OFF);
    StreamChunk *meta = reinterpret_cast<StreamChunk *>(smem + Cfg::META_OFF);

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
        int next = 0, round = 0;
        auto claim = [&]() -> int {
            const int s = next;
            if (round > 0) mbar_wait_or_flag(&empty[s], (unsigned)((round - 1) & 1), prm.wait_ns);
            if (++next == NS) {
                next = 0;
                ++round;
            }
            return s;
        };
        auto unit_chunks = [&](int64_t u) {
            StreamChunk m;
            m.tile = u % prm.ntiles;
            m.part = (int)(u / prm.ntiles);
            m.bb = (int)(m.tile / prm.nct);
            m.ct = (int)(m.tile - (int64_t)m.bb * prm.nct);
            m.first = m.part * prm.chunks_per_part;
            m.last = min(m.first + prm.chunks_per_part, prm.nchunks) - 1;
#pragma unroll 1
            for (int c = m.first; c <= m.last; ++c) {
                const int s = claim();
                m.chunk = c;
                meta[s] = m;
                Tin *stage = reinterpret_cast<Tin *>(smem + s * Cfg::STAGE_BYTES);
                mbar_arrive_expect_tx(&full[s], (unsigned)Cfg::STAGE_BYTES);
                tma_load_3d(stage, &maps.in[0], m.ct * 32, c * L, m.bb, &full[s]);
                tma_load_3d(stage + LC, &maps.in[1], m.ct * 32, c * L, m.bb, &full[s]);
            }
        };
        if (prm.ticket == nullptr) {  // round-robin units
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
#pragma unroll 1
        for (int k = 0; k < W; ++k) {
            const int s = claim();
            meta[s].chunk = -1;
            mbar_arrive(&full[s]);
        }
        return;
    }

    // ------------------------------------------------------------ chunk warps
    const int w = warp - 1;
    int64_t power_tile = -1;  // tile whose kernel powers `kp` holds
    LtiPowers<S, L> kp;
#pragma unroll 1
    for (int64_t j = w;; j += W) {
        const int s = (int)(j % NS);
        mbar_wait_or_flag(&full[s], (unsigned)((j / NS) & 1), prm.wait_ns);
        const StreamChunk m = meta[s];
        if (m.chunk < 0) break;
        const int64_t chunk = m.chunk;
        const int64_t tile = m.tile;
        const int64_t part = m.part;
        const int64_t bb = m.bb;
        const int64_t ct = m.ct;
        const int64_t t0 = chunk * L;
        const int64_t ch = ct * 32 + lane;
        const bool cvalid = ch < prm.HN;
        const int64_t first = m.first;
        const int64_t last = m.last;
        if (tile != power_tile) {
            lti_powers<S, L>(cvalid ? (double)prm.a[bb * prm.HN + ch] : 1.0, kp);
            power_tile = tile;
        }
        const Tin *stage = reinterpret_cast<const Tin *>(smem + s * Cfg::STAGE_BYTES);
        float x[L], y[L];  // phi, b; then the local convolutions
#pragma unroll
        for (int t = 0; t < L; ++t) {
            x[t] = to_f32(stage[t * 32 + lane]);
            y[t] = to_f32(stage[LC + t * 32 + lane]);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);

        // (1) local convolutions of each sub-block, in place (descending i:
        //     output i needs inputs <= i only)
#pragma unroll
        for (int q = 0; q < NSB; ++q) {
#pragma unroll
            for (int i = S - 1; i >= 1; --i) {
                float ax = x[q * S + i], ay = y[q * S + i];
#pragma unroll
                for (int m = 1; m <= i; ++m) {
                    ax = fmaf(kp.k[m], x[q * S + i - m], ax);
                    ay = fmaf(kp.n[m], y[q * S + i - m], ay);
                }
                x[q * S + i] = ax;
                y[q * S + i] = ay;
            }
        }
        // (2) exit of the chunk with zero entry
        float zx = 0.f, zy = 0.f;
#pragma unroll
        for (int q = 0; q < NSB; ++q) {
            zx = fmaf(kp.k[S], zx, x[q * S + S - 1]);
            zy = fmaf(kp.n[S], zy, y[q * S + S - 1]);
        }
        // (3) carry: the entering state from the previous chunk's warp, the
        //     prior at a tile's first chunk, or the previous run's state
        double lam_in = 0.0, eta_in = 0.0;
        if (j > 0) {
            const int ps = (int)((j - 1) % W);
            mbar_wait_or_flag(&carry_bar[ps], (unsigned)(((j - 1) / W) & 1), prm.wait_ns);
            lam_in = slots[ps * 64 + lane];
            eta_in = slots[ps * 64 + 32 + lane];
        }
        if (chunk == 0) {
            lam_in = cvalid ? (double)prm.lam0[bb * prm.HN + ch] : 1.0;
            eta_in = cvalid ? (double)prm.eta0[bb * prm.HN + ch] : 0.0;
        } else if (chunk == first) {
            const int64_t slot = tile * (prm.parts - 1) + (part - 1);
            if (warp_wait_flags(lane == 0 ? prm.part_flags + slot : nullptr, prm.wait_ns)) {
                lam_in = __ldcg(prm.part_state + slot * 64 + lane);
                eta_in = __ldcg(prm.part_state + slot * 64 + 32 + lane);
            } else {
                lam_in = __longlong_as_double(0x7ff8000000000000ll);
                eta_in = lam_in;
                if (lane == 0) atomicOr(&g_error_word, DEV_ERR_TIMEOUT);
            }
        }
        const double lam_out = fma(kp.kL, lam_in, (double)zx);
        const double eta_out = fma(kp.nL, eta_in, (double)zy);
        {
            const int ms = (int)(j % W);
            slots[ms * 64 + lane] = lam_out;
            slots[ms * 64 + 32 + lane] = eta_out;
            __syncwarp();
            if (lane == 0) mbar_arrive(&carry_bar[ms]);
            if (chunk == last && part + 1 < prm.parts) {
                const int64_t slot = tile * (prm.parts - 1) + part;
                prm.part_state[slot * 64 + lane] = lam_out;
                prm.part_state[slot * 64 + 32 + lane] = eta_out;
                __threadfence();
                __syncwarp();
                if (lane == 0) st_release_gpu(prm.part_flags + slot, 1u);
            }
        }
        // (4) final pass, sub-block by sub-block, into the output boxes
        float sl = (float)lam_in, se = (float)eta_in;
#pragma unroll
        for (int q = 0; q < NSB; ++q) {
#pragma unroll
            for (int i = 0; i < S; ++i) {
                x[q * S + i] = fmaf(kp.k[i + 1], sl, x[q * S + i]);
                y[q * S + i] = fmaf(kp.n[i + 1], se, y[q * S + i]);
            }
            sl = x[q * S + S - 1];
            se = y[q * S + S - 1];
        }
        // outputs straight from registers: one coalesced 128-byte row per
        // output and token (rows past T and lanes past H*N are not stored)
        if (cvalid) {
            const int nv = (int)(prm.T - t0 < L ? prm.T - t0 : L);
            const int64_t base = (bb * prm.T + t0) * prm.HN + ch;
            const int64_t hn = prm.HN;
            float *o0 = prm.out[0] + base, *o1 = prm.out[1] + base;
            float *o2 = prm.write_mu ? prm.out[2] + base : nullptr;
            float *o3 = prm.write_var ? prm.out[3] + base : nullptr;
            auto put = [&](int t) {
                const float v = rcp_hw(x[t]);
                __stcs(o0, x[t]);
                __stcs(o1, y[t]);
                if (o2) __stcs(o2, y[t] * v);
                if (o3) __stcs(o3, v);
                o0 += hn; o1 += hn;
                if (o2) o2 += hn;
                if (o3) o3 += hn;
            };
            if (nv == L) {
#pragma unroll
                for (int t = 0; t < L; ++t) put(t);
            } else {
#pragma unroll
                for (int t = 0; t < L; ++t)
                    if (t < nv) put(t);
            }
        }
    }
}

// Any shape (no TMA geometry needed): one thread per channel walks its
// sequence in sub-blocks of S tokens with plain loads, with the same local
// convolution and carry as above (the carry from sub-block to sub-block,
// kept in fp64).
template <typename Tin, int S>
__global__ void __launch_bounds__(128) kla_lti_seq_kernel(const LtiParams prm, const void *phi_v,
                                                          const void *b_v, float *lam_o, float *eta_o,
                                                          float *mu_o, float *var_o, int64_t C) {
    const int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= C) return;
    const int64_t bb = c / prm.HN;
    const int64_t ch = c - bb * prm.HN;
    const Tin *phi = static_cast<const Tin *>(phi_v);
    const Tin *b = static_cast<const Tin *>(b_v);
    LtiPowers<S, S> kp;
    lti_powers<S, S>((double)prm.a[c], kp);
    double lam = prm.lam0[c], eta = prm.eta0[c];
#pragma unroll 1
    for (int64_t t0 = 0; t0 < prm.T; t0 += S) {
        const int nv = (int)(prm.T - t0 < S ? prm.T - t0 : S);
        float x[S], y[S];
#pragma unroll
        for (int i = 0; i < S; ++i) {
            const int64_t idx = (bb * prm.T + t0 + i) * prm.HN + ch;
            x[i] = i < nv ? to_f32(phi[idx]) : 0.f;
            y[i] = i < nv ? to_f32(b[idx]) : 0.f;
        }
#pragma unroll
        for (int i = S - 1; i >= 1; --i) {
            float ax = x[i], ay = y[i];
#pragma unroll
            for (int m = 1; m <= i; ++m) {
                ax = fmaf(kp.k[m], x[i - m], ax);
                ay = fmaf(kp.n[m], y[i - m], ay);
            }
            x[i] = ax;
            y[i] = ay;
        }
        const float sl = (float)lam, se = (float)eta;
        const double zl = x[S - 1], ze = y[S - 1];
#pragma unroll
        for (int i = 0; i < S; ++i) {
            x[i] = fmaf(kp.k[i + 1], sl, x[i]);
            y[i] = fmaf(kp.n[i + 1], se, y[i]);
            if (i < nv) {
                const int64_t idx = (bb * prm.T + t0 + i) * prm.HN + ch;
                const float v = rcp_hw(x[i]);
                lam_o[idx] = x[i];
                eta_o[idx] = y[i];
                if (mu_o) mu_o[idx] = y[i] * v;
                if (var_o) var_o[idx] = v;
            }
        }
        lam = fma(kp.kL, lam, zl);  // kL = kappa_S here
        eta = fma(kp.nL, eta, ze);
    }
}

}  // namespace kla
