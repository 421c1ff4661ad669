// kla_backward.cuh -- gradients of the KLA filter scan (sm_100a).
//
// The KLA review claims end-to-end parallel training of the layer but gives no
// backward pass.  This is reverse-mode differentiation of the information-form
// recursion the forward kernels run.  Per channel, with lambda_0, eta_0 the
// prior and t = 1..T:
//
//   D_t = a_t^2 + p_t lambda_{t-1},  r_t = 1 / D_t,  f_t = a_t r_t (the gate),
//   lambda_t = lambda_{t-1} r_t + phi_t,  eta_t = f_t eta_{t-1} + b_t,
//   mu_t = eta_t / lambda_t,  var_t = 1 / lambda_t.
//
// Given a loss's gradients with respect to the four outputs (g_lambda, g_eta,
// g_mu, g_var), first fold mu and var into the two state outputs:
//
//   gl_t = g_lambda_t - v_t (g_mu_t mu_t + g_var_t v_t),  ge_t = g_eta_t + g_mu_t v_t
//   (v_t = 1 / lambda_t).
//
// The total derivatives E_t = dL/d eta_t and Lam_t = dL/d lambda_t then run
// BACKWARD in time through a linear recursion,
//
//   E_t   = ge_t + oE_{t+1},        Lam_t = gl_t + oL_{t+1},
//   oE_t  = f_t E_t,                oL_t  = f_t^2 Lam_t + c_t E_t,
//   c_t   = d eta_t / d lambda_{t-1} = -p_t f_t r_t eta_{t-1},
//   (f_t^2 = d lambda_t / d lambda_{t-1}, the identity the oracle's tests pin),
//
// with (oE, oL) = 0 after the last token, and every input's gradient is local:
//
//   d/d phi_t = Lam_t,   d/d b_t = E_t,
//   d/d a_t   = r_t^2 (-2 a_t lambda_{t-1} Lam_t + (p_t lambda_{t-1} - a_t^2) eta_{t-1} E_t),
//   d/d p_t   = -r_t^2 lambda_{t-1} (lambda_{t-1} Lam_t + a_t eta_{t-1} E_t),
//   d/d eta_0 = oE_1,   d/d lambda_0 = oL_1.
//
// Only a, p and the forward's lambda, eta are read (phi and b enter through
// lambda and eta).  The recursion's coefficients depend on the stored forward
// states only, so unlike the forward scan the backward one is linear in its
// carry: a chunk's effect on the carry is a 2x2 lower-triangular matrix
// [[m11, 0], [m21, m11^2]] plus an offset, composed without any
// renormalisation.
//
// Two kernels:
//   kla_backward_stream_kernel  the channel-owning streaming kernel, the
//       forward's K1 run backwards in time: a producer warp streams chunks of
//       L tokens x 32 channels (a, p, lambda and eta with one row of history,
//       the four output gradients) from the end of the sequence to its start
//       through a TMA ring; chunk warps copy a chunk into registers, (1) fold
//       it into its carry map, (2) take the carry from the warp of the later
//       chunk and hand the earlier one its carry, (3) re-run the exact
//       recursion from the carry and store the four input gradients through
//       double-buffered TMA-store boxes.  Tiles that do not balance over the
//       SMs are cut into runs taken by ticket (the latest run first); more
//       tiles than SMs, each long enough, are taken whole by ticket.
//   kla_backward_seq_kernel  one thread per channel walking the sequence
//       backwards with plain loads; for shapes the TMA geometry does not fit.
#pragma once

#include "kla_forward_stream.cuh"

namespace kla {

// Output gradients folded into the state outputs' gradients (gl, ge).
__device__ __forceinline__ void bwd_fold_outputs(float lam, float eta, float g_lam, float g_eta,
                                                 float g_mu, float g_var, float &gl, float &ge) {
    const float v = rcp_hw(lam);
    const float mu = eta * v;
    gl = g_lam - v * fmaf(g_mu, mu, g_var * v);
    ge = fmaf(g_mu, v, g_eta);
}

struct BwdGrads { float a, p, phi, b; };

// One token backwards: (E_, L_) is the gradient flowing in from the later
// tokens (oE_{t+1}, oL_{t+1}) and leaves as (oE_t, oL_t).  r = 1 / (a^2 + p
// lambda_{t-1}).
__device__ __forceinline__ BwdGrads bwd_token(float a, float p, float lp, float ep, float r,
                                              float gl, float ge, float &E_, float &L_) {
    const float E = ge + E_;
    const float Lm = gl + L_;
    const float f = a * r;
    const float c = -(p * r) * (f * ep);
    const float rr = r * r;
    BwdGrads g;
    g.a = rr * fmaf(-2.f * a * lp, Lm, (fmaf(p, lp, -(a * a)) * ep) * E);
    g.p = -(rr * lp) * fmaf(lp, Lm, (a * ep) * E);
    g.phi = Lm;
    g.b = E;
    E_ = f * E;
    L_ = fmaf(f * f, Lm, c * E);
    return g;
}

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

struct BwdParams {
    const void *a, *p;             // [B, T, H, N] inputs (plain-load kernel)
    const float *lam, *eta;        // [B, T, H, N] forward outputs (plain-load kernel)
    const float *g[4];             // g_lambda, g_eta, g_mu, g_var; null = zero (plain-load kernel)
    void *grad[4];                 // d/d a, p, phi, b; null = not wanted (plain-load kernel)
    const float *lam0, *eta0;      // [B, H, N] prior
    float *g_lam0, *g_eta0;        // [B, H, N] its gradients; null = not wanted
    int64_t T, HN, C;
    int64_t ntiles;                // B * ceil(HN / 32)
    int nct;                       // 32-channel tiles per batch row
    int nchunks;                   // ceil(T / L)
    unsigned g_mask;               // bit k: output gradient k present
    unsigned grad_mask;            // bit k: input gradient k wanted
    unsigned stage_tx;             // bytes one stage's TMA loads deliver
    uint64_t wait_ns;
    // Runs (parts > 1): unit u = q * ntiles + tile covers the tile's run
    // parts - 1 - q (the latest run first); run r enters at its last chunk
    // with the carry that run r + 1 published in part_state (flag part_flags).
    int parts, chunks_per_part;
    int64_t nunits;
    unsigned *ticket;              // unit counter (zeroed per call); null: round-robin units
    unsigned *part_flags;          // [ntiles][parts - 1]
    float *part_state;             // [ntiles][parts - 1][2][32]
    int64_t stall_chunk;           // test hook: this chunk's carry waits on a flag nothing sets (-1: off)
};

// What the producer tells the chunk warps about the chunk in a stage
// (computed once per work unit, so the chunk warps do no index division).
struct BwdChunk {
    int64_t tile;      // b * nct + channel tile
    int chunk;         // chunk index in the sequence; -1: no more work
    int run;           // the run of the tile this chunk belongs to
    int bb, ct;        // batch row, 32-channel tile within the row
    int run_lo, run_hi;  // first and last chunk of the run
};

struct BwdMaps {
    CUtensorMap in[8];   // a, p (input dtype), lambda, eta (box L + 1 rows), g_lambda, g_eta, g_mu, g_var
    CUtensorMap out[4];  // d/d a, p, phi, b (input dtype), box G rows
};

template <typename Tin, int L, int W, int NS, int G>
struct BwdTile {
    // Same ring discipline as the forward streaming kernel (chunk j in stage
    // j % NS, warp j % W; NS >= W keeps the mbarrier parities unambiguous).
    static_assert(NS >= W, "the stage ring must be at least as deep as the number of chunk warps");
    static_assert(L % G == 0, "output groups must tile the chunk");
    static constexpr int CW = 32;
    static constexpr int THREADS = 32 * (W + 1);
    static constexpr int IN_BYTES = L * CW * (int)sizeof(Tin);   // a or p
    static constexpr int ST_BYTES = (L + 1) * CW * 4;             // lambda or eta with one row of history
    static constexpr int GR_BYTES = L * CW * 4;                   // one output gradient
    static constexpr int OFF_P = IN_BYTES;
    static constexpr int OFF_LAM = 2 * IN_BYTES;
    static constexpr int OFF_ETA = OFF_LAM + ST_BYTES;
    static constexpr int OFF_G = OFF_ETA + ST_BYTES;
    static constexpr int STAGE_BYTES = OFF_G + 4 * GR_BYTES;
    static_assert(IN_BYTES % 128 == 0 && ST_BYTES % 128 == 0, "TMA destinations stay 128-byte aligned");
    static constexpr int OUTBOX_BYTES = G * CW * (int)sizeof(Tin);  // one gradient, one group
    static constexpr int OUTBUF_BYTES = 4 * OUTBOX_BYTES;
    static_assert(OUTBOX_BYTES % 128 == 0, "TMA store sources stay 128-byte aligned");
    static constexpr int OUT_OFF = NS * STAGE_BYTES;                 // [W][2][4][G][32]
    static constexpr int CARRY_OFF = OUT_OFF + W * 2 * OUTBUF_BYTES; // [W][2][32] fp32
    static constexpr int META_OFF = CARRY_OFF + W * 2 * CW * 4;      // [NS] BwdChunk
    static constexpr int BAR_OFF = align_up(META_OFF + NS * (int)sizeof(BwdChunk), 128);
    static constexpr int SMEM = align_up(BAR_OFF + (2 * NS + W) * 8, 128);
};

template <typename Tin, int L, int W, int NS, int G>
__global__ void __launch_bounds__(32 * (W + 1), 1)
kla_backward_stream_kernel(const BwdParams prm, const __grid_constant__ BwdMaps maps) {
    using Cfg = BwdTile<Tin, L, W, NS, G>;
    constexpr int LC = L * 32;
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + Cfg::BAR_OFF);
    uint64_t *empty = full + NS;
    uint64_t *carry_bar = empty + NS;
    float *slots = reinterpret_cast<float *>(smem + Cfg::CARRY_OFF);
    BwdChunk *meta = reinterpret_cast<BwdChunk *>(smem + Cfg::META_OFF);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    // Absent output gradients are read as zeros: clear their slots once.
    for (int k = 0; k < 4; ++k) {
        if (prm.g_mask >> k & 1u) continue;
        for (int s = 0; s < NS; ++s) {
            float *z = reinterpret_cast<float *>(smem + s * Cfg::STAGE_BYTES + Cfg::OFF_G + k * Cfg::GR_BYTES);
            for (int i = tid; i < LC; i += Cfg::THREADS) z[i] = 0.f;
        }
    }
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
        auto load = [&](const BwdChunk &m) {
            const int s = claim();
            const int x = m.ct * 32;
            const int y = m.chunk * L;
            const int bb = m.bb;
            meta[s] = m;
            unsigned char *stage = smem + s * Cfg::STAGE_BYTES;
            mbar_arrive_expect_tx(&full[s], prm.stage_tx);
            tma_load_3d(stage, &maps.in[0], x, y, bb, &full[s]);
            tma_load_3d(stage + Cfg::OFF_P, &maps.in[1], x, y, bb, &full[s]);
            // one row of history: the state entering the chunk (row -1 of
            // the first chunk lies outside the tensor and reads as zeros)
            tma_load_3d(stage + Cfg::OFF_LAM, &maps.in[2], x, y - 1, bb, &full[s]);
            tma_load_3d(stage + Cfg::OFF_ETA, &maps.in[3], x, y - 1, bb, &full[s]);
#pragma unroll
            for (int k = 0; k < 4; ++k)
                if (prm.g_mask >> k & 1u)
                    tma_load_3d(stage + Cfg::OFF_G + k * Cfg::GR_BYTES, &maps.in[4 + k], x, y, bb, &full[s]);
        };
        // one unit: the tile's run r, latest chunk first
        auto unit_chunks = [&](int64_t u) {
            BwdChunk m;
            m.tile = u % prm.ntiles;
            m.run = prm.parts - 1 - (int)(u / prm.ntiles);
            m.bb = (int)(m.tile / prm.nct);
            m.ct = (int)(m.tile - (int64_t)m.bb * prm.nct);
            m.run_lo = m.run * prm.chunks_per_part;
            m.run_hi = min(m.run_lo + prm.chunks_per_part, prm.nchunks) - 1;
#pragma unroll 1
            for (int c = m.run_hi; c >= m.run_lo; --c) {
                m.chunk = c;
                load(m);
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
    Tin *outbuf0 = reinterpret_cast<Tin *>(smem + Cfg::OUT_OFF + w * 2 * Cfg::OUTBUF_BYTES);
    int group_seq = 0;
    // This warp takes the CTA's chunks j = w, w + W, w + 2W, ...: chunk j sits
    // in stage j % NS (phase parity (j / NS) & 1), and its carry comes from
    // warp (j - 1) % W.  Tracked incrementally (W <= NS).
    int s = w;
    unsigned par = 0;
    const int prev_w = w > 0 ? w - 1 : W - 1;
#pragma unroll 1
    for (int k = 0;; ++k) {
        mbar_wait_or_flag(&full[s], par, prm.wait_ns);
        const BwdChunk m = meta[s];
        const int stage_s = s;
        s += W;
        if (s >= NS) {
            s -= NS;
            par ^= 1u;
        }
        if (m.chunk < 0) break;
        const bool has_prev = k > 0 || w > 0;                  // j > 0
        const unsigned prev_par = (unsigned)((w > 0 ? k : k - 1) & 1);  // ((j - 1) / W) & 1
        const int chunk = m.chunk;
        const int run = m.run;
        const int64_t tile = m.tile;
        const int64_t bb = m.bb;
        const int64_t ct = m.ct;
        const int64_t t0 = (int64_t)chunk * L;
        const int t_valid = (int)(prm.T - t0 < (int64_t)L ? prm.T - t0 : (int64_t)L);
        const int64_t ch = ct * 32 + lane;
        const bool cvalid = ch < prm.HN;
        const unsigned char *stage = smem + stage_s * Cfg::STAGE_BYTES;
        const Tin *sa = reinterpret_cast<const Tin *>(stage);
        const Tin *sp = reinterpret_cast<const Tin *>(stage + Cfg::OFF_P);
        const float *sl = reinterpret_cast<const float *>(stage + Cfg::OFF_LAM);  // row 0 = history
        const float *se = reinterpret_cast<const float *>(stage + Cfg::OFF_ETA);
        const float *sg = reinterpret_cast<const float *>(stage + Cfg::OFF_G);
        const int run_lo = m.run_lo;
        const int run_hi = m.run_hi;
        float prior_lam = 1.f, prior_eta = 0.f;
        if (chunk == 0 && cvalid) {
            prior_lam = prm.lam0[bb * prm.HN + ch];
            prior_eta = prm.eta0[bb * prm.HN + ch];
        }

        // Carry entering the chunk from the later tokens: from the warp of
        // the later chunk, zero after the last chunk, or published by the
        // tile's later run at a run's last chunk.
        auto carry_in = [&](float &cE, float &cL) {
            if (has_prev) {
                mbar_wait_or_flag(&carry_bar[prev_w], prev_par, prm.wait_ns);
                cE = slots[prev_w * 64 + lane];
                cL = slots[prev_w * 64 + 32 + lane];
            }
            if (chunk == prm.stall_chunk &&
                !warp_wait_flags(lane == 0 ? &g_never_set_word : nullptr, prm.wait_ns)) {
                cE = __int_as_float(0x7fc00000);  // ran out of time: poison what follows
                cL = cE;
                if (lane == 0) atomicOr(&g_error_word, DEV_ERR_TIMEOUT);
            } else if (chunk == prm.nchunks - 1) {
                cE = 0.f;
                cL = 0.f;
            } else if (chunk == run_hi) {
                const int64_t slot = tile * (prm.parts - 1) + run;
                if (warp_wait_flags(lane == 0 ? prm.part_flags + slot : nullptr, prm.wait_ns)) {
                    cE = __ldcg(prm.part_state + slot * 64 + lane);
                    cL = __ldcg(prm.part_state + slot * 64 + 32 + lane);
                } else {
                    cE = __int_as_float(0x7fc00000);
                    cL = cE;
                    if (lane == 0) atomicOr(&g_error_word, DEV_ERR_TIMEOUT);
                }
            }
        };
        // Carry leaving the chunk towards the earlier tokens.
        auto carry_out = [&](float oE, float oL) {
            slots[w * 64 + lane] = oE;
            slots[w * 64 + 32 + lane] = oL;
            __syncwarp();
            if (lane == 0) mbar_arrive(&carry_bar[w]);
            if (chunk == run_lo && run > 0) {
                const int64_t slot = tile * (prm.parts - 1) + (run - 1);
                prm.part_state[slot * 64 + lane] = oE;
                prm.part_state[slot * 64 + 32 + lane] = oL;
                __threadfence();
                __syncwarp();
                if (lane == 0) st_release_gpu(prm.part_flags + slot, 1u);
            }
        };
        auto group_begin = [&]() -> Tin * {
            Tin *buf = outbuf0 + (group_seq & 1) * (Cfg::OUTBUF_BYTES / (int)sizeof(Tin));
            if (group_seq >= 2) {
                if (lane == 0) bulk_wait_group_read<1>();
                __syncwarp();
            }
            return buf;
        };
        auto group_end = [&](Tin *buf, int q) {
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                const int ty = (int)(t0 + q * G);
                const int x = (int)(ct * 32);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    if (prm.grad_mask >> k & 1u) tma_store_3d(&maps.out[k], buf + k * G * 32, x, ty, (int)bb);
                bulk_commit_group();
            }
            ++group_seq;
        };
        auto put = [&](Tin *buf, int u, const BwdGrads &g) {
            buf[u * 32 + lane] = from_f32<Tin>(g.a);
            buf[G * 32 + u * 32 + lane] = from_f32<Tin>(g.p);
            buf[2 * G * 32 + u * 32 + lane] = from_f32<Tin>(g.phi);
            buf[3 * G * 32 + u * 32 + lane] = from_f32<Tin>(g.b);
        };
        auto prior_out = [&](float oE, float oL) {
            if (chunk == 0 && cvalid) {
                if (prm.g_eta0) prm.g_eta0[bb * prm.HN + ch] = oE;
                if (prm.g_lam0) prm.g_lam0[bb * prm.HN + ch] = oL;
            }
        };

        if (t_valid == L) {
            // Full chunk: into registers, stage released, then both passes.
            float xa[L], xp[L], xl[L + 1], xe[L + 1], xgl[L], xge[L];
#pragma unroll
            for (int t = 0; t <= L; ++t) {
                xl[t] = sl[t * 32 + lane];
                xe[t] = se[t * 32 + lane];
            }
#pragma unroll
            for (int t = 0; t < L; ++t) {
                const int i = t * 32 + lane;
                xa[t] = to_f32(sa[i]);
                xp[t] = to_f32(sp[i]);
                bwd_fold_outputs(xl[t + 1], xe[t + 1], sg[i], sg[LC + i], sg[2 * LC + i], sg[3 * LC + i],
                                 xgl[t], xge[t]);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage_s]);
            if (chunk == 0) {
                xl[0] = prior_lam;
                xe[0] = prior_eta;
            }
            // (1) the chunk's carry map: carry_out = [[m11, 0], [m21, m11^2]] carry_in + off
            float m11 = 1.f, m21 = 0.f, offE = 0.f, offL = 0.f;
#pragma unroll
            for (int t = L - 1; t >= 0; --t) {
                const float a = xa[t], p = xp[t];
                const float r = rcp_hw(fmaf(p, xl[t], a * a));
                const float f = a * r;
                const float f2 = f * f;
                const float c = -(p * r) * (f * xe[t]);
                const float El = xge[t] + offE;
                const float Ll = xgl[t] + offL;
                offE = f * El;
                offL = fmaf(f2, Ll, c * El);
                m21 = fmaf(c, m11, f2 * m21);
                m11 = f * m11;
            }
            // (2) carry
            float cE = 0.f, cL = 0.f;
            carry_in(cE, cL);
            carry_out(fmaf(m11, cE, offE), fmaf(m11 * m11, cL, fmaf(m21, cE, offL)));
            // (3) exact recursion from the carry, latest token first
#pragma unroll
            for (int q = L / G - 1; q >= 0; --q) {
                Tin *buf = group_begin();
#pragma unroll
                for (int u = G - 1; u >= 0; --u) {
                    const int t = q * G + u;
                    // r again (one multiply-add and one reciprocal are
                    // cheaper than keeping L more registers live)
                    const float r = rcp_hw(fmaf(xp[t], xl[t], xa[t] * xa[t]));
                    put(buf, u, bwd_token(xa[t], xp[t], xl[t], xe[t], r, xgl[t], xge[t], cE, cL));
                }
                group_end(buf, q);
            }
            prior_out(cE, cL);
        } else {
            // Ragged last chunk (processed first, carry zero): straight from
            // shared memory, released at the end; rows past T are clipped by
            // the TMA stores.
            float cE = 0.f, cL = 0.f;
            carry_in(cE, cL);
            const int ngroups = (t_valid + G - 1) / G;
#pragma unroll 1
            for (int q = ngroups - 1; q >= 0; --q) {
                Tin *buf = group_begin();
#pragma unroll 1
                for (int u = G - 1; u >= 0; --u) {
                    const int t = q * G + u;
                    if (t >= t_valid) continue;
                    const int i = t * 32 + lane;
                    const float lp = (t == 0 && chunk == 0) ? prior_lam : sl[i];
                    const float ep = (t == 0 && chunk == 0) ? prior_eta : se[i];
                    float gl, ge;
                    bwd_fold_outputs(sl[i + 32], se[i + 32], sg[i], sg[LC + i], sg[2 * LC + i], sg[3 * LC + i],
                                     gl, ge);
                    const float a = to_f32(sa[i]), p = to_f32(sp[i]);
                    const float r = rcp_hw(fmaf(p, lp, a * a));
                    put(buf, u, bwd_token(a, p, lp, ep, r, gl, ge, cE, cL));
                }
                group_end(buf, q);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage_s]);
            carry_out(cE, cL);
            prior_out(cE, cL);
        }
    }
    if (lane == 0) bulk_wait_group_all();
    __syncwarp();
}

// One thread per channel, backwards over the whole sequence, plain loads.
template <typename Tin>
__global__ void __launch_bounds__(128)
kla_backward_seq_kernel(const BwdParams prm) {
    const int64_t ch = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (ch >= prm.C) return;
    const int64_t bb = ch / prm.HN;
    const int64_t hn = ch - bb * prm.HN;
    const int64_t base = bb * prm.T * prm.HN + hn;
    const Tin *a_in = static_cast<const Tin *>(prm.a);
    const Tin *p_in = static_cast<const Tin *>(prm.p);
    Tin *out[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) out[k] = static_cast<Tin *>(prm.grad[k]);
    float E_ = 0.f, L_ = 0.f;
#pragma unroll 1
    for (int64_t t = prm.T - 1; t >= 0; --t) {
        const int64_t i = base + t * prm.HN;
        const float a = to_f32(a_in[i]), p = to_f32(p_in[i]);
        const float lp = t > 0 ? prm.lam[i - prm.HN] : prm.lam0[ch];
        const float ep = t > 0 ? prm.eta[i - prm.HN] : prm.eta0[ch];
        float gl, ge;
        bwd_fold_outputs(prm.lam[i], prm.eta[i], prm.g[0] ? prm.g[0][i] : 0.f, prm.g[1] ? prm.g[1][i] : 0.f,
                         prm.g[2] ? prm.g[2][i] : 0.f, prm.g[3] ? prm.g[3][i] : 0.f, gl, ge);
        const float r = rcp_hw(fmaf(p, lp, a * a));
        const BwdGrads g = bwd_token(a, p, lp, ep, r, gl, ge, E_, L_);
        if (out[0]) out[0][i] = from_f32<Tin>(g.a);
        if (out[1]) out[1][i] = from_f32<Tin>(g.p);
        if (out[2]) out[2][i] = from_f32<Tin>(g.phi);
        if (out[3]) out[3][i] = from_f32<Tin>(g.b);
    }
    if (prm.g_eta0) prm.g_eta0[ch] = E_;
    if (prm.g_lam0) prm.g_lam0[ch] = L_;
}

}  // namespace kla
