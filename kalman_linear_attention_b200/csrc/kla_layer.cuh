// kla_layer.cuh -- the KLA layer's filter with its input and output fused
// (sm_100a).
//
// A KLA layer with H heads, value dimension D and state expansion Ns runs
// H x D x Ns independent scalar filters (the review's diagonal model).  State
// channel (h, d, n) observes value coordinate d through the observation
// operator k_n:
//
//   evidence   phi_t = k_{t,n}^2 w_{t,d},   b_t = k_{t,n} w_{t,d} v_{t,d}
//              (w = Lambda^v, the value precision: the update adds k^2 Lambda^v,
//              KLA review "Circularity Check", Theorem 1)
//   filter     the information-form recursion of kla_device.cuh with the
//              channel's time-invariant decay a and process noise p
//   readout    y_{t,d} = sum_n q_{t,n} mu_{t,d,n},  s_{t,d} = sum_n q_{t,n}^2 var_{t,d,n}
//              (the readout operator applied to the posterior mean, and the
//              variance of that readout under the diagonal posterior)
//
// Unfused, the layer would write phi and b ([B, T, H, D, Ns]) for the scan to
// read, and the scan would write mu and var of the same size for the readout
// to read.  Here a CTA owns a tile of 32 state channels -- 32 / Ns value
// coordinates x all Ns state channels of one head -- for the whole sequence,
// exactly like kla_forward_stream_kernel, and per token reads only k, q (Ns
// values each, TMA) and v, w (32 / Ns values each, cp.async: rows of 8 bytes
// are below the TMA minimum), and writes only y and s.  The chunk warps form
// the evidence in registers, run the chunk aggregate / carry / recursion of
// the streaming kernel, and reduce the readout over the Ns lanes of a value
// coordinate through a per-warp transpose in shared memory (each lane then
// sums whole rows for L / Ns tokens and stores their y and s).
#pragma once

#include "kla_forward_stream.cuh"
#include "kla_step.cuh"

namespace kla {

// Tokens between two renormalisations of the layer's chunk aggregates: 4
// (measured 8-9% faster than 2 on the layer workload; the evidence of a
// layer, k^2 Lambda^v, keeps the row sums of M_t far below the 2^31 per token
// that this interval needs).
#ifndef KLA_LAYER_RENORM_EVERY
#define KLA_LAYER_RENORM_EVERY 4
#endif

struct LayerParams {
    const void *v, *w;             // [B, T, H, D] values, value precision (input dtype)
    const float *a, *p;            // [H, D, Ns] per-channel decay and process noise
    const float *lam0, *eta0;      // [B, H, D, Ns] prior
    float *y, *s;                  // [B, T, H, D] readouts; s may be null
    float *lam_T, *eta_T;          // [B, H, D, Ns] state after the last token; may be null
    int64_t T;
    int H, D;
    int64_t ntiles;                // B * H * dtiles
    int dtiles;                    // D / (32 / Ns) tiles per head
    int nchunks;
    uint64_t wait_ns;
    int parts, chunks_per_part;    // run splits, as in the streaming forward kernel
    int64_t nunits;
    unsigned *ticket;
    unsigned *part_flags;          // [ntiles][parts - 1]
    float *part_state;             // [ntiles][parts - 1][2][32]
};

struct LayerMaps {
    CUtensorMap k, q;              // [B, T, H, Ns] as {Ns, H, T, B}, box {Ns, 1, L, 1}
};

struct LayerChunk {
    int64_t tile;                  // (b * H + h) * dtiles + dt
    int chunk;                     // -1: no more work
    int part;
    int bb, hh, dt;
    int first, last;               // chunks of the run
};

template <typename Tin, int NSX, int L, int W, int NS>
struct LayerTile {
    static_assert(NS >= W, "the stage ring must be at least as deep as the number of chunk warps");
    static_assert(L == 32, "one producer lane per token of a chunk");
    static_assert(NSX == 8 || NSX == 16, "state expansion 8 or 16");
    static constexpr int DPW = 32 / NSX;                                     // value coordinates per tile
    static constexpr int VW_COPY = DPW * (int)sizeof(Tin);                   // bytes per token row of v or w
    static_assert(VW_COPY == 4 || VW_COPY == 8 || VW_COPY == 16, "cp.async copies 4, 8 or 16 bytes");
    static constexpr int KQ_BYTES = L * NSX * (int)sizeof(Tin);
    static constexpr int VW_BYTES = align_up(L * VW_COPY, 128);
    static constexpr int OFF_Q = KQ_BYTES;
    static constexpr int OFF_V = 2 * KQ_BYTES;
    static constexpr int OFF_W = OFF_V + VW_BYTES;
    static constexpr int OFF_AP = OFF_W + VW_BYTES;                          // a[32], p[32] fp32
    static constexpr int STAGE_BYTES = OFF_AP + 256;
    static_assert(KQ_BYTES % 128 == 0 && STAGE_BYTES % 128 == 0, "TMA destinations stay 128-byte aligned");
    static constexpr int THREADS = 32 * (W + 1);
    static constexpr int CARRY_OFF = NS * STAGE_BYTES;                       // [W][2][32] fp32
    static constexpr int META_OFF = CARRY_OFF + W * 2 * 32 * 4;              // [NS] LayerChunk
    // Readout transpose, per chunk warp: the q mu and q^2 var terms of a
    // chunk, [2][L][TROW] fp32.  Rows are padded to 36 floats so that the
    // 16-byte row reads of eight lanes (eight tokens) fall in distinct banks.
    static constexpr int TROW = 36;
    static constexpr int TBUF_BYTES = 2 * L * TROW * 4;
    static constexpr int TBUF_OFF = align_up(META_OFF + NS * (int)sizeof(LayerChunk), 128);
    static constexpr int BAR_OFF = align_up(TBUF_OFF + W * TBUF_BYTES, 128);
    static constexpr int SMEM = align_up(BAR_OFF + (2 * NS + W) * 8, 128);
};

// Asynchronous global -> shared copy of N bytes (N = 4, 8 or 16; both
// addresses N-byte aligned).
template <int N>
__device__ __forceinline__ void cp_async(void *smem_dst, const void *gmem_src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], %2;"
                 :: "r"(smem_u32(smem_dst)), "l"(gmem_src), "n"(N) : "memory");
}

// Arrive on `bar` once every cp.async this thread issued before has landed;
// the arrival is one of the barrier's expected arrivals (no count increment).
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t *bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" :: "r"(smem_u32(bar)) : "memory");
}

// 4-D tiled TMA load global -> shared::cta, completion on `bar`.
__device__ __forceinline__ void tma_load_4d(void *smem_dst, const CUtensorMap *map, int c0, int c1, int c2,
                                            int c3, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cta.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5}], [%6];"
        :: "r"(smem_u32(smem_dst)), "l"(reinterpret_cast<uint64_t>(map)),
           "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar))
        : "memory");
}

// Sum of M consecutive floats of shared memory (16-byte aligned), as a
// pairwise tree of float4 reads.
template <int M>
__device__ __forceinline__ float row_sum(const float *src) {
    static_assert(M % 4 == 0, "whole float4 reads");
    float part[M / 4];
#pragma unroll
    for (int c = 0; c < M / 4; ++c) {
        const float4 v = *reinterpret_cast<const float4 *>(src + 4 * c);
        part[c] = (v.x + v.y) + (v.z + v.w);
    }
#pragma unroll
    for (int step = 1; step < M / 4; step *= 2)
#pragma unroll
        for (int c = 0; c + step < M / 4; c += 2 * step) part[c] += part[c + step];
    return part[0];
}

template <typename Tin, int NSX, int L, int W, int NS>
__global__ void __launch_bounds__(32 * (W + 1), 1)
kla_layer_forward_kernel(const LayerParams prm, const __grid_constant__ LayerMaps maps) {
    using Cfg = LayerTile<Tin, NSX, L, W, NS>;
    constexpr int DPW = Cfg::DPW;
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + Cfg::BAR_OFF);
    uint64_t *empty = full + NS;
    uint64_t *carry_bar = empty + NS;
    float *slots = reinterpret_cast<float *>(smem + Cfg::CARRY_OFF);
    LayerChunk *meta = reinterpret_cast<LayerChunk *>(smem + Cfg::META_OFF);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 33);   // the producer's lane 0 (TMA bytes) + one cp.async arrival per lane
            mbar_init(&empty[s], 1);
        }
        for (int s = 0; s < W; ++s) mbar_init(&carry_bar[s], 1);
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == 0) {
        // ------------------------------------------------------ producer warp
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
        const Tin *vg = static_cast<const Tin *>(prm.v);
        const Tin *wg = static_cast<const Tin *>(prm.w);
        auto load = [&](const LayerChunk &m) {
            const int s = claim();
            unsigned char *stage = smem + s * Cfg::STAGE_BYTES;
            if (lane == 0) {
                meta[s] = m;
                mbar_arrive_expect_tx(&full[s], (unsigned)(2 * Cfg::KQ_BYTES));
                tma_load_4d(stage, &maps.k, 0, m.hh, m.chunk * L, m.bb, &full[s]);
                tma_load_4d(stage + Cfg::OFF_Q, &maps.q, 0, m.hh, m.chunk * L, m.bb, &full[s]);
            }
            // lane = token of the chunk (rows past T repeat row T - 1: read, never used)
            int64_t t = (int64_t)m.chunk * L + lane;
            t = t < prm.T ? t : prm.T - 1;
            const int64_t row = ((int64_t)m.bb * prm.T + t) * prm.H + m.hh;
            const int64_t col = (int64_t)m.dt * DPW;
            cp_async<Cfg::VW_COPY>(stage + Cfg::OFF_V + lane * Cfg::VW_COPY, vg + row * prm.D + col);
            cp_async<Cfg::VW_COPY>(stage + Cfg::OFF_W + lane * Cfg::VW_COPY, wg + row * prm.D + col);
            // the tile's 32 channel parameters (contiguous in [H, D, Ns])
            const int64_t pc = ((int64_t)m.hh * prm.D + col) * NSX + lane;
            cp_async<4>(stage + Cfg::OFF_AP + lane * 4, prm.a + pc);
            cp_async<4>(stage + Cfg::OFF_AP + 128 + lane * 4, prm.p + pc);
            cp_async_arrive_noinc(&full[s]);
        };
        auto unit_chunks = [&](int64_t u) {
            LayerChunk m;
            m.tile = u % prm.ntiles;
            m.part = (int)(u / prm.ntiles);
            const int64_t bh = m.tile / prm.dtiles;
            m.dt = (int)(m.tile - bh * prm.dtiles);
            m.bb = (int)(bh / prm.H);
            m.hh = (int)(bh - (int64_t)m.bb * prm.H);
            m.first = m.part * prm.chunks_per_part;
            m.last = min(m.first + prm.chunks_per_part, prm.nchunks) - 1;
#pragma unroll 1
            for (int c = m.first; c <= m.last; ++c) {
                m.chunk = c;
                load(m);
            }
        };
        if (prm.parts == 1) {
#pragma unroll 1
            for (int64_t u = blockIdx.x; u < prm.nunits; u += gridDim.x) unit_chunks(u);
        } else {
            // one ticket per unit, taken by lane 0 and shared with the warp
#pragma unroll 1
            for (;;) {
                unsigned tk = 0;
                if (lane == 0) tk = atomicAdd(prm.ticket, 1u);
                const int64_t u = (int64_t)__shfl_sync(0xffffffffu, tk, 0);
                if (u >= prm.nunits) break;
                unit_chunks(u);
            }
        }
        // one end marker for each chunk warp (33 arrivals, no bytes)
#pragma unroll 1
        for (int k = 0; k < W; ++k) {
            const int s = claim();
            if (lane == 0) {
                meta[s].chunk = -1;
                mbar_arrive(&full[s]);
            }
            mbar_arrive(&full[s]);
        }
        return;
    }

    // ------------------------------------------------------------ chunk warps
    const int w = warp - 1;
    const int n = lane % NSX;          // state channel of the value coordinate
    const int dl = lane / NSX;         // value coordinate within the tile
    float *ty = reinterpret_cast<float *>(smem + Cfg::TBUF_OFF + w * Cfg::TBUF_BYTES);  // [L][TROW]
    float *ts = ty + L * Cfg::TROW;
    int s = w;
    unsigned par = 0;
    const int prev_w = w > 0 ? w - 1 : W - 1;
#pragma unroll 1
    for (int k = 0;; ++k) {
        mbar_wait_or_flag(&full[s], par, prm.wait_ns);
        const LayerChunk m = meta[s];
        const int stage_s = s;
        s += W;
        if (s >= NS) {
            s -= NS;
            par ^= 1u;
        }
        if (m.chunk < 0) break;
        const bool has_prev = k > 0 || w > 0;
        const unsigned prev_par = (unsigned)((w > 0 ? k : k - 1) & 1);
        const int chunk = m.chunk;
        const int64_t t0 = (int64_t)chunk * L;
        const int t_valid = (int)(prm.T - t0 < (int64_t)L ? prm.T - t0 : (int64_t)L);
        const int64_t chan = m.tile * 32 + lane;                 // index into [B, H, D, Ns]
        const int d = m.dt * DPW + dl;
        const unsigned char *stage = smem + stage_s * Cfg::STAGE_BYTES;
        const Tin *sk = reinterpret_cast<const Tin *>(stage);
        const Tin *sq = reinterpret_cast<const Tin *>(stage + Cfg::OFF_Q);
        const Tin *sv = reinterpret_cast<const Tin *>(stage + Cfg::OFF_V);
        const Tin *sw = reinterpret_cast<const Tin *>(stage + Cfg::OFF_W);
        const float a = reinterpret_cast<const float *>(stage + Cfg::OFF_AP)[lane];
        const float p = reinterpret_cast<const float *>(stage + Cfg::OFF_AP + 128)[lane];
        float *yrow = prm.y + (((int64_t)m.bb * prm.T + t0) * prm.H + m.hh) * prm.D + d;
        float *srow = prm.s ? prm.s + (yrow - prm.y) : nullptr;
        const int64_t ystride = (int64_t)prm.H * prm.D;

        // State entering the chunk, as in the streaming forward kernel.
        auto chunk_carry = [&](const Agg &g, float &lam, float &eta) {
            if (has_prev) {
                mbar_wait_or_flag(&carry_bar[prev_w], prev_par, prm.wait_ns);
                lam = slots[prev_w * 64 + lane];
                eta = slots[prev_w * 64 + 32 + lane];
            }
            if (chunk == 0) {
                lam = prm.lam0[chan];
                eta = prm.eta0[chan];
            } else if (chunk == m.first) {
                const int64_t slot = m.tile * (prm.parts - 1) + (m.part - 1);
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
            slots[w * 64 + lane] = lo;
            slots[w * 64 + 32 + lane] = eo;
            __syncwarp();
            if (lane == 0) mbar_arrive(&carry_bar[w]);
            if (chunk == m.last && m.part + 1 < prm.parts) {
                const int64_t slot = m.tile * (prm.parts - 1) + m.part;
                prm.part_state[slot * 64 + lane] = lo;
                prm.part_state[slot * 64 + 32 + lane] = eo;
                __threadfence();
                __syncwarp();
                if (lane == 0) st_release_gpu(prm.part_flags + slot, 1u);
            }
        };
        // Readout of one token of a ragged chunk: sum over the Ns lanes of the
        // value coordinate with shuffles, stored by the coordinate's lane n = 0.
        auto readout = [&](int t, float q, const TokenOut &o) {
            float ym = q * o.mu;
            float sv2 = (q * q) * o.var;
#pragma unroll
            for (int off = NSX / 2; off >= 1; off >>= 1) {
                ym += __shfl_xor_sync(0xffffffffu, ym, off);
                sv2 += __shfl_xor_sync(0xffffffffu, sv2, off);
            }
            if (n == 0) {
                __stcs(yrow + t * ystride, ym);
                if (srow) __stcs(srow + t * ystride, sv2);
            }
        };
        auto final_state = [&](float lam, float eta) {
            if (chunk == prm.nchunks - 1 && prm.lam_T) {
                prm.lam_T[chan] = lam;
                prm.eta_T[chan] = eta;
            }
        };

        if (t_valid == L) {
            // Full chunk: evidence and readout operator into registers, stage
            // released, then the aggregate, the carry and the recursion.
            float xf[L], xb[L], xq[L];
#pragma unroll
            for (int t = 0; t < L; ++t) {
                const float kk = to_f32(sk[t * NSX + n]);
                const float ww = to_f32(sw[t * DPW + dl]);
                const float vv = to_f32(sv[t * DPW + dl]);
                xf[t] = (kk * kk) * ww;
                xb[t] = (kk * ww) * vv;
                xq[t] = to_f32(sq[t * NSX + n]);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage_s]);
            Agg g = agg_identity();
#pragma unroll
            for (int t = 0; t < L; ++t) {
                agg_push_token(g, a, p, xf[t], xb[t]);
                if (renorm_after_every<KLA_LAYER_RENORM_EVERY>(t)) agg_renorm(g);
            }
            agg_renorm(g);
            float lam = 0.f, eta = 0.f;
            chunk_carry(g, lam, eta);
            // The readout of a full chunk, transposed: every lane writes its
            // terms q mu and q^2 var of each token into the warp's buffer
            // (one row per token), then lane (dl, n) sums row n + r Ns of its
            // value coordinate dl for r = 0 .. L/Ns - 1 and stores y and s of
            // those tokens -- L / Ns sums of Ns terms per lane instead of a
            // shuffle butterfly per token.
#pragma unroll
            for (int t = 0; t < L; ++t) {
                const TokenOut o = filter_token(lam, eta, a, p, xf[t], xb[t]);
                ty[t * Cfg::TROW + lane] = xq[t] * o.mu;
                ts[t * Cfg::TROW + lane] = (xq[t] * xq[t]) * o.var;
            }
            __syncwarp();
#pragma unroll
            for (int r = 0; r < L / NSX; ++r) {
                const int tok = r * NSX + n;
                const float sy = row_sum<NSX>(ty + tok * Cfg::TROW + dl * NSX);
                __stcs(yrow + tok * ystride, sy);
                if (srow) __stcs(srow + tok * ystride, row_sum<NSX>(ts + tok * Cfg::TROW + dl * NSX));
            }
            __syncwarp();
            final_state(lam, eta);
        } else {
            // Ragged last chunk, straight from shared memory.
            Agg g = agg_identity();
#pragma unroll 1
            for (int t = 0; t < t_valid; ++t) {
                const float kk = to_f32(sk[t * NSX + n]);
                const float ww = to_f32(sw[t * DPW + dl]);
                agg_push_token(g, a, p, (kk * kk) * ww, (kk * ww) * to_f32(sv[t * DPW + dl]));
                if (renorm_after_every<KLA_LAYER_RENORM_EVERY>(t)) agg_renorm(g);
            }
            agg_renorm(g);
            float lam = 0.f, eta = 0.f;
            chunk_carry(g, lam, eta);
#pragma unroll 1
            for (int t = 0; t < t_valid; ++t) {
                const float kk = to_f32(sk[t * NSX + n]);
                const float ww = to_f32(sw[t * DPW + dl]);
                readout(t, to_f32(sq[t * NSX + n]),
                        filter_token(lam, eta, a, p, (kk * kk) * ww, (kk * ww) * to_f32(sv[t * DPW + dl])));
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage_s]);
            final_state(lam, eta);
        }
    }
}

// ---------------------------------------------------------------------------
// One decode token of the layer: the recurrent counterpart of the kernel
// above (as kla_step_*_kernel is of the scan).  Grid y runs over the B H
// (sequence, head) rows, grid x over the D Ns state channels of a row, one
// thread per channel c = d Ns + n; a warp holds 32 / Ns whole value
// coordinates (D Ns is a multiple of 32), so the readout reduces over lanes
// as above.  No index division in the loop.
struct LayerStepParams {
    const void *k, *q;             // [B, H, Ns] this token's operators
    const void *v, *w;             // [B, H, D] this token's values and precisions
    const float *a, *p;            // [H, D, Ns]
    float *lam, *eta;              // [B, H, D, Ns] state, in place
    float *y, *s;                  // [B, H, D]; s may be null
    int64_t BH;                    // B H rows
    int H, D, DN;                  // DN = D Ns
};

template <typename Tin, int NSX>
__global__ void __launch_bounds__(256) kla_layer_step_kernel(const LayerStepParams prm) {
    grid_dependency_wait();
    allow_dependent_launch();
    const int c = blockIdx.x * blockDim.x + threadIdx.x;    // channel within the row
    if (c >= prm.DN) return;                                // whole warps (DN is a multiple of 32)
    const int n = c % NSX;
    const int d = c / NSX;
    const Tin *kg = static_cast<const Tin *>(prm.k);
    const Tin *qg = static_cast<const Tin *>(prm.q);
    const Tin *vg = static_cast<const Tin *>(prm.v);
    const Tin *wg = static_cast<const Tin *>(prm.w);
    for (int64_t bh = blockIdx.y; bh < prm.BH; bh += gridDim.y) {
        const int h = (int)((unsigned)bh % (unsigned)prm.H);   // B H < 2^31
        const int64_t row = bh * prm.DN + c;                 // [B, H, D, Ns] index
        const int64_t vd = bh * prm.D + d;                   // [B, H, D] index
        const float kk = to_f32(kg[bh * NSX + n]);
        const float qq = to_f32(qg[bh * NSX + n]);
        const float ww = to_f32(wg[vd]);
        const float vv = to_f32(vg[vd]);
        const int pc = h * prm.DN + c;
        float lam = prm.lam[row], eta = prm.eta[row];
        const TokenOut o = filter_token(lam, eta, prm.a[pc], prm.p[pc], (kk * kk) * ww, (kk * ww) * vv);
        prm.lam[row] = lam;
        prm.eta[row] = eta;
        float ym = qq * o.mu;
        float sv2 = (qq * qq) * o.var;
#pragma unroll
        for (int off = NSX / 2; off >= 1; off >>= 1) {
            ym += __shfl_xor_sync(0xffffffffu, ym, off);
            sv2 += __shfl_xor_sync(0xffffffffu, sv2, off);
        }
        if (n == 0) {
            prm.y[vd] = ym;
            if (prm.s) prm.s[vd] = sv2;
        }
    }
}

}  // namespace kla
