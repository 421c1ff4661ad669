// kla_forward_wide.cuh -- the forward scan for problems with many channels
// (sm_100a).
//
// When the channels alone give every SM several warps of work, the scan
// needs no token-parallel machinery: one warp walks a tile of CW channels of
// one batch row through the whole sequence with the plain per-token
// recursion of kla_device.cuh (filter_token), lane = channel.  Without chunk
// aggregates or carries, a token costs one pass instead of the chunked
// kernels' two.
//
// What such a kernel needs is bytes in flight: a warp streams its tile
// through its own ring of NSTG shared-memory stages of L tokens, each filled
// by TMA bulk-tensor loads (box {CW, L, 1} of a, p, phi, b) that lane 0
// issues NSTG chunks ahead and that complete on the stage's mbarrier.  After
// a chunk's L tokens the warp refills the stage with the chunk NSTG ahead of
// it in its own sequence of (unit, chunk) items.  Outputs leave as direct
// coalesced stores from registers (CW x 4 bytes per output and token).
//
// CW is 32 (fp32 inputs: a 128-byte row per input and token) or 16 (bf16
// inputs: 32 bytes, one sector, so that a batch of B x H*N / 16 tiles still
// gives every SM its warps); with CW = 16 the upper half-warp idles, which
// costs issue slots the kernel has to spare.  Units (batch row, channel
// tile) are dealt to the grid's CTAs round-robin and, inside a CTA, to its
// warps; rows past T arrive as zeros from TMA and are not stored; lanes past
// H*N load zeros and store nothing.  Every wait is bounded.
#pragma once

#include "kla_forward_stream.cuh"

namespace kla {

struct WideParams {
    const float *lam0, *eta0;      // [B, H, N]
    float *out[4];                 // lambda, eta, mu, var; mu / var may be null
    int64_t T, HN;
    int64_t ntile;                 // channel tiles per batch row: ceil(HN / CW)
    int64_t nunits;                // B * ntile
    int nchunks;                   // ceil(T / L)
    uint64_t wait_ns;
};

template <typename Tin, int CW, int L, int NSTG, int NWARP>
struct WideTile {
    static constexpr int STAGE_BYTES = 4 * L * CW * (int)sizeof(Tin);  // [4][L][CW]
    static_assert(STAGE_BYTES % 128 == 0, "stages stay 128-byte aligned");
    static constexpr int WARP_BYTES = NSTG * STAGE_BYTES;
    static constexpr int BAR_OFF = NWARP * WARP_BYTES;                // [NWARP][NSTG] mbarriers
    static constexpr int SMEM = align_up(BAR_OFF + NWARP * NSTG * 8, 128);
};

template <typename Tin, int CW, int L, int NSTG, int NWARP>
__global__ void __launch_bounds__(32 * NWARP, 1)
kla_forward_wide_kernel(const WideParams prm, const __grid_constant__ FwdMaps maps) {
    using Cfg = WideTile<Tin, CW, L, NSTG, NWARP>;
    extern __shared__ __align__(128) unsigned char smem[];
    const int w = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    unsigned char *ring = smem + w * Cfg::WARP_BYTES;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + Cfg::BAR_OFF) + w * NSTG;
    if (lane == 0) {
        for (int s = 0; s < NSTG; ++s) mbar_init(&full[s], 1);
        fence_mbar_init();
    }
    __syncwarp();

    // This warp's units: u = blockIdx.x + gridDim.x * (w + NWARP * k), k = 0, 1, ...
    const int64_t ustep = (int64_t)gridDim.x * NWARP;
    const int64_t ufirst = blockIdx.x + (int64_t)gridDim.x * w;
    // item i of the warp = chunk (i % nchunks) of its (i / nchunks)-th unit
    const int64_t nitems = ufirst < prm.nunits ? ((prm.nunits - 1 - ufirst) / ustep + 1) * prm.nchunks : 0;
    auto issue = [&](int64_t item) {  // lane 0: the TMA loads of one item into its stage
        const int64_t u = ufirst + (item / prm.nchunks) * ustep;
        const int chunk = (int)(item % prm.nchunks);
        const int bb = (int)(u / prm.ntile);
        const int ct = (int)(u - (int64_t)bb * prm.ntile);
        const int s = (int)(item % NSTG);
        Tin *stage = reinterpret_cast<Tin *>(ring + s * Cfg::STAGE_BYTES);
        mbar_arrive_expect_tx(&full[s], (unsigned)Cfg::STAGE_BYTES);
#pragma unroll
        for (int q = 0; q < 4; ++q)
            tma_load_3d(stage + q * L * CW, &maps.in[q], ct * CW, chunk * L, bb, &full[s]);
    };
    if (lane == 0)
        for (int64_t i = 0; i < NSTG && i < nitems; ++i) issue(i);

    float lam = 0.f, eta = 0.f;
    int64_t chan = 0, row0 = 0;  // this lane's channel and the element index of token 0 of its unit
    bool active = false;
#pragma unroll 1
    for (int64_t item = 0; item < nitems; ++item) {
        const int chunk = (int)(item % prm.nchunks);
        if (chunk == 0) {  // a new unit: its prior
            const int64_t u = ufirst + (item / prm.nchunks) * ustep;
            const int64_t bb = u / prm.ntile;
            const int64_t ct = u - bb * prm.ntile;
            chan = ct * CW + lane;
            active = lane < CW && chan < prm.HN;
            row0 = bb * prm.T * prm.HN + chan;
            lam = active ? prm.lam0[bb * prm.HN + chan] : 1.f;
            eta = active ? prm.eta0[bb * prm.HN + chan] : 0.f;
        }
        const int s = (int)(item % NSTG);
        mbar_wait_or_flag(&full[s], (unsigned)((item / NSTG) & 1), prm.wait_ns);
        const Tin *stage = reinterpret_cast<const Tin *>(ring + s * Cfg::STAGE_BYTES);
        const int64_t t0 = (int64_t)chunk * L;
        const int nv = (int)(prm.T - t0 < L ? prm.T - t0 : L);
        const int c = lane < CW ? lane : 0;  // idle lanes of a half warp read lane 0's column
        float *o0 = prm.out[0] + row0 + t0 * prm.HN;
        float *o1 = prm.out[1] + row0 + t0 * prm.HN;
        float *o2 = prm.out[2] ? prm.out[2] + row0 + t0 * prm.HN : nullptr;
        float *o3 = prm.out[3] ? prm.out[3] + row0 + t0 * prm.HN : nullptr;
#pragma unroll 4
        for (int t = 0; t < nv; ++t) {
            const int i = t * CW + c;
            const TokenOut o = filter_token(lam, eta, to_f32(stage[i]), to_f32(stage[L * CW + i]),
                                            to_f32(stage[2 * L * CW + i]), to_f32(stage[3 * L * CW + i]));
            if (active) {
                const int64_t off = (int64_t)t * prm.HN;
                __stcs(o0 + off, o.lam);
                __stcs(o1 + off, o.eta);
                if (o2) __stcs(o2 + off, o.mu);
                if (o3) __stcs(o3 + off, o.var);
            }
        }
        __syncwarp();  // every lane has read the stage
        if (lane == 0 && item + NSTG < nitems) {
            fence_proxy_async_smem();  // the warp's reads of the stage before the copy that refills it
            issue(item + NSTG);
        }
    }
}

}  // namespace kla
