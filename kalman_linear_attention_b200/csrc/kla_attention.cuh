// kla_attention.cuh -- the Kalman attention weights of the information mean
// (sm_100a).
//
// Between two tokens s <= t of one channel the information mean of the later
// token responds to the earlier one through the gates between them: the
// affine recursion eta_k = f_k eta_{k-1} + b_k (KLA review, "Core claim")
// unrolls into
//
//   eta_t = F(t, s) eta_s + sum_{r = s+1..t} F(t, r) b_r,
//   F(t, s) = prod_{k = s+1..t} f_k,   f_k = a_k / (a_k^2 + p_k lambda_{k-1}),
//
// a lower-triangular matrix of weights per channel -- the review's "Kalman
// Attention Matrix" (minor comment on its App. E.3/E.4).  By the telescoping
// denominators of the Moebius product it also equals prod(a) / (C lambda_s +
// D) with [[A, B], [C, D]] = M_t ... M_{s+1}.
//
// One CTA owns one window of W tokens of one batch row and a tile of 32 x VEC
// channels.  Its threads first form the window's gates from a, p and the
// forward scan's stored lambda (one reciprocal per token and channel, into
// shared memory); then each warp writes whole columns s of the W x W matrix,
// lane = VEC channels: the running product down the column is one multiply
// per entry, and every entry, the zeros above the diagonal included, leaves
// with one streaming store of 16 bytes (VEC = 4) per lane.  Output traffic
// (W^2 floats per channel and window) dominates: the kernel is bound by HBM
// writes.
#pragma once

#include "kla_device.cuh"

namespace kla {

struct AttnParams {
    const void *a, *p;             // [B, T, H, N], input dtype
    const float *lam;              // [B, T, H, N] posterior precision of the forward scan
    float *F;                      // [B, nwin, W, W, H, N]
    int64_t T, HN;
    int64_t t0, span;              // tokens [t0, t0 + span), cut into windows of W
    int W, nwin;
    int64_t nct;                   // channel tiles (of 32 x VEC) per batch row
};

// VEC consecutive floats: streaming (evict-first) global store, shared load.
__device__ __forceinline__ void st_cs_vec(float *dst, const float (&v)[1]) { __stcs(dst, v[0]); }
__device__ __forceinline__ void st_cs_vec(float *dst, const float (&v)[4]) {
    __stcs(reinterpret_cast<float4 *>(dst), make_float4(v[0], v[1], v[2], v[3]));
}
__device__ __forceinline__ void lds_vec(float (&v)[1], const float *src) { v[0] = *src; }
__device__ __forceinline__ void lds_vec(float (&v)[4], const float *src) {
    const float4 x = *reinterpret_cast<const float4 *>(src);
    v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
}

// Grid: one CTA per (batch row, window, channel tile), flattened on x as
// ((b * nwin) + window) * nct + tile.  Dynamic shared memory: W * 32 * VEC
// floats of gates.
template <typename Tin, int VEC>
__global__ void __launch_bounds__(256) kla_attention_kernel(const AttnParams prm) {
    constexpr int CW = 32 * VEC;
    extern __shared__ __align__(16) float gates[];  // [W][CW]
    const int64_t cta = blockIdx.x;
    const int64_t tile = cta % prm.nct;
    const int64_t bw = cta / prm.nct;
    const int win = (int)(bw % prm.nwin);
    const int64_t bb = bw / prm.nwin;
    const int64_t start = prm.t0 + (int64_t)win * prm.W;
    const int64_t left = prm.t0 + prm.span - start;
    const int nv = (int)(left < (int64_t)prm.W ? left : (int64_t)prm.W);  // tokens of this window in the span
    const int64_t c0 = tile * CW;
    const Tin *ag = static_cast<const Tin *>(prm.a);
    const Tin *pg = static_cast<const Tin *>(prm.p);

    // 1) the gate of every window token after the first (the first one's is
    //    never used: F(t, s) takes the gates of tokens s+1..t); each thread
    //    issues the loads of GU elements before their arithmetic
    constexpr int GU = 8;
    for (int base = threadIdx.x; base < nv * CW; base += GU * blockDim.x) {
        float av[GU], pv[GU], lv[GU];
#pragma unroll
        for (int u = 0; u < GU; ++u) {
            const int idx = base + u * blockDim.x;
            const int k = idx / CW;
            const int c = idx - k * CW;
            av[u] = 0.f; pv[u] = 1.f; lv[u] = 1.f;  // an unused gate: 0
            if (idx < nv * CW && k >= 1 && c0 + c < prm.HN) {
                const int64_t row = (bb * prm.T + start + k) * prm.HN + c0 + c;
                av[u] = to_f32(ag[row]);
                pv[u] = to_f32(pg[row]);
                lv[u] = __ldg(prm.lam + row - prm.HN);  // lambda_{k-1}: this channel, previous token
            }
        }
#pragma unroll
        for (int u = 0; u < GU; ++u) {
            const int idx = base + u * blockDim.x;
            if (idx < nv * CW) gates[idx] = av[u] * rcp_hw(fmaf(pv[u], lv[u], av[u] * av[u]));
        }
    }
    __syncthreads();

    // 2) columns: warp w writes columns w, w + nwarps, ...; every column holds
    //    W entries, so the stores are balanced across warps
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int nwarps = blockDim.x >> 5;
    const bool cvalid = c0 + lane * VEC < prm.HN;  // VEC = 4 needs H*N % 4 == 0: whole vectors
    const int64_t WW = (int64_t)prm.W * prm.W;
    float *Fcta = prm.F + ((bb * prm.nwin + win) * WW) * prm.HN + c0 + lane * VEC;
    const float *glane = gates + lane * VEC;
    const int64_t row_step = (int64_t)prm.W * prm.HN;  // elements from row i to row i + 1 of a column
#pragma unroll 1
    for (int j = warp; j < prm.W; j += nwarps) {
        if (!cvalid) continue;
        float f[VEC];
#pragma unroll
        for (int v = 0; v < VEC; ++v) f[v] = 1.f;
        const float zero[VEC] = {};
        float *dst = Fcta + (int64_t)j * prm.HN;
        // rows above the diagonal (and the whole column past the span): zeros
        const int lo = j < nv ? j : prm.W;
#pragma unroll 4
        for (int i = 0; i < lo; ++i, dst += row_step) st_cs_vec(dst, zero);
        if (j >= nv) continue;
        // the diagonal, then the running product of the gates down the column
        st_cs_vec(dst, f);
        dst += row_step;
#pragma unroll 4
        for (int i = j + 1; i < nv; ++i, dst += row_step) {
            float g[VEC];
            lds_vec(g, glane + i * CW);
#pragma unroll
            for (int v = 0; v < VEC; ++v) f[v] *= g[v];
            st_cs_vec(dst, f);
        }
        // rows past the span
#pragma unroll 4
        for (int i = nv; i < prm.W; ++i, dst += row_step) st_cs_vec(dst, zero);
    }
}

}  // namespace kla
