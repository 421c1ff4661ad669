// kla_forward_wide.cuh -- the forward scan for problems with many channels
// (sm_100a).
//
// When the channels alone give every SM several warps of work, the scan
// needs no token-parallel machinery at all: one warp walks VEC x 32
// consecutive channels of one batch row through the whole sequence, lane =
// VEC channels, applying the plain per-token recursion of kla_device.cuh
// (filter_token) token after token.  Each lane thus runs VEC independent
// recursion chains side by side, its loads of a, p, phi, b and its streaming
// stores of lambda, eta, mu, var are 4 x VEC bytes wide (fully used 128-byte
// lines across the warp), and the loads of D tokens are issued before their
// arithmetic so that D x 4 x 32 x VEC x elem bytes per warp are in flight.
// There is no chunk aggregate, no carry, no shared memory and no wait: per
// token-channel it issues roughly a quarter of the instructions of the
// chunked kernels, and every byte crosses HBM once.  The results are the
// per-token recursion from the prior, exactly as the other kernels' second
// pass computes it.
#pragma once

#include "kla_device.cuh"

namespace kla {

struct WideParams {
    const void *in[4];             // a, p, phi, b [B, T, H, N]
    const float *lam0, *eta0;      // [B, H, N]
    float *out[4];                 // lambda, eta, mu, var; mu / var may be null
    int64_t T, HN;
    int64_t nwt;                   // warp tiles (of 32 x VEC channels) per batch row
    int64_t nunits;                // B * nwt
};

// VEC consecutive values of an input at element index i (i a multiple of
// VEC), widened to fp32; streaming (evict-first) loads.
template <typename Tin, int VEC> struct WideLd;
template <> struct WideLd<float, 4> {
    static __device__ __forceinline__ void load(const void *p, int64_t i, float (&v)[4]) {
        const float4 x = __ldcs(reinterpret_cast<const float4 *>(static_cast<const float *>(p) + i));
        v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
    }
};
template <> struct WideLd<float, 2> {
    static __device__ __forceinline__ void load(const void *p, int64_t i, float (&v)[2]) {
        const float2 x = __ldcs(reinterpret_cast<const float2 *>(static_cast<const float *>(p) + i));
        v[0] = x.x; v[1] = x.y;
    }
};
template <> struct WideLd<__nv_bfloat16, 4> {
    static __device__ __forceinline__ void load(const void *p, int64_t i, float (&v)[4]) {
        const uint2 u = __ldcs(reinterpret_cast<const uint2 *>(static_cast<const __nv_bfloat16 *>(p) + i));
        v[0] = __uint_as_float(u.x << 16); v[1] = __uint_as_float(u.x & 0xffff0000u);
        v[2] = __uint_as_float(u.y << 16); v[3] = __uint_as_float(u.y & 0xffff0000u);
    }
};
template <> struct WideLd<__nv_bfloat16, 2> {
    static __device__ __forceinline__ void load(const void *p, int64_t i, float (&v)[2]) {
        const unsigned u = __ldcs(reinterpret_cast<const unsigned *>(static_cast<const __nv_bfloat16 *>(p) + i));
        v[0] = __uint_as_float(u << 16); v[1] = __uint_as_float(u & 0xffff0000u);
    }
};

template <int VEC> struct WideSt;
template <> struct WideSt<4> {
    static __device__ __forceinline__ void store(float *p, int64_t i, const float (&v)[4]) {
        __stcs(reinterpret_cast<float4 *>(p + i), make_float4(v[0], v[1], v[2], v[3]));
    }
};
template <> struct WideSt<2> {
    static __device__ __forceinline__ void store(float *p, int64_t i, const float (&v)[2]) {
        __stcs(reinterpret_cast<float2 *>(p + i), make_float2(v[0], v[1]));
    }
};

// One warp per (batch row, tile of 32 x VEC channels); WARPS warps per CTA.
// Needs H*N % VEC == 0 and every array aligned to 4 x VEC bytes (2 x VEC for
// bf16 inputs).
template <typename Tin, int VEC, int D, int WARPS>
__global__ void __launch_bounds__(32 * WARPS) kla_forward_wide_kernel(const WideParams prm) {
    const int64_t unit = (int64_t)blockIdx.x * WARPS + (threadIdx.x >> 5);
    if (unit >= prm.nunits) return;
    const int lane = threadIdx.x & 31;
    const int64_t bb = unit / prm.nwt;
    const int64_t c = (unit - bb * prm.nwt) * (32 * VEC) + lane * VEC;
    if (c >= prm.HN) return;  // whole vectors: H*N is a multiple of VEC
    float lam[VEC], eta[VEC];
#pragma unroll
    for (int v = 0; v < VEC; ++v) {  // the prior: scalar loads (its alignment is not checked)
        lam[v] = prm.lam0[bb * prm.HN + c + v];
        eta[v] = prm.eta0[bb * prm.HN + c + v];
    }
    const int64_t base = bb * prm.T * prm.HN + c;
    float *const lo = prm.out[0], *const eo = prm.out[1], *const mo = prm.out[2], *const vo = prm.out[3];
#pragma unroll 1
    for (int64_t t0 = 0; t0 < prm.T; t0 += D) {
        const int n = (int)(prm.T - t0 < D ? prm.T - t0 : D);
        float xa[D][VEC], xp[D][VEC], xf[D][VEC], xb[D][VEC];
#pragma unroll
        for (int u = 0; u < D; ++u) {
            if (u < n) {
                const int64_t i = base + (t0 + u) * prm.HN;
                WideLd<Tin, VEC>::load(prm.in[0], i, xa[u]);
                WideLd<Tin, VEC>::load(prm.in[1], i, xp[u]);
                WideLd<Tin, VEC>::load(prm.in[2], i, xf[u]);
                WideLd<Tin, VEC>::load(prm.in[3], i, xb[u]);
            }
        }
#pragma unroll
        for (int u = 0; u < D; ++u) {
            if (u < n) {
                float ol[VEC], oe[VEC], om[VEC], ov[VEC];
#pragma unroll
                for (int v = 0; v < VEC; ++v) {
                    const TokenOut o = filter_token(lam[v], eta[v], xa[u][v], xp[u][v], xf[u][v], xb[u][v]);
                    ol[v] = o.lam; oe[v] = o.eta; om[v] = o.mu; ov[v] = o.var;
                }
                const int64_t i = base + (t0 + u) * prm.HN;
                WideSt<VEC>::store(lo, i, ol);
                WideSt<VEC>::store(eo, i, oe);
                if (mo != nullptr) WideSt<VEC>::store(mo, i, om);
                if (vo != nullptr) WideSt<VEC>::store(vo, i, ov);
            }
        }
    }
}

}  // namespace kla
