// kla_step.cuh -- one recurrent decode token of the KLA filter (sm_100a).
//
// Constant work per token and channel: the running posterior (lambda, eta)
// is a sufficient summary of everything the filter has seen ("Kalman filter"
// primer, section 6.2), so decoding one token is one application of the
// per-token recursion to the resident state.  Purely elementwise and
// HBM-bound: 16 (fp32) or 8 (bf16) bytes of inputs, 8 bytes of state read,
// 8 written, and up to 8 bytes of outputs per channel.
#pragma once

#include "kla_device.cuh"

namespace kla {

struct StepParams {
    const void *in[4];   // a, p, phi, b of this token, [C]
    float *lam, *eta;    // state, [C], in place
    float *mu, *var;     // outputs, [C], may be null
    int64_t C;
};

template <typename Tin> struct Vec4In;
template <> struct Vec4In<float> {
    static __device__ __forceinline__ float4 load(const void *p, int64_t i) {
        return __ldcs(reinterpret_cast<const float4 *>(p) + i);
    }
};
template <> struct Vec4In<__nv_bfloat16> {
    static __device__ __forceinline__ float4 load(const void *p, int64_t i) {
        const uint2 u = __ldcs(reinterpret_cast<const uint2 *>(p) + i);
        float4 f;
        f.x = __uint_as_float(u.x << 16); f.y = __uint_as_float(u.x & 0xffff0000u);
        f.z = __uint_as_float(u.y << 16); f.w = __uint_as_float(u.y & 0xffff0000u);
        return f;
    }
};

// Programmatic dependent launch: the kernel may start while the previous
// kernel on the stream is still running.  Before `griddepcontrol.wait` it only
// prefetches its token inputs into L2 (L2 is the point of coherence, so a
// prefetch can never expose a stale value); every load and store happens
// after the wait, which guarantees that the previous kernel has completed and
// its writes are visible.
__device__ __forceinline__ void prefetch_l2(const void *p) {
    asm volatile("prefetch.global.L2 [%0];" :: "l"(p));
}

// Four channels per thread; every pointer 16-byte aligned (8 for bf16
// inputs) and C a multiple of 4.
template <typename Tin>
__global__ void __launch_bounds__(256) kla_step_vec4_kernel(const StepParams prm) {
    const int64_t n4 = prm.C >> 2;
    constexpr int VEC_BYTES = 4 * (int)sizeof(Tin);
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n4;
         i += (int64_t)gridDim.x * blockDim.x)
        if ((threadIdx.x & 7) == 0)  // one prefetch per 128-byte line (8 threads x 16 bytes, fp32)
#pragma unroll
            for (int k = 0; k < 4; ++k)
                prefetch_l2(static_cast<const char *>(prm.in[k]) + i * VEC_BYTES);
    grid_dependency_wait();
    allow_dependent_launch();
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n4;
         i += (int64_t)gridDim.x * blockDim.x) {
        const float4 a = Vec4In<Tin>::load(prm.in[0], i);
        const float4 p = Vec4In<Tin>::load(prm.in[1], i);
        const float4 phi = Vec4In<Tin>::load(prm.in[2], i);
        const float4 b = Vec4In<Tin>::load(prm.in[3], i);
        float4 lam = reinterpret_cast<const float4 *>(prm.lam)[i];
        float4 eta = reinterpret_cast<const float4 *>(prm.eta)[i];
        const TokenOut o0 = filter_token(lam.x, eta.x, a.x, p.x, phi.x, b.x);
        const TokenOut o1 = filter_token(lam.y, eta.y, a.y, p.y, phi.y, b.y);
        const TokenOut o2 = filter_token(lam.z, eta.z, a.z, p.z, phi.z, b.z);
        const TokenOut o3 = filter_token(lam.w, eta.w, a.w, p.w, phi.w, b.w);
        reinterpret_cast<float4 *>(prm.lam)[i] = lam;
        reinterpret_cast<float4 *>(prm.eta)[i] = eta;
        if (prm.mu != nullptr)
            __stcs(reinterpret_cast<float4 *>(prm.mu) + i, make_float4(o0.mu, o1.mu, o2.mu, o3.mu));
        if (prm.var != nullptr)
            __stcs(reinterpret_cast<float4 *>(prm.var) + i, make_float4(o0.var, o1.var, o2.var, o3.var));
    }
}

// Any size and alignment: one channel per thread.
template <typename Tin>
__global__ void __launch_bounds__(256) kla_step_scalar_kernel(const StepParams prm) {
    grid_dependency_wait();
    allow_dependent_launch();
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < prm.C;
         i += (int64_t)gridDim.x * blockDim.x) {
        const float a = to_f32(static_cast<const Tin *>(prm.in[0])[i]);
        const float p = to_f32(static_cast<const Tin *>(prm.in[1])[i]);
        const float phi = to_f32(static_cast<const Tin *>(prm.in[2])[i]);
        const float b = to_f32(static_cast<const Tin *>(prm.in[3])[i]);
        float lam = prm.lam[i], eta = prm.eta[i];
        const TokenOut o = filter_token(lam, eta, a, p, phi, b);
        prm.lam[i] = lam;
        prm.eta[i] = eta;
        if (prm.mu != nullptr) prm.mu[i] = o.mu;
        if (prm.var != nullptr) prm.var[i] = o.var;
    }
}

}  // namespace kla
