// kla_device.cuh -- device-side building blocks of the KLA filter kernels
// (sm_100a): the projective 3x3 chunk aggregate, bounded waits, and thin
// inline-PTX wrappers for mbarriers, TMA bulk-tensor copies and
// acquire/release flags.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

namespace kla {

// ---------------------------------------------------------------------------
// Error word shared by all kernels of this library on one device.  Bit 0: a
// bounded wait ran out.  Read and cleared by kla_get_error().
// ---------------------------------------------------------------------------
enum : unsigned { DEV_ERR_TIMEOUT = 1u };

// This header is compiled into exactly one translation unit (kla.cu), which
// owns these two words: the error word, and a word that stays zero (the
// target of the failure-path test hooks).
__device__ unsigned g_error_word;
__device__ unsigned g_never_set_word;

// ---------------------------------------------------------------------------
// The chunk aggregate.
//
// One token of the filter acts on the homogeneous state (n, d, h), with
// lambda = n / d and eta = h / d, through the block-lower-triangular matrix
//
//   G_t = [[ 1 + p phi,  a^2 phi, 0 ],
//          [ p,          a^2,     0 ],
//          [ b p,        b a^2,   a ]].
//
// Its top-left 2x2 block is the Moebius matrix M_t of the precision map (Pith
// review of "Kalman Linear Attention", "What carries the argument"); the last
// row carries the gated affine information-mean recursion eta_t = f_t
// eta_{t-1} + b_t with f_t = a_t / (a_t^2 + p_t lambda_{t-1}):
//   h_t / d_t = (b_t d_t + a_t h_{t-1}) / d_t = b_t + a_t eta_{t-1} / (p_t
//   lambda_{t-1} + a_t^2).
// So both recursions of the review (the Moebius scan and the "second",
// affine scan) become ONE associative product of such matrices, and the
// aggregate of a chunk does not depend on the state entering it.  Like M_t
// (defined up to a nonzero scalar, review reference [13]) the aggregate is
// projective: it is rescaled by exact powers of two to stay in range.
// Seven entries are live.
// ---------------------------------------------------------------------------
struct Agg {
    float m11, m12, m21, m22;  // Moebius block
    float g1, g2;              // information row, first two columns
    float A;                   // information row, last column (product of a)
};

__device__ __forceinline__ Agg agg_identity() {
    Agg g;
    g.m11 = 1.f; g.m12 = 0.f; g.m21 = 0.f; g.m22 = 1.f;
    g.g1 = 0.f; g.g2 = 0.f; g.A = 1.f;
    return g;
}

// Rescale by 2^-e so that the largest Moebius entry lies in [1, 2).  A
// multiplication by a power of two is exact, so the represented map -- and
// every later rounding -- is unchanged: how often this runs does not change
// any result bit (barring overflow).  The kernels run it every
// KLA_RENORM_EVERY-th token (2 by default); between two runs the largest
// entry grows at most by the largest row sum of M_t to that power, so
// entries stay finite while 1 + p phi + a^2 phi + p + a^2 < 2^(126 /
// KLA_RENORM_EVERY) per token (2^63 by default).
#ifndef KLA_RENORM_EVERY
#define KLA_RENORM_EVERY 2
#endif
constexpr int kRenormEvery = KLA_RENORM_EVERY;
static_assert(kRenormEvery >= 1 && kRenormEvery <= 8, "renormalisation interval");
__device__ __forceinline__ constexpr bool renorm_after(int t) { return (t + 1) % kRenormEvery == 0; }
// The same with another interval E (E-th powers of the row sums must stay
// below 2^126: row sums below 2^(126 / E) per token).
template <int E>
__device__ __forceinline__ constexpr bool renorm_after_every(int t) { return (t + 1) % E == 0; }
__device__ __forceinline__ void agg_renorm(Agg &g) {
    const float mx = fmaxf(fmaxf(fabsf(g.m11), fabsf(g.m12)), fmaxf(fabsf(g.m21), fabsf(g.m22)));
    int e = (__float_as_int(mx) >> 23) & 0xff;  // biased exponent of the max
    e = min(max(e, 1), 253);
    const float s = __int_as_float((254 - e) << 23);  // 2^(127 - e)
    g.m11 *= s; g.m12 *= s; g.m21 *= s; g.m22 *= s;
    g.g1 *= s; g.g2 *= s; g.A *= s;
}

// g <- G_t * g : append one token (a, p, phi, b) after the span g covers.
// M_t factors as [[1, phi], [0, 1]] * [[1, 0], [p, a^2]]: the predict step
// (the denominator row becomes p n + a^2 d) followed by the update step (the
// numerator row gains phi times the new denominator row) -- the matrix form
// of "prior precision, then add the token's evidence precision".  Six
// multiply-adds instead of ten, all on non-negative numbers.
__device__ __forceinline__ void agg_push_token(Agg &g, float a, float p, float phi, float b) {
    const float a2 = a * a;
    const float d1 = fmaf(p, g.m11, a2 * g.m21);   // predict: denominator row
    const float d2 = fmaf(p, g.m12, a2 * g.m22);
    g.m11 = fmaf(phi, d1, g.m11);                  // update: numerator row
    g.m12 = fmaf(phi, d2, g.m12);
    g.m21 = d1;
    g.m22 = d2;
    g.g1 = fmaf(b, d1, a * g.g1);                  // information row
    g.g2 = fmaf(b, d2, a * g.g2);
    g.A *= a;
}

// X * Y : the span of Y followed by the span of X.
__device__ __forceinline__ Agg agg_compose(const Agg &X, const Agg &Y) {
    Agg r;
    r.m11 = fmaf(X.m11, Y.m11, X.m12 * Y.m21);
    r.m12 = fmaf(X.m11, Y.m12, X.m12 * Y.m22);
    r.m21 = fmaf(X.m21, Y.m11, X.m22 * Y.m21);
    r.m22 = fmaf(X.m21, Y.m12, X.m22 * Y.m22);
    r.g1 = fmaf(X.g1, Y.m11, fmaf(X.g2, Y.m21, X.A * Y.g1));
    r.g2 = fmaf(X.g1, Y.m12, fmaf(X.g2, Y.m22, X.A * Y.g2));
    r.A = X.A * Y.A;
    return r;
}

// Hardware reciprocal (PTX rcp.approx.ftz.f32, one MUFU instruction; the PTX
// ISA bounds its error by 1 ulp for normal inputs).  The filter's state is
// positive and far from the subnormal range under the documented
// preconditions, and its error per token is damped by the contraction of the
// recursion, so this keeps the results well inside the parity tolerance.
__device__ __forceinline__ float rcp_hw(float x) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// State (lambda, eta) after the span of g, entered with (lam, eta).
__device__ __forceinline__ void agg_apply(const Agg &g, float &lam, float &eta) {
    const float n = fmaf(g.m11, lam, g.m12);
    const float d = fmaf(g.m21, lam, g.m22);
    const float h = fmaf(g.g1, lam, fmaf(g.A, eta, g.g2));
    const float rd = rcp_hw(d);
    lam = n * rd;
    eta = h * rd;
}

// One token of the filter in information form, on fp32 state:
//   den = a^2 + p lambda, prior precision lambda / den, gate f = a / den,
//   lambda' = lambda / den + phi, eta' = f eta + b, mu = eta' / lambda',
//   var = 1 / lambda'.
struct TokenOut { float lam, eta, mu, var; };

__device__ __forceinline__ TokenOut filter_token(float &lam, float &eta,
                                                 float a, float p, float phi, float b) {
    const float den = fmaf(p, lam, a * a);
    const float r = rcp_hw(den);
    lam = fmaf(lam, r, phi);
    eta = fmaf(a * r, eta, b);
    const float v = rcp_hw(lam);
    TokenOut o;
    o.lam = lam; o.eta = eta; o.mu = eta * v; o.var = v;
    return o;
}

// ---------------------------------------------------------------------------
// Loads
// ---------------------------------------------------------------------------
template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
    return __bfloat162float(x);
}

// ---------------------------------------------------------------------------
// Programmatic dependent launch
// ---------------------------------------------------------------------------
// A kernel launched with programmatic stream serialization may become
// resident as soon as every CTA of the kernel before it on the stream has
// executed `griddepcontrol.launch_dependents` (or exited); `griddepcontrol.wait`
// then blocks the calling thread until that kernel has completed and its
// writes are visible.  In a kernel launched without the attribute the wait
// returns at once.
__device__ __forceinline__ void grid_dependency_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void allow_dependent_launch() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------------------
// Time and flags
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned *p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release_gpu(unsigned *p, unsigned v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" :: "l"(p), "r"(v) : "memory");
}

// Warp-wide bounded wait: every lane of the warp calls it with its own flag
// pointer (or nullptr for "nothing to wait for"); returns true once every
// lane's flag is nonzero, false when `limit_ns` ran out first.  The final
// __syncwarp orders each lane's acquire before every lane's later loads.
// The iteration cap is a second bound in case the global timer misbehaves.
#ifndef KLA_SPIN_NS_MAX
#define KLA_SPIN_NS_MAX 1024
#endif
__device__ __forceinline__ bool warp_wait_flags(const unsigned *flag, uint64_t limit_ns) {
    const uint64_t t0 = globaltimer_ns();
    unsigned ns = 32;
    for (uint32_t it = 0; it < (1u << 22); ++it) {
        const unsigned v = flag != nullptr ? ld_acquire_gpu(flag) : 1u;
        if (__all_sync(0xffffffffu, v != 0u)) {
            __syncwarp();
            return true;
        }
        const bool late = (globaltimer_ns() - t0) > limit_ns;
        if (__any_sync(0xffffffffu, late)) return false;
        __nanosleep(ns);
        ns = ns < KLA_SPIN_NS_MAX ? ns * 2 : KLA_SPIN_NS_MAX;
    }
    return false;
}

// ---------------------------------------------------------------------------
// mbarrier (shared::cta) and TMA bulk-tensor copies
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, unsigned count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(smem_u32(bar)), "r"(count) : "memory");
}

// Make the initialised barrier visible to the async (TMA) proxy.
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, unsigned bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
                 :: "r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, unsigned parity) {
    uint32_t ok;
    asm volatile("{\n\t.reg .pred P;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 P, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, P;\n\t}"
                 : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    return ok != 0;
}

// Bounded wait for phase `parity` of `bar`; false when `limit_ns` ran out.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, unsigned parity, uint64_t limit_ns) {
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 0; it < (1u << 22); ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if (globaltimer_ns() - t0 > limit_ns) return false;
    }
    return false;
}

// 3-D tiled TMA load global -> shared::cta, completion on `bar`.
__device__ __forceinline__ void tma_load_3d(void *smem_dst, const CUtensorMap *map,
                                            int x, int y, int z, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cta.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];"
        :: "r"(smem_u32(smem_dst)), "l"(reinterpret_cast<uint64_t>(map)),
           "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
        : "memory");
}

// 3-D tiled TMA store shared::cta -> global (bulk async-group completion).
__device__ __forceinline__ void tma_store_3d(const CUtensorMap *map, const void *smem_src,
                                             int x, int y, int z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4}], [%1];"
        :: "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(smem_src)),
           "r"(x), "r"(y), "r"(z)
        : "memory");
}

__device__ __forceinline__ void bulk_commit_group() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Wait until every committed bulk store has finished READING shared memory.
__device__ __forceinline__ void bulk_wait_group_read_all() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// Order this thread's generic-proxy shared-memory writes before later
// async-proxy (TMA) reads of them.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" :: "l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

}  // namespace kla
