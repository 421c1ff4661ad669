// kla.cu -- host side of the C ABI declared in include/kla.h: argument
// checks, workspace layout, TMA tensor maps and kernel launches.  Every step
// of the filter and of its gradients runs in the kernels of kla_forward.cuh,
// kla_forward_stream.cuh, kla_step.cuh and kla_backward.cuh; this file only
// validates, describes memory and launches.
#include "kla.h"

#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <set>
#include <utility>

#include "kla_backward.cuh"
#include "kla_forward.cuh"
#include "kla_forward_stream.cuh"
#include "kla_attention.cuh"
#include "kla_layer.cuh"
#include "kla_lti.cuh"
#include "kla_step.cuh"

#define KLA_API extern "C" __attribute__((visibility("default")))

namespace {

using kla::FwdMaps;
using kla::FwdParams;
using kla::StepParams;

// Tile geometry of the forward scan: L tokens x CW channels per CTA, R rows
// of threads (S = L / R tokens per thread).
// (Overridable at build time for tuning sweeps.)
#ifndef KLA_TILE_L
#define KLA_TILE_L 64
#endif
#ifndef KLA_TILE_CW
#define KLA_TILE_CW 64
#endif
#ifndef KLA_TILE_R
#define KLA_TILE_R 4
#endif
#ifndef KLA_CKPT
#define KLA_CKPT 8
#endif
constexpr int kL = KLA_TILE_L;
constexpr int kCW = KLA_TILE_CW;
constexpr int kR = KLA_TILE_R;
constexpr int kNW = kCW / 32;
// Checkpoint interval of the cross-chunk carry, in chunks (<= 32: one lane
// of the look-back warp per flag).
constexpr int kCkpt = KLA_CKPT;
static_assert(kCkpt >= 1 && kCkpt <= 32, "checkpoint interval must be 1..32");

// Channel-owning streaming kernel: chunk length, chunk warps, output group,
// ring stages.  The chunk warps hold a whole chunk in registers (4 x L floats
// per thread); up to 12 warps = 3 per SM sub-partition allow 168 registers
// per thread.
#ifndef KLA_STREAM_L
#define KLA_STREAM_L 32
#endif
// Chunk warps: 6 for fp32 (7 warps in all, up to 255 registers per thread,
// a 10-stage ring of 16 KB stages); measured on the long workload against 5,
// 7 and 9 chunk warps on the same GPU: 6 was 3-7% faster than each.  7 for
// bf16 (8 KB stages, a 21-stage ring): on the LM-layer shape 2.7% faster than
// 11 warps at 168 registers, and 6 or 8 were slower.
#ifndef KLA_STREAM_W_F32
#define KLA_STREAM_W_F32 6
#endif
#ifndef KLA_STREAM_W_BF16
#define KLA_STREAM_W_BF16 7
#endif
// Tokens per output box (one TMA store per output per box): 8 (measured 4-6%
// faster than 4 on the long workload, and with 7 bf16 chunk warps 18% faster
// than 4 on the LM-layer shape; same-box A/B).
#ifndef KLA_STREAM_G_F32
#define KLA_STREAM_G_F32 8
#endif
#ifndef KLA_STREAM_G_BF16
#define KLA_STREAM_G_BF16 8
#endif
#ifndef KLA_STREAM_SMEM
#define KLA_STREAM_SMEM (227 * 1024)
#endif
#ifndef KLA_STREAM_MAX_STAGES
#define KLA_STREAM_MAX_STAGES 24
#endif
constexpr int kSL = KLA_STREAM_L;
template <typename Tin> constexpr int stream_warps() {
    return sizeof(Tin) == 4 ? KLA_STREAM_W_F32 : KLA_STREAM_W_BF16;
}
template <typename Tin> constexpr int stream_group() {
    return sizeof(Tin) == 4 ? KLA_STREAM_G_F32 : KLA_STREAM_G_BF16;
}
// Two channels per lane (bf16 inputs with H*N >= 64): 64-channel tiles of
// KLA_STREAM2_L-token chunks (the same registers per thread as 32 tokens x
// one channel), chunk warps and output group.  On the LM-layer shape: 5%
// faster than one channel per lane with 8-token output groups, no faster
// with 4, slower with 6 chunk warps; one 16-token group per chunk in a
// single buffer (KLA_STREAM2_NBUF, half the bulk stores) 2% faster than two
// double-buffered 8-token groups.
#ifndef KLA_STREAM2_L
#define KLA_STREAM2_L 16
#endif
#ifndef KLA_STREAM2_W
#define KLA_STREAM2_W 7
#endif
#ifndef KLA_STREAM2_G
#define KLA_STREAM2_G 16
#endif
template <typename Tin> constexpr int stream2_warps() { return KLA_STREAM2_W; }
template <typename Tin> constexpr int stream2_group() { return KLA_STREAM2_G; }
// 1 disables the two-channel layout (sweeps)
#ifndef KLA_STREAM2_OFF
#define KLA_STREAM2_OFF 0
#endif


// Ring stages that fit beside the per-warp output buffers and carry slots.
template <typename Tin, int VEC = 1>
constexpr int stream_stages() {
    constexpr int W = VEC == 1 ? stream_warps<Tin>() : stream2_warps<Tin>();
    constexpr int G = VEC == 1 ? stream_group<Tin>() : stream2_group<Tin>();
    constexpr int L = VEC == 1 ? kSL : KLA_STREAM2_L;
    constexpr int CW = 32 * VEC;
    const int stage = 4 * L * CW * (int)sizeof(Tin);
    constexpr int NBUF = VEC == 1 ? KLA_STREAM_NBUF : KLA_STREAM2_NBUF;
    const int fixed = W * NBUF * 4 * G * CW * 4 + W * 2 * CW * 4 + W * 8 + 2048;
    const int ns = (KLA_STREAM_SMEM - fixed) / stage;
    return ns > KLA_STREAM_MAX_STAGES ? KLA_STREAM_MAX_STAGES : ns;
}

// 0: choose by shape; 1: the chunked kernel with cross-CTA carries; 2: the
// channel-owning streaming kernel (test hook kla_debug_force_forward_kernel).
std::atomic<int> g_force_kernel{0};


constexpr size_t kHeaderBytes = 256;  // ticket counter + padding
constexpr int kMaxGrid = 0x7fffffff;

std::atomic<uint64_t> g_wait_ns{1000000000ull};
std::atomic<int64_t> g_stall_chunk{-1};

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool mul_ok(int64_t a, int64_t b, int64_t *out) {
    if (a < 0 || b < 0) return false;
    if (a != 0 && b > INT64_MAX / a) return false;
    *out = a * b;
    return true;
}

size_t dtype_size(kla_dtype_t d) { return d == KLA_BF16 ? 2 : 4; }

bool dtype_ok(kla_dtype_t d) { return d == KLA_F32 || d == KLA_BF16; }

struct Range {
    uintptr_t lo, hi;
};

bool overlaps(const Range &x, const Range &y) {
    return x.lo < y.hi && y.lo < x.hi;
}

// Any two of `outs` overlap, or any output overlaps any input.
bool any_overlap(const Range *outs, int n_out, const Range *ins, int n_in) {
    for (int i = 0; i < n_out; ++i) {
        if (outs[i].lo == outs[i].hi) continue;
        for (int j = i + 1; j < n_out; ++j)
            if (outs[j].lo != outs[j].hi && overlaps(outs[i], outs[j])) return true;
        for (int j = 0; j < n_in; ++j)
            if (ins[j].lo != ins[j].hi && overlaps(outs[i], ins[j])) return true;
    }
    return false;
}

Range range_of(const void *p, int64_t bytes) {
    const uintptr_t lo = reinterpret_cast<uintptr_t>(p);
    return Range{lo, p ? lo + (uintptr_t)bytes : lo};
}

// Workspace layout of one forward call.
struct FwdLayout {
    int64_t nct = 0, nchunks = 0, tiles = 0;
    size_t flags_off = 0, agg_off = 0, incl_off = 0, clear_bytes = 0, total = 0;
};

bool fwd_layout(int64_t B, int64_t T, int64_t HN, FwdLayout *lay) {
    lay->nct = (HN + kCW - 1) / kCW;
    lay->nchunks = (T + kL - 1) / kL;
    int64_t bt = 0, tiles = 0;
    if (!mul_ok(B, lay->nct, &bt) || !mul_ok(bt, lay->nchunks, &tiles)) return false;
    if (tiles > kMaxGrid) return false;
    lay->tiles = tiles;
    lay->flags_off = kHeaderBytes;
    const size_t flags_bytes = round_up((size_t)tiles * kNW * sizeof(unsigned), 256);
    lay->agg_off = lay->flags_off + flags_bytes;
    lay->incl_off = lay->agg_off + round_up((size_t)tiles * 7 * kCW * sizeof(float), 256);
    lay->total = lay->incl_off + round_up((size_t)tiles * 2 * kCW * sizeof(float), 256);
    lay->clear_bytes = kHeaderBytes + flags_bytes;
    return true;
}

// ---- TMA tensor maps --------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
        cudaGetLastError();
    });
    return fn;
}

// [B, T, HN] tensor viewed as dims {HN, T, B}, box {kCW, kL, 1}.
bool encode_map(CUtensorMap *m, const void *base, CUtensorMapDataType dt, size_t esz,
                int64_t B, int64_t T, int64_t HN) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)HN, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t strides[2] = {(cuuint64_t)(HN * esz), (cuuint64_t)(T * HN * esz)};
    const cuuint32_t box[3] = {(cuuint32_t)kCW, (cuuint32_t)kL, 1u};
    const cuuint32_t estr[3] = {1u, 1u, 1u};
    return fn(m, dt, 3, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ---- per-device launch attributes ------------------------------------------
template <typename K>
cudaError_t ensure_smem_attr(K kernel, int smem) {
    static std::mutex mu;
    static std::set<std::pair<int, const void *>> done;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const auto key = std::make_pair(dev, reinterpret_cast<const void *>(kernel));
    std::lock_guard<std::mutex> lock(mu);
    if (done.count(key)) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e == cudaSuccess) done.insert(key);
    return e;
}

// Launch of a scan kernel that follows a workspace clear on the stream.  With
// `after_clear` it is the clear kernel's programmatic dependent: it becomes
// resident while the clear runs, and its griddepcontrol.wait (which every
// kernel launched this way executes before it touches the workspace) holds it
// until the clear is done.  Everything before the clear on the stream has
// completed by the time the clear starts, so the scan's inputs are ready.
template <typename... P, typename... A>
cudaError_t launch_scan_kernel(void (*kernel)(P...), int64_t grid, int threads, size_t smem,
                               cudaStream_t stream, bool after_clear, A &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3((unsigned)threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = after_clear ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<A>(args)...);
}

template <typename Tin, bool TMA>
cudaError_t launch_forward(const FwdParams &prm, const FwdMaps &maps, int64_t tiles,
                           cudaStream_t stream) {
    using Cfg = kla::FwdTile<Tin, kL, kCW, kR>;
    auto kernel = kla::kla_forward_kernel<Tin, kL, kCW, kR, TMA>;
    cudaError_t e = ensure_smem_attr(kernel, Cfg::SMEM);
    if (e != cudaSuccess) return e;
    return launch_scan_kernel(kernel, tiles, Cfg::THREADS, Cfg::SMEM, stream, true, prm, maps);
}

int sm_count() {
    static std::mutex mu;
    static int count[256] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 256) return 148;
    std::lock_guard<std::mutex> lock(mu);
    if (count[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        count[dev] = n;
    }
    return count[dev];
}

template <typename Tin, int VEC = 1>
cudaError_t launch_forward_stream(const kla::StreamParams &prm, const FwdMaps &maps, cudaStream_t stream) {
    constexpr int W = VEC == 1 ? stream_warps<Tin>() : stream2_warps<Tin>();
    constexpr int G = VEC == 1 ? stream_group<Tin>() : stream2_group<Tin>();
    constexpr int L = VEC == 1 ? kSL : KLA_STREAM2_L;
    constexpr int NS = stream_stages<Tin, VEC>();
    using Cfg = kla::StreamTile<Tin, L, W, NS, G, VEC>;
    static_assert(NS >= 2 && Cfg::SMEM <= 227 * 1024, "stream kernel shared memory");
    const int64_t grid = std::min<int64_t>(prm.nunits, sm_count());
    if constexpr (VEC == 1) {
        auto kernel = kla::kla_forward_stream_kernel<Tin, L, W, NS, G>;
        cudaError_t e = ensure_smem_attr(kernel, Cfg::SMEM);
        if (e != cudaSuccess) return e;
        kernel<<<(unsigned)grid, Cfg::THREADS, Cfg::SMEM, stream>>>(prm, maps);
    } else {
        auto kernel = kla::kla_forward_stream_vec_kernel<Tin, L, W, NS, G, VEC>;
        cudaError_t e = ensure_smem_attr(kernel, Cfg::SMEM);
        if (e != cudaSuccess) return e;
        return launch_scan_kernel(kernel, grid, Cfg::THREADS, Cfg::SMEM, stream, prm.ticket != nullptr, prm, maps);
    }
    return cudaGetLastError();
}

// [B, T, HN] tensor viewed as dims {HN, T, B}, box {box_x, rows, 1}.
bool encode_stream_map(CUtensorMap *m, const void *base, CUtensorMapDataType dt, size_t esz,
                       int64_t B, int64_t T, int64_t HN, int rows, int box_x = 32) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)HN, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t strides[2] = {(cuuint64_t)(HN * esz), (cuuint64_t)(T * HN * esz)};
    const cuuint32_t box[3] = {(cuuint32_t)box_x, (cuuint32_t)rows, 1u};
    const cuuint32_t estr[3] = {1u, 1u, 1u};
    return fn(m, dt, 3, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Runs per tile for the streaming kernel: the number P <= KLA_STREAM_MAX_PARTS
// of runs per tile whose units (tiles x P) fill the SMs' rounds best, among
// those that keep at least 8 chunks per run; 1 when there are fewer than two
// tiles per SM (a later run's predecessor must have been ticketed a full
// round earlier, or the run would wait).  Ties go to fewer runs.
#ifndef KLA_STREAM_MAX_PARTS
#define KLA_STREAM_MAX_PARTS 4
#endif
int stream_parts(int64_t ntiles, int64_t nchunks, int min_rounds = 2) {
    // min_rounds: the fewest rounds of tiles (tiles / SMs) for which runs are
    // cut; a run's predecessor is ticketed ntiles tickets before it
    const int64_t G = sm_count();
    if (ntiles < min_rounds * G) return 1;
    int best = 1;
    double best_balance = 0.0;
    for (int P = 1; P <= KLA_STREAM_MAX_PARTS; ++P) {
        if (P > 1 && (nchunks + P - 1) / P < 8) break;
        const int64_t U = ntiles * P;
        const int64_t rounds = (U + G - 1) / G;
        const double balance = (double)U / (double)(rounds * G);
        if (balance > best_balance + 0.01) {
            best = P;
            best_balance = balance;
        }
    }
    return best;
}

// Whole tiles by ticket: with more tiles than SMs, each at least 8 chunks
// long, the tiles are handed out by ticket (a workspace counter) so that a
// CTA on a faster SM takes more of them; CTAs with equal round-robin shares
// finish up to 30% apart on some shapes.  Shorter tiles stay round-robin.
// `uneven_only`: only when the tiles do not divide evenly over the SMs (the
// backward scan: 16% faster ticketed on B=256, H*N=512, T=512, but 5% slower
// on the LM-layer shape at B=37, 16 tiles per SM exactly).
bool whole_tiles_ticketed(int64_t ntiles, int64_t nchunks, bool uneven_only = false) {
    const int64_t sms = sm_count();
    return ntiles > sms && nchunks >= 8 && (!uneven_only || ntiles % sms != 0);
}

// Workspace of the streaming kernel when it splits tiles into runs: a header
// (ticket), one ready flag per (tile, run boundary), the states at the run
// boundaries.
struct StreamWs {
    size_t flags_off = 0, state_off = 0, clear_bytes = 0, total = 0;
};
StreamWs stream_ws_layout(int64_t ntiles, int parts, int cw = 32) {
    StreamWs w;
    const size_t nb = (size_t)ntiles * (size_t)(parts - 1);
    w.flags_off = kHeaderBytes;
    w.state_off = w.flags_off + round_up(nb * sizeof(unsigned), 256);
    w.clear_bytes = w.state_off;
    w.total = w.state_off + round_up(nb * 2 * (size_t)cw * sizeof(float), 256);
    return w;
}

// The streaming forward kernel's layout for a call: two channels per lane
// for bf16 inputs of at least 64 channels per batch row, else one.
struct StreamGeom {
    int vec, cw, L;
    int64_t ntiles, nct, nchunks;
    int parts;
    bool ticketed;  // units taken by ticket (a workspace counter) rather than round-robin
};
StreamGeom stream_geom(int64_t B, int64_t T, int64_t HN, size_t esz) {
    StreamGeom g;
    g.vec = (esz == 2 && HN >= 64 && !KLA_STREAM2_OFF) ? 2 : 1;
    g.cw = 32 * g.vec;
    g.L = g.vec == 2 ? KLA_STREAM2_L : kSL;
    g.nct = (HN + g.cw - 1) / g.cw;
    g.ntiles = B * g.nct;
    g.nchunks = (T + g.L - 1) / g.L;
    g.parts = stream_parts(g.ntiles, g.nchunks, g.vec == 2 ? 1 : 2);
    // Whole tiles are ticketed too when there are more than the SMs and each
    // is at least 8 chunks long: a CTA on a faster SM then takes more of them
    // (CTAs with equal round-robin shares finish up to 30% apart on some
    // shapes: B=256, H*N=512, T=512 fp32 12% faster ticketed, the LM-layer
    // shape at B=37 8%); shorter tiles stay round-robin (the stiff shape,
    // 4 chunks per tile, 2-3% slower ticketed).
    g.ticketed = g.parts > 1 || whole_tiles_ticketed(g.ntiles, g.nchunks);
    return g;
}

// 2: the channel-owning streaming kernel -- its TMA geometry holds (16-byte
//    aligned inputs and outputs, H*N*elem a multiple of 16 bytes, H*N >= 32,
//    T >= one chunk) and there are at least 0.8 x (SM count) tiles of 32
//    channels to keep the GPU busy -- or at least 0.4 x (SM count) tiles of
//    at most 16 chunks (short sequences: 64 tiles of 8-16 chunks measured
//    5-15% faster streaming, of 32 chunks even; 16-32 tiles slower) -- or
//    the test hook forces it;
// 1: the chunked kernel with cross-CTA carries (any shape).
int forward_kernel_choice(int64_t B, int64_t T, int64_t HN, size_t esz, const void *a, const void *p,
                          const void *phi, const void *b, const void *o0, const void *o1, const void *o2,
                          const void *o3) {
    const int force = g_force_kernel.load();
    if (force == 1) return 1;
    const bool geometry = (HN * (int64_t)esz) % 16 == 0 && T >= kSL && HN >= 32 && aligned16(a) &&
                          aligned16(p) && aligned16(phi) && aligned16(b) && aligned16(o0) && aligned16(o1) &&
                          aligned16(o2) && aligned16(o3) && encode_fn() != nullptr;
    if (!geometry) return 1;
    if (force == 2) return 2;
    const int64_t ntiles32 = B * ((HN + 31) / 32);
    const int64_t sms = sm_count();
    if (ntiles32 * 5 >= sms * 4) return 2;
    return ntiles32 * 5 >= sms * 2 && (T + kSL - 1) / kSL <= 16 ? 2 : 1;
}

cudaError_t launch_clear(void *ws, size_t bytes, cudaStream_t stream) {
    const int64_t n16 = (int64_t)(bytes / 16);
    const int threads = 256;
    const int64_t blocks = std::min<int64_t>((n16 + threads - 1) / threads, 148 * 8);
    kla::kla_clear_kernel<<<(unsigned)std::max<int64_t>(blocks, 1), threads, 0, stream>>>(
        static_cast<uint4 *>(ws), n16);
    return cudaGetLastError();
}

}  // namespace

KLA_API int kla_abi_version(void) { return KLA_ABI_VERSION; }

KLA_API const char *kla_strerror(kla_status_t s) {
    switch (s) {
        case KLA_OK: return "KLA_OK";
        case KLA_ERR_INVALID_ARG: return "KLA_ERR_INVALID_ARG: invalid argument";
        case KLA_ERR_UNSUPPORTED_DTYPE: return "KLA_ERR_UNSUPPORTED_DTYPE: dtype must be KLA_F32 or KLA_BF16";
        case KLA_ERR_WORKSPACE_TOO_SMALL: return "KLA_ERR_WORKSPACE_TOO_SMALL: workspace below the required size";
        case KLA_ERR_CUDA: return "KLA_ERR_CUDA: a CUDA call failed";
        case KLA_ERR_TIMEOUT: return "KLA_ERR_TIMEOUT: a device-side bounded wait ran out";
        case KLA_ERR_MISALIGNED: return "KLA_ERR_MISALIGNED: workspace must be 256-byte aligned";
        case KLA_ERR_TOO_LARGE:
            return "KLA_ERR_TOO_LARGE: the problem needs more scratch than the library's static array "
                   "(KLA_STATIC_SCRATCH_BYTES); use kla_scan_forward with a caller-allocated workspace";
    }
    return "unknown kla_status_t";
}

KLA_API kla_status_t kla_scan_forward_workspace_size(int64_t B, int64_t T, int64_t H, int64_t N,
                                                     kla_dtype_t in_dtype, size_t *bytes) {
    if (!bytes || B < 0 || T < 0 || H < 0 || N < 0) return KLA_ERR_INVALID_ARG;
    if (!dtype_ok(in_dtype)) return KLA_ERR_UNSUPPORTED_DTYPE;
    int64_t HN = 0;
    if (!mul_ok(H, N, &HN)) return KLA_ERR_INVALID_ARG;
    if (B == 0 || T == 0 || HN == 0) {
        *bytes = 0;
        return KLA_OK;
    }
    FwdLayout lay;
    if (!fwd_layout(B, T, HN, &lay)) return KLA_ERR_INVALID_ARG;
    const StreamGeom sg = stream_geom(B, T, HN, dtype_size(in_dtype));
    const StreamWs sw = stream_ws_layout(sg.ntiles, KLA_STREAM_MAX_PARTS, sg.cw);  // the most runs stream_parts picks
    *bytes = std::max(lay.total, sw.total);
    return KLA_OK;
}

KLA_API kla_status_t kla_scan_forward(const void *a, const void *p, const void *phi, const void *b,
                                      kla_dtype_t in_dtype, const float *lambda0, const float *eta0,
                                      float *lambda_out, float *eta_out, float *mu_out,
                                      float *var_out, int64_t B, int64_t T, int64_t H, int64_t N,
                                      void *workspace, size_t workspace_bytes, void *stream) {
    if (B < 0 || T < 0 || H < 0 || N < 0) return KLA_ERR_INVALID_ARG;
    if (!dtype_ok(in_dtype)) return KLA_ERR_UNSUPPORTED_DTYPE;
    int64_t HN = 0, C = 0, BT = 0, elems = 0;
    if (!mul_ok(H, N, &HN) || !mul_ok(B, HN, &C) || !mul_ok(B, T, &BT) || !mul_ok(BT, HN, &elems))
        return KLA_ERR_INVALID_ARG;
    if (elems == 0) return KLA_OK;
    if (!a || !p || !phi || !b || !lambda0 || !eta0 || !lambda_out || !eta_out)
        return KLA_ERR_INVALID_ARG;
    const size_t esz = dtype_size(in_dtype);
    int64_t in_bytes = 0, out_bytes = 0;
    if (!mul_ok(elems, (int64_t)esz, &in_bytes) || !mul_ok(elems, 4, &out_bytes))
        return KLA_ERR_INVALID_ARG;
    // the workspace is written too: it may overlap no input and no output
    const Range outs[5] = {range_of(lambda_out, out_bytes), range_of(eta_out, out_bytes),
                           range_of(mu_out, out_bytes), range_of(var_out, out_bytes),
                           range_of(workspace, (int64_t)workspace_bytes)};
    const Range ins[6] = {range_of(a, in_bytes), range_of(p, in_bytes), range_of(phi, in_bytes),
                          range_of(b, in_bytes), range_of(lambda0, C * 4), range_of(eta0, C * 4)};
    if (any_overlap(outs, 5, ins, 6)) return KLA_ERR_INVALID_ARG;

    FwdLayout lay;
    if (!fwd_layout(B, T, HN, &lay)) return KLA_ERR_INVALID_ARG;
    size_t need = 0;
    if (kla_scan_forward_workspace_size(B, T, H, N, in_dtype, &need) != KLA_OK) return KLA_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < need) return KLA_ERR_WORKSPACE_TOO_SMALL;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return KLA_ERR_MISALIGNED;
    if (T > INT32_MAX || HN > INT32_MAX || B > INT32_MAX || lay.nct > INT32_MAX ||
        lay.nchunks > INT32_MAX)
        return KLA_ERR_INVALID_ARG;

    unsigned char *ws = static_cast<unsigned char *>(workspace);
    FwdParams prm;
    prm.in[0] = a; prm.in[1] = p; prm.in[2] = phi; prm.in[3] = b;
    prm.lam0 = lambda0; prm.eta0 = eta0;
    prm.out[0] = lambda_out; prm.out[1] = eta_out; prm.out[2] = mu_out; prm.out[3] = var_out;
    prm.T = T; prm.HN = HN;
    prm.tiles_per_chunk = B * lay.nct;
    prm.nct = (int)lay.nct;
    prm.nchunks = (int)lay.nchunks;
    prm.ticket = reinterpret_cast<unsigned *>(ws);
    prm.flags = reinterpret_cast<unsigned *>(ws + lay.flags_off);
    prm.agg_ws = reinterpret_cast<float *>(ws + lay.agg_off);
    prm.incl_ws = reinterpret_cast<float *>(ws + lay.incl_off);
    prm.ckpt = kCkpt;
    prm.wait_ns = g_wait_ns.load();
    prm.stall_chunk = g_stall_chunk.load();

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const CUtensorMapDataType tdt =
        in_dtype == KLA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;

    const int choice = forward_kernel_choice(B, T, HN, esz, a, p, phi, b, lambda_out, eta_out, mu_out, var_out);
    // The channel-owning streaming kernel when forward_kernel_choice picks it
    // (it needs no workspace beyond its run splits); otherwise the chunked
    // kernel below.
    if (choice == 2) {
        const StreamGeom sg = stream_geom(B, T, HN, esz);
        const int G = in_dtype == KLA_F32 ? (sg.vec == 2 ? stream2_group<float>() : stream_group<float>())
                                          : (sg.vec == 2 ? stream2_group<__nv_bfloat16>() : stream_group<__nv_bfloat16>());
        FwdMaps smaps;
        std::memset(&smaps, 0, sizeof(smaps));
        const void *ins4[4] = {a, p, phi, b};
        bool ok = true;
        for (int k = 0; k < 4 && ok; ++k)
            ok = encode_stream_map(&smaps.in[k], ins4[k], tdt, esz, B, T, HN, sg.L, sg.cw);
        float *outs4[4] = {lambda_out, eta_out, mu_out, var_out};
        for (int k = 0; k < 4 && ok; ++k)
            if (outs4[k])
                ok = encode_stream_map(&smaps.out[k], outs4[k], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, B, T, HN, G, sg.cw);
        if (ok) {
            kla::StreamParams sp;
            sp.lam0 = lambda0; sp.eta0 = eta0;
            sp.out[0] = lambda_out; sp.out[1] = eta_out; sp.out[2] = mu_out; sp.out[3] = var_out;
            sp.write_mu = mu_out != nullptr; sp.write_var = var_out != nullptr;
            sp.T = T; sp.HN = HN; sp.ntiles = sg.ntiles;
            sp.nct = (int)sg.nct;
            sp.nchunks = (int)sg.nchunks;
            sp.wait_ns = g_wait_ns.load();
            sp.stall_chunk = g_stall_chunk.load() >= 0 ? g_stall_chunk.load() * kL / sg.L : -1;
            sp.parts = sg.parts;
            sp.chunks_per_part = (sp.nchunks + sp.parts - 1) / sp.parts;  // (the kernels cut runs 4:3:2:1)
            sp.nunits = sp.ntiles * sp.parts;
            sp.ticket = reinterpret_cast<unsigned *>(ws);
            sp.part_flags = nullptr;
            sp.part_state = nullptr;
            if (sp.parts > 1) {
                const StreamWs sw = stream_ws_layout(sp.ntiles, sp.parts, sg.cw);
                if (sw.total > workspace_bytes) return KLA_ERR_WORKSPACE_TOO_SMALL;  // size function out of step
                sp.part_flags = reinterpret_cast<unsigned *>(ws + sw.flags_off);
                sp.part_state = reinterpret_cast<float *>(ws + sw.state_off);
                if (launch_clear(ws, sw.clear_bytes, st) != cudaSuccess) return KLA_ERR_CUDA;
            } else if (sg.ticketed) {
                if (launch_clear(ws, stream_ws_layout(sp.ntiles, 1, sg.cw).clear_bytes, st) != cudaSuccess)
                    return KLA_ERR_CUDA;
            } else {
                sp.ticket = nullptr;  // round-robin units, no workspace
            }
            cudaError_t es;
            if (in_dtype == KLA_F32)
                es = launch_forward_stream<float>(sp, smaps, st);
            else
                es = sg.vec == 2 ? launch_forward_stream<__nv_bfloat16, 2>(sp, smaps, st)
                                 : launch_forward_stream<__nv_bfloat16>(sp, smaps, st);
            return es == cudaSuccess ? KLA_OK : KLA_ERR_CUDA;
        }
    }

    // TMA boxes when the geometry allows them; plain loads otherwise.
    FwdMaps maps;
    std::memset(&maps, 0, sizeof(maps));
    bool tma = (HN * (int64_t)esz) % 16 == 0 && T >= kL && HN >= kCW;
    const void *ptrs[8] = {a, p, phi, b, lambda_out, eta_out, mu_out, var_out};
    for (int k = 0; k < 8 && tma; ++k)
        if (ptrs[k] && !aligned16(ptrs[k])) tma = false;
    if (tma) {
        for (int k = 0; k < 4 && tma; ++k) tma = encode_map(&maps.in[k], ptrs[k], tdt, esz, B, T, HN);
        for (int k = 0; k < 4 && tma; ++k)
            if (ptrs[4 + k])
                tma = encode_map(&maps.out[k], ptrs[4 + k], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, B, T, HN);
    }

    if (launch_clear(ws, lay.clear_bytes, st) != cudaSuccess) return KLA_ERR_CUDA;
    cudaError_t e;
    if (in_dtype == KLA_F32)
        e = tma ? launch_forward<float, true>(prm, maps, lay.tiles, st)
                : launch_forward<float, false>(prm, maps, lay.tiles, st);
    else
        e = tma ? launch_forward<__nv_bfloat16, true>(prm, maps, lay.tiles, st)
                : launch_forward<__nv_bfloat16, false>(prm, maps, lay.tiles, st);
    return e == cudaSuccess ? KLA_OK : KLA_ERR_CUDA;
}

KLA_API kla_status_t kla_scan_step(const void *a, const void *p, const void *phi, const void *b,
                                   kla_dtype_t in_dtype, float *lambda_state, float *eta_state,
                                   float *mu_out, float *var_out, int64_t B, int64_t H, int64_t N,
                                   void *stream) {
    if (B < 0 || H < 0 || N < 0) return KLA_ERR_INVALID_ARG;
    if (!dtype_ok(in_dtype)) return KLA_ERR_UNSUPPORTED_DTYPE;
    int64_t HN = 0, C = 0;
    if (!mul_ok(H, N, &HN) || !mul_ok(B, HN, &C)) return KLA_ERR_INVALID_ARG;
    if (C == 0) return KLA_OK;
    if (!a || !p || !phi || !b || !lambda_state || !eta_state) return KLA_ERR_INVALID_ARG;
    const size_t esz = dtype_size(in_dtype);
    int64_t in_bytes = 0, st_bytes = 0;
    if (!mul_ok(C, (int64_t)esz, &in_bytes) || !mul_ok(C, 4, &st_bytes)) return KLA_ERR_INVALID_ARG;
    const Range outs[4] = {range_of(lambda_state, st_bytes), range_of(eta_state, st_bytes),
                           range_of(mu_out, st_bytes), range_of(var_out, st_bytes)};
    const Range ins[4] = {range_of(a, in_bytes), range_of(p, in_bytes), range_of(phi, in_bytes),
                          range_of(b, in_bytes)};
    if (any_overlap(outs, 4, ins, 4)) return KLA_ERR_INVALID_ARG;

    StepParams prm;
    prm.in[0] = a; prm.in[1] = p; prm.in[2] = phi; prm.in[3] = b;
    prm.lam = lambda_state; prm.eta = eta_state; prm.mu = mu_out; prm.var = var_out;
    prm.C = C;

    const uintptr_t in_align = esz == 4 ? 15u : 7u;
    bool vec = (C % 4) == 0;
    const void *ins_p[4] = {a, p, phi, b};
    for (int k = 0; k < 4; ++k)
        if (reinterpret_cast<uintptr_t>(ins_p[k]) & in_align) vec = false;
    const void *outs_p[4] = {lambda_state, eta_state, mu_out, var_out};
    for (int k = 0; k < 4; ++k)
        if (outs_p[k] && !aligned16(outs_p[k])) vec = false;

    const int threads = 256;
    const int64_t work = vec ? C / 4 : C;
    // Two CTAs per SM at most, grid-stride beyond (B=256, H=32, N=128 fp32,
    // graph of 256 steps: 5.09-5.12 us per token against 5.29 with one CTA
    // per 256 vectors (1024 CTAs), 5.91 with one per SM and 6.3-6.8 with
    // three or four).
    const int64_t blocks =
        std::max<int64_t>(1, std::min<int64_t>((work + threads - 1) / threads, (int64_t)sm_count() * 2));
    // Programmatic dependent launch: consecutive decode steps overlap the next
    // step's launch and input prefetch with the current step's tail (the
    // kernels wait for the preceding grid before touching the state).
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)blocks);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e;
    if (in_dtype == KLA_F32)
        e = vec ? cudaLaunchKernelEx(&cfg, kla::kla_step_vec4_kernel<float>, prm)
                : cudaLaunchKernelEx(&cfg, kla::kla_step_scalar_kernel<float>, prm);
    else
        e = vec ? cudaLaunchKernelEx(&cfg, kla::kla_step_vec4_kernel<__nv_bfloat16>, prm)
                : cudaLaunchKernelEx(&cfg, kla::kla_step_scalar_kernel<__nv_bfloat16>, prm);
    return e == cudaSuccess ? KLA_OK : KLA_ERR_CUDA;
}

KLA_API kla_status_t kla_get_error(void *stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return KLA_ERR_CUDA;
    if (cudaGetLastError() != cudaSuccess) return KLA_ERR_CUDA;
    unsigned word = 0;
    if (cudaMemcpyFromSymbol(&word, kla::g_error_word, sizeof(word)) != cudaSuccess) return KLA_ERR_CUDA;
    if (word == 0u) return KLA_OK;
    const unsigned zero = 0u;
    if (cudaMemcpyToSymbol(kla::g_error_word, &zero, sizeof(zero)) != cudaSuccess) return KLA_ERR_CUDA;
    return KLA_ERR_TIMEOUT;
}

KLA_API kla_status_t kla_set_wait_limit_ns(uint64_t ns) {
    if (ns == 0) return KLA_ERR_INVALID_ARG;
    g_wait_ns.store(ns);
    return KLA_OK;
}

KLA_API kla_status_t kla_debug_unset_flag_wait(void *stream) {
    kla::kla_unset_flag_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(g_wait_ns.load());
    return cudaGetLastError() == cudaSuccess ? KLA_OK : KLA_ERR_CUDA;
}

KLA_API int kla_forward_chunk_tokens(void) { return kL; }

KLA_API kla_status_t kla_scan_forward_plan(int64_t B, int64_t T, int64_t H, int64_t N, kla_dtype_t in_dtype,
                                           const void *a, const void *p, const void *phi, const void *b,
                                           int *kernel, int *launches) {
    if (!kernel || !launches || B < 0 || T < 0 || H < 0 || N < 0) return KLA_ERR_INVALID_ARG;
    if (!dtype_ok(in_dtype)) return KLA_ERR_UNSUPPORTED_DTYPE;
    int64_t HN = 0, BT = 0, elems = 0;
    if (!mul_ok(H, N, &HN) || !mul_ok(B, T, &BT) || !mul_ok(BT, HN, &elems)) return KLA_ERR_INVALID_ARG;
    if (elems == 0) {
        *kernel = 0;
        *launches = 0;
        return KLA_OK;
    }
    // outputs come from the caching allocator (aligned); only the inputs are passed here
    *kernel = forward_kernel_choice(B, T, HN, dtype_size(in_dtype), a, p, phi, b, nullptr, nullptr, nullptr,
                                    nullptr);
    *launches = 2;  // chunked kernel: workspace clear + scan
    if (*kernel == 2) *launches = stream_geom(B, T, HN, dtype_size(in_dtype)).ticketed ? 2 : 1;
    return KLA_OK;
}

KLA_API kla_status_t kla_debug_force_forward_kernel(int which) {
    if (which < 0 || which > 2) return KLA_ERR_INVALID_ARG;
    g_force_kernel.store(which);
    return KLA_OK;
}

KLA_API kla_status_t kla_debug_stall_chunk(int64_t chunk) {
    if (chunk < -1) return KLA_ERR_INVALID_ARG;
    g_stall_chunk.store(chunk);
    return KLA_OK;
}

// ---------------------------------------------------------------------------
// kla_scan_forward_static: kla_scan_forward without a caller-provided
// workspace, for callers that cannot allocate device memory.
//
// The carry scratch is this file-scope device array, KLA_STATIC_SCRATCH_BYTES
// long.  Every device that loads the library holds one copy of it until the
// process exits.  Host code cannot use the array's name as a device address
// (in host code it names a host-side shadow), so the device address is looked
// up once per device with cudaGetSymbolAddress, with that device current, on
// the first call made on it, and cached.
// ---------------------------------------------------------------------------
namespace {

static __device__ __align__(256) unsigned char g_static_scratch[KLA_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 256;

// Device address of g_static_scratch on the current device (nullptr on error).
void *static_scratch_address() {
    static std::mutex mu;
    static void *addr[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (addr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        addr[dev] = p;
    }
    return addr[dev];
}

}  // namespace

KLA_API kla_status_t kla_scan_forward_static(const void *a, const void *p, const void *phi,
                                             const void *b, kla_dtype_t in_dtype,
                                             const float *lambda0, const float *eta0,
                                             float *lambda_out, float *eta_out, float *mu_out,
                                             float *var_out, int64_t B, int64_t T, int64_t H,
                                             int64_t N, void *stream) {
    size_t need = 0;
    const kla_status_t st = kla_scan_forward_workspace_size(B, T, H, N, in_dtype, &need);
    if (st != KLA_OK) return st;
    if (need > (size_t)KLA_STATIC_SCRATCH_BYTES) return KLA_ERR_TOO_LARGE;
    if (need == 0)  // empty problem: validate and return without touching the device
        return kla_scan_forward(a, p, phi, b, in_dtype, lambda0, eta0, lambda_out, eta_out, mu_out,
                                var_out, B, T, H, N, nullptr, 0, stream);
    void *scratch = static_scratch_address();
    if (scratch == nullptr) return KLA_ERR_CUDA;
    // kla_scan_forward zeroes the part of the scratch that must start at zero
    // (ticket counter and ready flags) on `stream` before its scan kernel.
    return kla_scan_forward(a, p, phi, b, in_dtype, lambda0, eta0, lambda_out, eta_out, mu_out,
                            var_out, B, T, H, N, scratch, (size_t)KLA_STATIC_SCRATCH_BYTES, stream);
}

// ---------------------------------------------------------------------------
// Gradients: kla_scan_backward (kernels in kla_backward.cuh).
// ---------------------------------------------------------------------------
namespace {

// Backward streaming kernel: chunk length (16 tokens: a chunk warp holds six
// L-token arrays and two (L+1)-token arrays of its chunk in registers), chunk
// warps and output group per dtype; the ring takes what shared memory is left.
#ifndef KLA_BWD_L
#define KLA_BWD_L 16
#endif
// 6 (fp32) and 7 (bf16) chunk warps, at up to 210 registers per thread:
// same-GPU sweeps over 4-9 warps and 4-16 token output groups put these
// first (fp32 long workload 96-97% of the copy bandwidth; 9 warps, capped at
// 168 registers and spilling, 90%).
#ifndef KLA_BWD_W_F32
#define KLA_BWD_W_F32 6
#endif
#ifndef KLA_BWD_W_BF16
#define KLA_BWD_W_BF16 7
#endif
#ifndef KLA_BWD_G_F32
#define KLA_BWD_G_F32 8
#endif
#ifndef KLA_BWD_G_BF16
#define KLA_BWD_G_BF16 8
#endif
constexpr int kBL = KLA_BWD_L;
template <typename Tin> constexpr int bwd_warps() { return sizeof(Tin) == 4 ? KLA_BWD_W_F32 : KLA_BWD_W_BF16; }
template <typename Tin> constexpr int bwd_group() { return sizeof(Tin) == 4 ? KLA_BWD_G_F32 : KLA_BWD_G_BF16; }
template <typename Tin>
constexpr int bwd_stages() {
    constexpr int W = bwd_warps<Tin>();
    constexpr int G = bwd_group<Tin>();
    const int stage = 2 * kBL * 32 * (int)sizeof(Tin) + 2 * (kBL + 1) * 32 * 4 + 4 * kBL * 32 * 4;
    const int fixed = W * 2 * 4 * G * 32 * (int)sizeof(Tin) + W * 2 * 32 * 4 + W * 8 + 2048;
    const int ns = (KLA_STREAM_SMEM - fixed) / stage;
    return ns > KLA_STREAM_MAX_STAGES ? KLA_STREAM_MAX_STAGES : ns;
}

// 0: choose by shape; 1: the one-thread-per-channel kernel; 2: the streaming
// kernel (test hook kla_debug_force_backward_kernel).
std::atomic<int> g_force_bwd_kernel{0};

// 2 when the streaming kernel's TMA geometry holds (16-byte aligned arrays,
// H*N*elem a multiple of 16 bytes, H*N >= 32, T >= 1) and the tensor-map
// encoder is available; 1 otherwise (or when forced).
int backward_kernel_choice(int64_t T, int64_t HN, size_t esz, const void *const *ptrs, int nptrs) {
    if (g_force_bwd_kernel.load() == 1 || T == 0) return 1;
    bool ok = (HN * (int64_t)esz) % 16 == 0 && HN >= 32 && encode_fn() != nullptr;
    for (int k = 0; k < nptrs && ok; ++k)
        if (ptrs[k] && !aligned16(ptrs[k])) ok = false;
    return ok ? 2 : 1;
}

template <typename Tin>
cudaError_t launch_backward_stream(const kla::BwdParams &prm, const kla::BwdMaps &maps, cudaStream_t stream) {
    constexpr int W = bwd_warps<Tin>();
    constexpr int G = bwd_group<Tin>();
    constexpr int NS = bwd_stages<Tin>();
    using Cfg = kla::BwdTile<Tin, kBL, W, NS, G>;
    static_assert(NS >= W && Cfg::SMEM <= 227 * 1024, "backward kernel shared memory");
    auto kernel = kla::kla_backward_stream_kernel<Tin, kBL, W, NS, G>;
    cudaError_t e = ensure_smem_attr(kernel, Cfg::SMEM);
    if (e != cudaSuccess) return e;
    const int64_t grid = std::min<int64_t>(prm.nunits, sm_count());
    kernel<<<(unsigned)grid, Cfg::THREADS, Cfg::SMEM, stream>>>(prm, maps);
    return cudaGetLastError();
}

template <typename Tin>
unsigned bwd_stage_tx(unsigned g_mask) {
    unsigned tx = 2u * kBL * 32u * (unsigned)sizeof(Tin) + 2u * (kBL + 1) * 32u * 4u;
    for (int k = 0; k < 4; ++k)
        if (g_mask >> k & 1u) tx += kBL * 32u * 4u;
    return tx;
}

template <typename Tin>
cudaError_t launch_backward_seq(const kla::BwdParams &prm, cudaStream_t stream) {
    const int threads = 128;
    const int64_t blocks = (prm.C + threads - 1) / threads;
    kla::kla_backward_seq_kernel<Tin><<<(unsigned)blocks, threads, 0, stream>>>(prm);
    return cudaGetLastError();
}

}  // namespace

KLA_API kla_status_t kla_scan_backward_workspace_size(int64_t B, int64_t T, int64_t H, int64_t N,
                                                      kla_dtype_t in_dtype, size_t *bytes) {
    if (!bytes || B < 0 || T < 0 || H < 0 || N < 0) return KLA_ERR_INVALID_ARG;
    if (!dtype_ok(in_dtype)) return KLA_ERR_UNSUPPORTED_DTYPE;
    int64_t HN = 0, BT = 0, elems = 0;
    if (!mul_ok(H, N, &HN) || !mul_ok(B, T, &BT) || !mul_ok(BT, HN, &elems)) return KLA_ERR_INVALID_ARG;
    if (elems == 0) {
        *bytes = 0;
        return KLA_OK;
    }
    *bytes = stream_ws_layout(B * ((HN + 31) / 32), KLA_STREAM_MAX_PARTS).total;
    return KLA_OK;
}

KLA_API kla_status_t kla_scan_backward(const void *a, const void *p, kla_dtype_t in_dtype,
                                       const float *lambda0, const float *eta0,
                                       const float *lambda_out, const float *eta_out,
                                       const float *g_lambda, const float *g_eta, const float *g_mu,
                                       const float *g_var, void *grad_a, void *grad_p, void *grad_phi,
                                       void *grad_b, float *grad_lambda0, float *grad_eta0,
                                       int64_t B, int64_t T, int64_t H, int64_t N,
                                       void *workspace, size_t workspace_bytes, void *stream) {
    if (B < 0 || T < 0 || H < 0 || N < 0) return KLA_ERR_INVALID_ARG;
    if (!dtype_ok(in_dtype)) return KLA_ERR_UNSUPPORTED_DTYPE;
    int64_t HN = 0, C = 0, BT = 0, elems = 0;
    if (!mul_ok(H, N, &HN) || !mul_ok(B, HN, &C) || !mul_ok(B, T, &BT) || !mul_ok(BT, HN, &elems))
        return KLA_ERR_INVALID_ARG;
    if (C == 0) return KLA_OK;
    if (!lambda0 || !eta0) return KLA_ERR_INVALID_ARG;
    if (elems > 0 && (!a || !p || !lambda_out || !eta_out)) return KLA_ERR_INVALID_ARG;
    const size_t esz = dtype_size(in_dtype);
    int64_t in_bytes = 0, f_bytes = 0, c_bytes = 0;
    if (!mul_ok(elems, (int64_t)esz, &in_bytes) || !mul_ok(elems, 4, &f_bytes) || !mul_ok(C, 4, &c_bytes))
        return KLA_ERR_INVALID_ARG;
    const Range outs[7] = {range_of(grad_a, in_bytes), range_of(grad_p, in_bytes), range_of(grad_phi, in_bytes),
                           range_of(grad_b, in_bytes), range_of(grad_lambda0, c_bytes),
                           range_of(grad_eta0, c_bytes), range_of(workspace, (int64_t)workspace_bytes)};
    const Range ins[10] = {range_of(a, in_bytes), range_of(p, in_bytes), range_of(lambda0, c_bytes),
                           range_of(eta0, c_bytes), range_of(lambda_out, f_bytes), range_of(eta_out, f_bytes),
                           range_of(g_lambda, f_bytes), range_of(g_eta, f_bytes), range_of(g_mu, f_bytes),
                           range_of(g_var, f_bytes)};
    if (any_overlap(outs, 7, ins, 10)) return KLA_ERR_INVALID_ARG;
    size_t need = 0;
    if (kla_scan_backward_workspace_size(B, T, H, N, in_dtype, &need) != KLA_OK) return KLA_ERR_INVALID_ARG;
    if (need > 0 && (!workspace || workspace_bytes < need)) return KLA_ERR_WORKSPACE_TOO_SMALL;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return KLA_ERR_MISALIGNED;
    if (T > INT32_MAX - 1 || HN > INT32_MAX || B > INT32_MAX) return KLA_ERR_INVALID_ARG;

    kla::BwdParams prm;
    std::memset(&prm, 0, sizeof(prm));
    prm.a = a; prm.p = p; prm.lam = lambda_out; prm.eta = eta_out;
    prm.g[0] = g_lambda; prm.g[1] = g_eta; prm.g[2] = g_mu; prm.g[3] = g_var;
    prm.grad[0] = grad_a; prm.grad[1] = grad_p; prm.grad[2] = grad_phi; prm.grad[3] = grad_b;
    prm.lam0 = lambda0; prm.eta0 = eta0; prm.g_lam0 = grad_lambda0; prm.g_eta0 = grad_eta0;
    prm.T = T; prm.HN = HN; prm.C = C;
    prm.wait_ns = g_wait_ns.load();
    prm.stall_chunk = -1;
    for (int k = 0; k < 4; ++k) {
        if (prm.g[k]) prm.g_mask |= 1u << k;
        if (prm.grad[k]) prm.grad_mask |= 1u << k;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const void *ptrs[14] = {a, p, lambda_out, eta_out, g_lambda, g_eta, g_mu, g_var,
                            grad_a, grad_p, grad_phi, grad_b, nullptr, nullptr};

    if (backward_kernel_choice(T, HN, esz, ptrs, 12) == 2) {
        const CUtensorMapDataType tdt =
            in_dtype == KLA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
        const int G = in_dtype == KLA_F32 ? bwd_group<float>() : bwd_group<__nv_bfloat16>();
        kla::BwdMaps maps;
        std::memset(&maps, 0, sizeof(maps));
        bool ok = encode_stream_map(&maps.in[0], a, tdt, esz, B, T, HN, kBL) &&
                  encode_stream_map(&maps.in[1], p, tdt, esz, B, T, HN, kBL) &&
                  encode_stream_map(&maps.in[2], lambda_out, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, B, T, HN, kBL + 1) &&
                  encode_stream_map(&maps.in[3], eta_out, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, B, T, HN, kBL + 1);
        for (int k = 0; k < 4 && ok; ++k)
            if (prm.g[k])
                ok = encode_stream_map(&maps.in[4 + k], prm.g[k], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, B, T, HN, kBL);
        for (int k = 0; k < 4 && ok; ++k)
            if (prm.grad[k]) ok = encode_stream_map(&maps.out[k], prm.grad[k], tdt, esz, B, T, HN, G);
        if (ok) {
            prm.ntiles = B * ((HN + 31) / 32);
            prm.nct = (int)((HN + 31) / 32);
            prm.nchunks = (int)((T + kBL - 1) / kBL);
            prm.stage_tx = in_dtype == KLA_F32 ? bwd_stage_tx<float>(prm.g_mask)
                                               : bwd_stage_tx<__nv_bfloat16>(prm.g_mask);
            prm.stall_chunk = g_stall_chunk.load() >= 0 ? g_stall_chunk.load() * kL / kBL : -1;
            prm.parts = stream_parts(prm.ntiles, prm.nchunks);
            prm.chunks_per_part = (prm.nchunks + prm.parts - 1) / prm.parts;
            prm.nunits = prm.ntiles * prm.parts;
            unsigned char *ws = static_cast<unsigned char *>(workspace);
            prm.ticket = reinterpret_cast<unsigned *>(ws);
            if (prm.parts > 1) {
                const StreamWs sw = stream_ws_layout(prm.ntiles, prm.parts);
                if (sw.total > workspace_bytes) return KLA_ERR_WORKSPACE_TOO_SMALL;
                prm.part_flags = reinterpret_cast<unsigned *>(ws + sw.flags_off);
                prm.part_state = reinterpret_cast<float *>(ws + sw.state_off);
                if (launch_clear(ws, sw.clear_bytes, st) != cudaSuccess) return KLA_ERR_CUDA;
            } else if (whole_tiles_ticketed(prm.ntiles, prm.nchunks, true)) {
                if (launch_clear(ws, stream_ws_layout(prm.ntiles, 1).clear_bytes, st) != cudaSuccess)
                    return KLA_ERR_CUDA;
            } else {
                prm.ticket = nullptr;  // round-robin units, no workspace
            }
            const cudaError_t e = in_dtype == KLA_F32 ? launch_backward_stream<float>(prm, maps, st)
                                                      : launch_backward_stream<__nv_bfloat16>(prm, maps, st);
            return e == cudaSuccess ? KLA_OK : KLA_ERR_CUDA;
        }
    }
    const cudaError_t e = in_dtype == KLA_F32 ? launch_backward_seq<float>(prm, st)
                                              : launch_backward_seq<__nv_bfloat16>(prm, st);
    return e == cudaSuccess ? KLA_OK : KLA_ERR_CUDA;
}

KLA_API kla_status_t kla_scan_backward_plan(int64_t B, int64_t T, int64_t H, int64_t N, kla_dtype_t in_dtype,
                                            const void *a, const void *p, int *kernel, int *launches) {
    if (!kernel || !launches || B < 0 || T < 0 || H < 0 || N < 0) return KLA_ERR_INVALID_ARG;
    if (!dtype_ok(in_dtype)) return KLA_ERR_UNSUPPORTED_DTYPE;
    int64_t HN = 0, C = 0;
    if (!mul_ok(H, N, &HN) || !mul_ok(B, HN, &C)) return KLA_ERR_INVALID_ARG;
    if (C == 0) {
        *kernel = 0;
        *launches = 0;
        return KLA_OK;
    }
    const void *ptrs[2] = {a, p};
    *kernel = backward_kernel_choice(T, HN, dtype_size(in_dtype), ptrs, 2);
    *launches = 1;
    const int64_t bnt = B * ((HN + 31) / 32), bnc = (T + kBL - 1) / kBL;
    if (*kernel == 2 && (stream_parts(bnt, bnc) > 1 || whole_tiles_ticketed(bnt, bnc, true))) *launches = 2;
    return KLA_OK;
}

KLA_API kla_status_t kla_debug_force_backward_kernel(int which) {
    if (which < 0 || which > 2) return KLA_ERR_INVALID_ARG;
    g_force_bwd_kernel.store(which);
    return KLA_OK;
}

// ---------------------------------------------------------------------------
// The fused KLA layer: kla_layer_forward (kernel in kla_layer.cuh).
// ---------------------------------------------------------------------------
namespace {

// Chunk warps and ring stages of the layer kernel.  Its stages are small
// (k and q of 32 tokens, v and w of 32 / Ns value coordinates: 4.9 KB for
// fp32, Ns = 16) and the readout adds shuffles to every token, so it runs 11
// chunk warps (12 in all: 168 registers) over a 16-stage ring.
#ifndef KLA_LAYER_W
#define KLA_LAYER_W 11
#endif
#ifndef KLA_LAYER_NS
#define KLA_LAYER_NS 16
#endif
constexpr int kLayerL = 32;

template <typename Tin, int NSX>
cudaError_t launch_layer(const kla::LayerParams &prm, const kla::LayerMaps &maps, cudaStream_t stream) {
    using Cfg = kla::LayerTile<Tin, NSX, kLayerL, KLA_LAYER_W, KLA_LAYER_NS>;
    static_assert(Cfg::SMEM <= 227 * 1024, "layer kernel shared memory");
    auto kernel = kla::kla_layer_forward_kernel<Tin, NSX, kLayerL, KLA_LAYER_W, KLA_LAYER_NS>;
    cudaError_t e = ensure_smem_attr(kernel, Cfg::SMEM);
    if (e != cudaSuccess) return e;
    const int64_t grid = std::min<int64_t>(prm.nunits, sm_count());
    kernel<<<(unsigned)grid, Cfg::THREADS, Cfg::SMEM, stream>>>(prm, maps);
    return cudaGetLastError();
}

// [B, T, H, Ns] tensor viewed as dims {Ns, H, T, B}, box {Ns, 1, 32, 1}.
bool encode_layer_map(CUtensorMap *m, const void *base, CUtensorMapDataType dt, size_t esz, int64_t B,
                      int64_t T, int64_t H, int64_t Ns) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[4] = {(cuuint64_t)Ns, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)(Ns * esz), (cuuint64_t)(H * Ns * esz),
                                   (cuuint64_t)(T * H * Ns * esz)};
    const cuuint32_t box[4] = {(cuuint32_t)Ns, 1u, (cuuint32_t)kLayerL, 1u};
    const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
    return fn(m, dt, 4, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tiles of 32 state channels: (32 / Ns) value coordinates x Ns.
bool layer_shape_ok(int64_t D, int64_t Ns) { return (Ns == 8 || Ns == 16) && D % (32 / Ns) == 0; }

}  // namespace

KLA_API kla_status_t kla_layer_forward_workspace_size(int64_t B, int64_t T, int64_t H, int64_t D, int64_t Ns,
                                                      kla_dtype_t in_dtype, size_t *bytes) {
    if (!bytes || B < 0 || T < 0 || H < 0 || D < 0 || Ns < 0) return KLA_ERR_INVALID_ARG;
    if (!dtype_ok(in_dtype)) return KLA_ERR_UNSUPPORTED_DTYPE;
    if (!layer_shape_ok(D, Ns)) return KLA_ERR_INVALID_ARG;
    int64_t BH = 0, tiles = 0;
    if (!mul_ok(B, H, &BH) || !mul_ok(BH, D / (32 / Ns), &tiles)) return KLA_ERR_INVALID_ARG;
    if (tiles == 0 || T == 0) {
        *bytes = 0;
        return KLA_OK;
    }
    *bytes = stream_ws_layout(tiles, KLA_STREAM_MAX_PARTS).total;
    return KLA_OK;
}

KLA_API kla_status_t kla_layer_forward(const void *k, const void *q, const void *v, const void *w,
                                       kla_dtype_t in_dtype, const float *a, const float *p,
                                       const float *lambda0, const float *eta0, float *y, float *s,
                                       float *lambda_T, float *eta_T, int64_t B, int64_t T, int64_t H,
                                       int64_t D, int64_t Ns, void *workspace, size_t workspace_bytes,
                                       void *stream) {
    if (B < 0 || T < 0 || H < 0 || D < 0 || Ns < 0) return KLA_ERR_INVALID_ARG;
    if (!dtype_ok(in_dtype)) return KLA_ERR_UNSUPPORTED_DTYPE;
    if (!layer_shape_ok(D, Ns)) return KLA_ERR_INVALID_ARG;
    if ((lambda_T == nullptr) != (eta_T == nullptr)) return KLA_ERR_INVALID_ARG;
    int64_t BT = 0, BTH = 0, kq_elems = 0, vw_elems = 0, HD = 0, chans = 0, BH = 0;
    if (!mul_ok(B, T, &BT) || !mul_ok(BT, H, &BTH) || !mul_ok(BTH, Ns, &kq_elems) || !mul_ok(BTH, D, &vw_elems) ||
        !mul_ok(H, D, &HD) || !mul_ok(B, H, &BH) || !mul_ok(BH, D * Ns, &chans))
        return KLA_ERR_INVALID_ARG;
    if (chans == 0) return KLA_OK;
    const size_t esz = dtype_size(in_dtype);
    if (!a || !p || !lambda0 || !eta0) return KLA_ERR_INVALID_ARG;
    if (T > 0 && (!k || !q || !v || !w || !y)) return KLA_ERR_INVALID_ARG;
    const void *aligned_ins[4] = {k, q, v, w};
    for (int i = 0; i < 4; ++i)
        if (aligned_ins[i] && !aligned16(aligned_ins[i])) return KLA_ERR_INVALID_ARG;
    const Range outs[5] = {range_of(y, vw_elems * 4), range_of(s, vw_elems * 4), range_of(lambda_T, chans * 4),
                           range_of(eta_T, chans * 4), range_of(workspace, (int64_t)workspace_bytes)};
    const Range ins[8] = {range_of(k, kq_elems * (int64_t)esz), range_of(q, kq_elems * (int64_t)esz),
                          range_of(v, vw_elems * (int64_t)esz), range_of(w, vw_elems * (int64_t)esz),
                          range_of(a, HD * Ns * 4), range_of(p, HD * Ns * 4), range_of(lambda0, chans * 4),
                          range_of(eta0, chans * 4)};
    if (any_overlap(outs, 5, ins, 8)) return KLA_ERR_INVALID_ARG;
    size_t need = 0;
    if (kla_layer_forward_workspace_size(B, T, H, D, Ns, in_dtype, &need) != KLA_OK) return KLA_ERR_INVALID_ARG;
    if (need > 0 && (!workspace || workspace_bytes < need)) return KLA_ERR_WORKSPACE_TOO_SMALL;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return KLA_ERR_MISALIGNED;
    if (T > INT32_MAX - 64 || H > INT32_MAX || D > INT32_MAX || B > INT32_MAX) return KLA_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (T == 0) {
        // no tokens: the final state is the prior
        if (lambda_T) {
            if (cudaMemcpyAsync(lambda_T, lambda0, (size_t)chans * 4, cudaMemcpyDeviceToDevice, st) != cudaSuccess ||
                cudaMemcpyAsync(eta_T, eta0, (size_t)chans * 4, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
                return KLA_ERR_CUDA;
        }
        return KLA_OK;
    }
    const CUtensorMapDataType tdt =
        in_dtype == KLA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    kla::LayerMaps maps;
    std::memset(&maps, 0, sizeof(maps));
    if (!encode_layer_map(&maps.k, k, tdt, esz, B, T, H, Ns) || !encode_layer_map(&maps.q, q, tdt, esz, B, T, H, Ns))
        return KLA_ERR_CUDA;
    kla::LayerParams prm;
    std::memset(&prm, 0, sizeof(prm));
    prm.v = v; prm.w = w; prm.a = a; prm.p = p; prm.lam0 = lambda0; prm.eta0 = eta0;
    prm.y = y; prm.s = s; prm.lam_T = lambda_T; prm.eta_T = eta_T;
    prm.T = T; prm.H = (int)H; prm.D = (int)D;
    prm.dtiles = (int)(D / (32 / Ns));
    prm.ntiles = BH * prm.dtiles;
    prm.nchunks = (int)((T + kLayerL - 1) / kLayerL);
    prm.wait_ns = g_wait_ns.load();
    prm.parts = stream_parts(prm.ntiles, prm.nchunks);
    prm.chunks_per_part = (prm.nchunks + prm.parts - 1) / prm.parts;
    prm.nunits = prm.ntiles * prm.parts;
    unsigned char *ws = static_cast<unsigned char *>(workspace);
    prm.ticket = reinterpret_cast<unsigned *>(ws);
    if (prm.parts > 1) {
        const StreamWs sw = stream_ws_layout(prm.ntiles, prm.parts);
        if (sw.total > workspace_bytes) return KLA_ERR_WORKSPACE_TOO_SMALL;
        prm.part_flags = reinterpret_cast<unsigned *>(ws + sw.flags_off);
        prm.part_state = reinterpret_cast<float *>(ws + sw.state_off);
        if (launch_clear(ws, sw.clear_bytes, st) != cudaSuccess) return KLA_ERR_CUDA;
    }
    cudaError_t e;
    if (in_dtype == KLA_F32)
        e = Ns == 8 ? launch_layer<float, 8>(prm, maps, st) : launch_layer<float, 16>(prm, maps, st);
    else
        e = Ns == 8 ? launch_layer<__nv_bfloat16, 8>(prm, maps, st) : launch_layer<__nv_bfloat16, 16>(prm, maps, st);
    return e == cudaSuccess ? KLA_OK : KLA_ERR_CUDA;
}

KLA_API kla_status_t kla_layer_step(const void *k, const void *q, const void *v, const void *w,
                                    kla_dtype_t in_dtype, const float *a, const float *p, float *lambda_state,
                                    float *eta_state, float *y, float *s, int64_t B, int64_t H, int64_t D,
                                    int64_t Ns, void *stream) {
    if (B < 0 || H < 0 || D < 0 || Ns < 0) return KLA_ERR_INVALID_ARG;
    if (!dtype_ok(in_dtype)) return KLA_ERR_UNSUPPORTED_DTYPE;
    if (!layer_shape_ok(D, Ns)) return KLA_ERR_INVALID_ARG;
    int64_t BH = 0, DN = 0, C = 0, HDN = 0, BHD = 0;
    if (!mul_ok(B, H, &BH) || !mul_ok(D, Ns, &DN) || !mul_ok(BH, DN, &C) || !mul_ok(H, DN, &HDN) ||
        !mul_ok(BH, D, &BHD))
        return KLA_ERR_INVALID_ARG;
    if (C == 0) return KLA_OK;
    if (!k || !q || !v || !w || !a || !p || !lambda_state || !eta_state || !y) return KLA_ERR_INVALID_ARG;
    if (DN > INT32_MAX) return KLA_ERR_INVALID_ARG;
    const int64_t esz = (int64_t)dtype_size(in_dtype);
    const Range outs[4] = {range_of(lambda_state, C * 4), range_of(eta_state, C * 4), range_of(y, BHD * 4),
                           range_of(s, BHD * 4)};
    const Range ins[6] = {range_of(k, BH * Ns * esz), range_of(q, BH * Ns * esz), range_of(v, BHD * esz),
                          range_of(w, BHD * esz), range_of(a, HDN * 4), range_of(p, HDN * 4)};
    if (any_overlap(outs, 4, ins, 6)) return KLA_ERR_INVALID_ARG;
    kla::LayerStepParams prm;
    prm.k = k; prm.q = q; prm.v = v; prm.w = w; prm.a = a; prm.p = p;
    prm.lam = lambda_state; prm.eta = eta_state; prm.y = y; prm.s = s;
    prm.BH = BH; prm.H = (int)H; prm.D = (int)D; prm.DN = (int)DN;
    if (HDN > INT32_MAX || BH > INT32_MAX) return KLA_ERR_INVALID_ARG;
    const int threads = 256;
    const int64_t bx = (DN + threads - 1) / threads;
    // two CTAs per SM at most, grid-stride over the rows beyond (B=256, H=4,
    // D=32, Ns=16, graph of 256 steps: 4.13 us per token against 4.70 with
    // up to 16 per SM and 5.64 with 4, as for kla_scan_step)
    const int64_t by =
        std::max<int64_t>(1, std::min<int64_t>(BH, std::max<int64_t>(1, (int64_t)sm_count() * 2 / bx)));
    // programmatic dependent launch, as for kla_scan_step
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)bx, (unsigned)std::min<int64_t>(by, 65535));
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e;
    if (in_dtype == KLA_F32)
        e = Ns == 8 ? cudaLaunchKernelEx(&cfg, kla::kla_layer_step_kernel<float, 8>, prm)
                    : cudaLaunchKernelEx(&cfg, kla::kla_layer_step_kernel<float, 16>, prm);
    else
        e = Ns == 8 ? cudaLaunchKernelEx(&cfg, kla::kla_layer_step_kernel<__nv_bfloat16, 8>, prm)
                    : cudaLaunchKernelEx(&cfg, kla::kla_layer_step_kernel<__nv_bfloat16, 16>, prm);
    return e == cudaSuccess ? KLA_OK : KLA_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// The Kalman attention weights: kla_attention_weights (kernel in
// kla_attention.cuh).
// ---------------------------------------------------------------------------
KLA_API kla_status_t kla_attention_weights(const void *a, const void *p, kla_dtype_t in_dtype,
                                           const float *lambda_out, float *F, int64_t B, int64_t T,
                                           int64_t H, int64_t N, int64_t t0, int64_t span, int64_t W,
                                           void *stream) {
    if (B < 0 || T < 0 || H < 0 || N < 0 || t0 < 0 || span < 0) return KLA_ERR_INVALID_ARG;
    if (W < 1 || W > KLA_ATTENTION_MAX_WINDOW) return KLA_ERR_INVALID_ARG;
    if (!dtype_ok(in_dtype)) return KLA_ERR_UNSUPPORTED_DTYPE;
    if (t0 > T || span > T - t0) return KLA_ERR_INVALID_ARG;
    int64_t HN = 0, BT = 0, elems = 0;
    if (!mul_ok(H, N, &HN) || !mul_ok(B, T, &BT) || !mul_ok(BT, HN, &elems)) return KLA_ERR_INVALID_ARG;
    if (span == 0 || B == 0 || HN == 0) return KLA_OK;
    if (!a || !p || !lambda_out || !F) return KLA_ERR_INVALID_ARG;
    const int64_t nwin = (span + W - 1) / W;
    int64_t bw = 0, bww = 0, f_elems = 0, f_bytes = 0, in_bytes = 0, l_bytes = 0;
    if (!mul_ok(B, nwin, &bw) || !mul_ok(bw, W * W, &bww) || !mul_ok(bww, HN, &f_elems) ||
        !mul_ok(f_elems, 4, &f_bytes) || !mul_ok(elems, (int64_t)dtype_size(in_dtype), &in_bytes) ||
        !mul_ok(elems, 4, &l_bytes))
        return KLA_ERR_INVALID_ARG;
    const Range outs[1] = {range_of(F, f_bytes)};
    const Range ins[3] = {range_of(a, in_bytes), range_of(p, in_bytes), range_of(lambda_out, l_bytes)};
    if (any_overlap(outs, 1, ins, 3)) return KLA_ERR_INVALID_ARG;
    const bool vec4 = HN % 4 == 0 && aligned16(F);
    const int cw = vec4 ? 128 : 32;
    const int64_t nct = (HN + cw - 1) / cw;
    int64_t grid = 0;
    if (!mul_ok(bw, nct, &grid) || grid > kMaxGrid || nwin > INT32_MAX) return KLA_ERR_INVALID_ARG;
    kla::AttnParams prm;
    prm.a = a; prm.p = p; prm.lam = lambda_out; prm.F = F;
    prm.T = T; prm.HN = HN; prm.t0 = t0; prm.span = span;
    prm.W = (int)W; prm.nwin = (int)nwin; prm.nct = nct;
    const size_t smem = (size_t)W * cw * sizeof(float);  // <= 32 KB
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (in_dtype == KLA_F32) {
        if (vec4) kla::kla_attention_kernel<float, 4><<<(unsigned)grid, 256, smem, st>>>(prm);
        else kla::kla_attention_kernel<float, 1><<<(unsigned)grid, 256, smem, st>>>(prm);
    } else {
        if (vec4) kla::kla_attention_kernel<__nv_bfloat16, 4><<<(unsigned)grid, 256, smem, st>>>(prm);
        else kla::kla_attention_kernel<__nv_bfloat16, 1><<<(unsigned)grid, 256, smem, st>>>(prm);
    }
    return cudaGetLastError() == cudaSuccess ? KLA_OK : KLA_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// The convolutional form of deterministic time-invariant channels:
// kla_scan_forward_lti (kernels in kla_lti.cuh).
// ---------------------------------------------------------------------------
namespace {

// Chunk warps of the convolutional-form kernel (the chunk in registers is
// half the general scan's: phi and b only) and tokens per sub-block of its
// local convolutions.
#ifndef KLA_LTI_W
#define KLA_LTI_W 8
#endif
#ifndef KLA_LTI_S
#define KLA_LTI_S 8
#endif
constexpr int kLtiL = 32;

template <typename Tin>
constexpr int lti_stages() {
    constexpr int W = KLA_LTI_W;
    const int stage = 2 * kLtiL * 32 * (int)sizeof(Tin);
    const int fixed = W * 2 * 32 * 8 + W * 8 + 2048;
    const int ns = (KLA_STREAM_SMEM - fixed) / stage;
    return ns > KLA_STREAM_MAX_STAGES ? KLA_STREAM_MAX_STAGES : ns;
}

template <typename Tin>
cudaError_t launch_lti_stream(const kla::LtiParams &prm, const kla::LtiMaps &maps, cudaStream_t stream) {
    constexpr int NS = lti_stages<Tin>();
    using Cfg = kla::LtiTile<Tin, kLtiL, KLA_LTI_W, NS>;
    static_assert(NS >= KLA_LTI_W && Cfg::SMEM <= 227 * 1024, "convolutional-form kernel shared memory");
    auto kernel = kla::kla_lti_stream_kernel<Tin, kLtiL, KLA_LTI_S, KLA_LTI_W, NS>;
    cudaError_t e = ensure_smem_attr(kernel, Cfg::SMEM);
    if (e != cudaSuccess) return e;
    const int64_t grid = std::min<int64_t>(prm.nunits, sm_count());
    kernel<<<(unsigned)grid, Cfg::THREADS, Cfg::SMEM, stream>>>(prm, maps);
    return cudaGetLastError();
}

// Run-split workspace of the convolutional form: ticket, one flag per run
// boundary, fp64 (lambda, eta) of 32 channels per boundary.
StreamWs lti_ws_layout(int64_t ntiles, int parts) {
    StreamWs w;
    const size_t nb = (size_t)ntiles * (size_t)(parts - 1);
    w.flags_off = kHeaderBytes;
    w.state_off = w.flags_off + round_up(nb * sizeof(unsigned), 256);
    w.clear_bytes = w.state_off;
    w.total = w.state_off + round_up(nb * 64 * sizeof(double), 256);
    return w;
}

// 2: the streaming kernel (TMA loads as for the general streaming scan:
// 16-byte aligned phi and b, H*N*elem a multiple of 16 bytes, H*N >= 32,
// T >= 32); 1: one thread per channel (any shape).
int lti_kernel_choice(int64_t T, int64_t HN, size_t esz, const void *const *ptrs, int n) {
    bool ok = (HN * (int64_t)esz) % 16 == 0 && T >= kLtiL && HN >= 32 && encode_fn() != nullptr;
    for (int k = 0; k < n && ok; ++k)
        if (ptrs[k] && !aligned16(ptrs[k])) ok = false;
    return ok ? 2 : 1;
}

}  // namespace

KLA_API kla_status_t kla_scan_forward_lti_workspace_size(int64_t B, int64_t T, int64_t H, int64_t N,
                                                         kla_dtype_t in_dtype, size_t *bytes) {
    if (!bytes || B < 0 || T < 0 || H < 0 || N < 0) return KLA_ERR_INVALID_ARG;
    if (!dtype_ok(in_dtype)) return KLA_ERR_UNSUPPORTED_DTYPE;
    int64_t HN = 0, BT = 0, elems = 0;
    if (!mul_ok(H, N, &HN) || !mul_ok(B, T, &BT) || !mul_ok(BT, HN, &elems)) return KLA_ERR_INVALID_ARG;
    *bytes = elems == 0 ? 0 : lti_ws_layout(B * ((HN + 31) / 32), KLA_STREAM_MAX_PARTS).total;
    return KLA_OK;
}

KLA_API kla_status_t kla_scan_forward_lti(const float *a, const void *phi, const void *b, kla_dtype_t in_dtype,
                                          const float *lambda0, const float *eta0, float *lambda_out,
                                          float *eta_out, float *mu_out, float *var_out, int64_t B, int64_t T,
                                          int64_t H, int64_t N, void *workspace, size_t workspace_bytes,
                                          void *stream) {
    if (B < 0 || T < 0 || H < 0 || N < 0) return KLA_ERR_INVALID_ARG;
    if (!dtype_ok(in_dtype)) return KLA_ERR_UNSUPPORTED_DTYPE;
    int64_t HN = 0, C = 0, BT = 0, elems = 0;
    if (!mul_ok(H, N, &HN) || !mul_ok(B, HN, &C) || !mul_ok(B, T, &BT) || !mul_ok(BT, HN, &elems))
        return KLA_ERR_INVALID_ARG;
    if (elems == 0) return KLA_OK;
    if (!a || !phi || !b || !lambda0 || !eta0 || !lambda_out || !eta_out) return KLA_ERR_INVALID_ARG;
    const size_t esz = dtype_size(in_dtype);
    int64_t in_bytes = 0, out_bytes = 0;
    if (!mul_ok(elems, (int64_t)esz, &in_bytes) || !mul_ok(elems, 4, &out_bytes)) return KLA_ERR_INVALID_ARG;
    const Range outs[5] = {range_of(lambda_out, out_bytes), range_of(eta_out, out_bytes),
                           range_of(mu_out, out_bytes), range_of(var_out, out_bytes),
                           range_of(workspace, (int64_t)workspace_bytes)};
    const Range ins[5] = {range_of(a, C * 4), range_of(phi, in_bytes), range_of(b, in_bytes),
                          range_of(lambda0, C * 4), range_of(eta0, C * 4)};
    if (any_overlap(outs, 5, ins, 5)) return KLA_ERR_INVALID_ARG;
    size_t need = 0;
    if (kla_scan_forward_lti_workspace_size(B, T, H, N, in_dtype, &need) != KLA_OK) return KLA_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < need) return KLA_ERR_WORKSPACE_TOO_SMALL;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return KLA_ERR_MISALIGNED;
    if (T > INT32_MAX - 64 || HN > INT32_MAX || B > INT32_MAX) return KLA_ERR_INVALID_ARG;

    kla::LtiParams prm;
    std::memset(&prm, 0, sizeof(prm));
    prm.a = a; prm.lam0 = lambda0; prm.eta0 = eta0;
    prm.out[0] = lambda_out; prm.out[1] = eta_out; prm.out[2] = mu_out; prm.out[3] = var_out;
    prm.T = T; prm.HN = HN;
    prm.write_mu = mu_out != nullptr; prm.write_var = var_out != nullptr;
    prm.wait_ns = g_wait_ns.load();
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const void *ptrs[6] = {phi, b, lambda_out, eta_out, mu_out, var_out};
    if (lti_kernel_choice(T, HN, esz, ptrs, 2) == 2) {  // phi and b: the outputs are stored without TMA
        const CUtensorMapDataType tdt =
            in_dtype == KLA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
        kla::LtiMaps maps;
        std::memset(&maps, 0, sizeof(maps));
        const bool ok = encode_stream_map(&maps.in[0], phi, tdt, esz, B, T, HN, kLtiL) &&
                         encode_stream_map(&maps.in[1], b, tdt, esz, B, T, HN, kLtiL);
        if (ok) {
            prm.ntiles = B * ((HN + 31) / 32);
            prm.nct = (int)((HN + 31) / 32);
            prm.nchunks = (int)((T + kLtiL - 1) / kLtiL);
            prm.parts = stream_parts(prm.ntiles, prm.nchunks);
            prm.chunks_per_part = (prm.nchunks + prm.parts - 1) / prm.parts;
            prm.nunits = prm.ntiles * prm.parts;
            unsigned char *ws = static_cast<unsigned char *>(workspace);
            prm.ticket = reinterpret_cast<unsigned *>(ws);
            if (prm.parts > 1) {
                const StreamWs sw = lti_ws_layout(prm.ntiles, prm.parts);
                if (sw.total > workspace_bytes) return KLA_ERR_WORKSPACE_TOO_SMALL;
                prm.part_flags = reinterpret_cast<unsigned *>(ws + sw.flags_off);
                prm.part_state = reinterpret_cast<double *>(ws + sw.state_off);
                if (launch_clear(ws, sw.clear_bytes, st) != cudaSuccess) return KLA_ERR_CUDA;
            } else if (whole_tiles_ticketed(prm.ntiles, prm.nchunks)) {
                if (launch_clear(ws, lti_ws_layout(prm.ntiles, 1).clear_bytes, st) != cudaSuccess)
                    return KLA_ERR_CUDA;
            } else {
                prm.ticket = nullptr;  // round-robin units, no workspace
            }
            const cudaError_t e = in_dtype == KLA_F32 ? launch_lti_stream<float>(prm, maps, st)
                                                      : launch_lti_stream<__nv_bfloat16>(prm, maps, st);
            return e == cudaSuccess ? KLA_OK : KLA_ERR_CUDA;
        }
    }
    const int threads = 128;
    const int64_t blocks = (C + threads - 1) / threads;
    if (in_dtype == KLA_F32)
        kla::kla_lti_seq_kernel<float, KLA_LTI_S><<<(unsigned)blocks, threads, 0, st>>>(
            prm, phi, b, lambda_out, eta_out, mu_out, var_out, C);
    else
        kla::kla_lti_seq_kernel<__nv_bfloat16, KLA_LTI_S><<<(unsigned)blocks, threads, 0, st>>>(
            prm, phi, b, lambda_out, eta_out, mu_out, var_out, C);
    return cudaGetLastError() == cudaSuccess ? KLA_OK : KLA_ERR_CUDA;
}

KLA_API kla_status_t kla_scan_forward_lti_plan(int64_t B, int64_t T, int64_t H, int64_t N, kla_dtype_t in_dtype,
                                               const void *phi, const void *b, int *kernel, int *launches) {
    if (!kernel || !launches || B < 0 || T < 0 || H < 0 || N < 0) return KLA_ERR_INVALID_ARG;
    if (!dtype_ok(in_dtype)) return KLA_ERR_UNSUPPORTED_DTYPE;
    int64_t HN = 0, BT = 0, elems = 0;
    if (!mul_ok(H, N, &HN) || !mul_ok(B, T, &BT) || !mul_ok(BT, HN, &elems)) return KLA_ERR_INVALID_ARG;
    if (elems == 0) {
        *kernel = 0;
        *launches = 0;
        return KLA_OK;
    }
    const void *ptrs[2] = {phi, b};
    *kernel = lti_kernel_choice(T, HN, dtype_size(in_dtype), ptrs, 2);
    *launches = 1;
    const int64_t lnt = B * ((HN + 31) / 32), lnc = (T + kLtiL - 1) / kLtiL;
    if (*kernel == 2 && (stream_parts(lnt, lnc) > 1 || whole_tiles_ticketed(lnt, lnc))) *launches = 2;
    return KLA_OK;
}
