// kla_host.cu -- the forward scan on HOST buffers, with the host<->device copies
// pipelined against the scan (C ABI: kla_scan_forward_host*).
//
// The sequence is cut into blocks of t_block tokens.  Block k goes through
// three stages on three streams: its inputs are copied to the device (copy
// stream), the scan runs on the caller's stream starting from the state
// leaving block k-1 -- the last row of that block's lambda / eta, exactly the
// continuation kla_scan_step uses -- and its outputs are copied back (a second
// copy stream).  Two device slots alternate, so the copy of block k+1 in, the
// scan of block k and the copy of block k-1 out overlap; host->device and
// device->host traffic use the two directions of the link at once.  The
// filter itself runs only in the kernels behind kla_scan_forward.
#include "kla.h"

#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#define KLA_API extern "C" __attribute__((visibility("default")))

namespace {

constexpr int kSlots = 2;
constexpr int kMaxDevices = 256;

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool mul_ok(int64_t a, int64_t b, int64_t *out) {
    if (a < 0 || b < 0) return false;
    if (a != 0 && b > INT64_MAX / a) return false;
    *out = a * b;
    return true;
}

// Two copy streams and the events that order the pipeline, made once per
// device (non-blocking streams, timing-free events).
struct DeviceQueues {
    bool ready = false;
    cudaStream_t h2d = nullptr, d2h = nullptr;
    cudaEvent_t loaded[kSlots], scanned[kSlots], stored[kSlots];
};

DeviceQueues *device_queues() {
    static std::mutex mu;
    static DeviceQueues q[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    DeviceQueues &d = q[dev];
    if (!d.ready) {
        if (cudaStreamCreateWithFlags(&d.h2d, cudaStreamNonBlocking) != cudaSuccess) return nullptr;
        if (cudaStreamCreateWithFlags(&d.d2h, cudaStreamNonBlocking) != cudaSuccess) return nullptr;
        for (int s = 0; s < kSlots; ++s) {
            if (cudaEventCreateWithFlags(&d.loaded[s], cudaEventDisableTiming) != cudaSuccess ||
                cudaEventCreateWithFlags(&d.scanned[s], cudaEventDisableTiming) != cudaSuccess ||
                cudaEventCreateWithFlags(&d.stored[s], cudaEventDisableTiming) != cudaSuccess)
                return nullptr;
        }
        d.ready = true;
    }
    return &d;
}

int64_t pick_block(int64_t T, int64_t t_block) {
    if (t_block > 0) return t_block < T ? t_block : T;
    // about sixty-four blocks (the first copy in and the last copy out are
    // not overlapped), whole chunks of 64 tokens, at least 64 tokens.  On the
    // long workload (4.3 GB each way) 64 blocks took 94-95 ms a call against
    // 101 ms for 16, 100 for 32, 98 for 128 and 106 for 8.
    int64_t tb = (T + 63) / 64;
    tb = (tb + 63) / 64 * 64;
    if (tb < 64) tb = 64;
    return tb < T ? tb : T;
}

struct HostLayout {
    int64_t tb = 0;              // tokens per block
    size_t in_block = 0;         // bytes of one input array block   [B, tb, HN]
    size_t out_block = 0;        // bytes of one output array block  [B, tb, HN] fp32
    size_t prior = 0;            // bytes of one prior array         [B, HN] fp32
    size_t slot = 0;             // 4 inputs + 4 outputs + 2 prior arrays, 256-aligned
    size_t scan_ws = 0;          // kla_scan_forward workspace for one block
    size_t total = 0;
};

kla_status_t host_layout(int64_t B, int64_t T, int64_t H, int64_t N, kla_dtype_t dt, int64_t t_block,
                         HostLayout *lay) {
    if (B < 0 || T < 0 || H < 0 || N < 0 || t_block < 0) return KLA_ERR_INVALID_ARG;
    if (dt != KLA_F32 && dt != KLA_BF16) return KLA_ERR_UNSUPPORTED_DTYPE;
    int64_t HN = 0, C = 0;
    if (!mul_ok(H, N, &HN) || !mul_ok(B, HN, &C)) return KLA_ERR_INVALID_ARG;
    lay->tb = pick_block(T, t_block);
    int64_t elems = 0;
    if (!mul_ok(C, lay->tb, &elems)) return KLA_ERR_INVALID_ARG;
    const size_t esz = dt == KLA_BF16 ? 2 : 4;
    lay->in_block = round_up((size_t)elems * esz, 256);
    lay->out_block = round_up((size_t)elems * 4, 256);
    lay->prior = round_up((size_t)C * 4, 256);
    lay->slot = 4 * lay->in_block + 4 * lay->out_block + 2 * lay->prior;
    size_t ws = 0;
    const kla_status_t st = kla_scan_forward_workspace_size(B, lay->tb, H, N, dt, &ws);
    if (st != KLA_OK) return st;
    lay->scan_ws = round_up(ws, 256);
    lay->total = kSlots * lay->slot + lay->scan_ws;
    return KLA_OK;
}

// Copy block rows [t0, t0 + tb) of a [B, T, HN] array between a host array and
// a dense device block [B, tb, HN] (one 2-D copy: B rows of tb * HN elements;
// the device block is dense for its own length, as the scan expects).
cudaError_t copy_block(void *dst, const void *src, bool to_device, int64_t B, int64_t T, int64_t HN,
                       int64_t t0, int64_t tb, size_t esz, cudaStream_t s) {
    const size_t row = (size_t)(tb * HN) * esz;
    const size_t host_pitch = (size_t)(T * HN) * esz;
    const size_t dev_pitch = row;
    const size_t host_off = (size_t)(t0 * HN) * esz;
    if (to_device)
        return cudaMemcpy2DAsync(dst, dev_pitch, static_cast<const char *>(src) + host_off, host_pitch, row,
                                 (size_t)B, cudaMemcpyHostToDevice, s);
    return cudaMemcpy2DAsync(static_cast<char *>(dst) + host_off, host_pitch, src, dev_pitch, row, (size_t)B,
                             cudaMemcpyDeviceToHost, s);
}

}  // namespace

KLA_API kla_status_t kla_scan_forward_host_workspace_size(int64_t B, int64_t T, int64_t H, int64_t N,
                                                          kla_dtype_t in_dtype, int64_t t_block,
                                                          size_t *bytes) {
    if (!bytes) return KLA_ERR_INVALID_ARG;
    HostLayout lay;
    const kla_status_t st = host_layout(B, T, H, N, in_dtype, t_block, &lay);
    if (st != KLA_OK) return st;
    *bytes = (B == 0 || T == 0 || H * N == 0) ? 0 : lay.total;
    return KLA_OK;
}

KLA_API kla_status_t kla_scan_forward_host(const void *a, const void *p, const void *phi, const void *b,
                                           kla_dtype_t in_dtype, const float *lambda0, const float *eta0,
                                           float *lambda_out, float *eta_out, float *mu_out, float *var_out,
                                           int64_t B, int64_t T, int64_t H, int64_t N, int64_t t_block,
                                           void *workspace, size_t workspace_bytes, void *stream) {
    HostLayout lay;
    kla_status_t st = host_layout(B, T, H, N, in_dtype, t_block, &lay);
    if (st != KLA_OK) return st;
    const int64_t HN = H * N;
    if (B == 0 || T == 0 || HN == 0) return KLA_OK;
    if (!a || !p || !phi || !b || !lambda0 || !eta0 || !lambda_out || !eta_out) return KLA_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < lay.total) return KLA_ERR_WORKSPACE_TOO_SMALL;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return KLA_ERR_MISALIGNED;
    DeviceQueues *q = device_queues();
    if (!q) return KLA_ERR_CUDA;

    const size_t esz = in_dtype == KLA_BF16 ? 2 : 4;
    const int64_t C = B * HN;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    char *ws = static_cast<char *>(workspace);
    char *scan_ws = ws + kSlots * lay.slot;
    const void *ins[4] = {a, p, phi, b};
    float *outs[4] = {lambda_out, eta_out, mu_out, var_out};
    const int64_t nblocks = (T + lay.tb - 1) / lay.tb;

    struct Slot {
        char *in[4];
        float *out[4];
        float *lam0, *eta0;
    } slot[kSlots];
    for (int s = 0; s < kSlots; ++s) {
        char *base = ws + s * lay.slot;
        for (int k = 0; k < 4; ++k) slot[s].in[k] = base + k * lay.in_block;
        for (int k = 0; k < 4; ++k)
            slot[s].out[k] = reinterpret_cast<float *>(base + 4 * lay.in_block + k * lay.out_block);
        slot[s].lam0 = reinterpret_cast<float *>(base + 4 * lay.in_block + 4 * lay.out_block);
        slot[s].eta0 = reinterpret_cast<float *>(base + 4 * lay.in_block + 4 * lay.out_block + lay.prior);
    }

    // the copy streams start after everything already enqueued on the caller's stream
    if (cudaEventRecord(q->scanned[1], cs) != cudaSuccess) return KLA_ERR_CUDA;
    if (cudaStreamWaitEvent(q->h2d, q->scanned[1], 0) != cudaSuccess) return KLA_ERR_CUDA;
    if (cudaStreamWaitEvent(q->d2h, q->scanned[1], 0) != cudaSuccess) return KLA_ERR_CUDA;

    for (int64_t k = 0; k < nblocks; ++k) {
        const int s = (int)(k % kSlots);
        const int64_t t0 = k * lay.tb;
        const int64_t tb = T - t0 < lay.tb ? T - t0 : lay.tb;
        Slot &S = slot[s];
        // 1. inputs in: the slot's previous scan must be done with them
        if (k >= kSlots && cudaStreamWaitEvent(q->h2d, q->scanned[s], 0) != cudaSuccess) return KLA_ERR_CUDA;
        for (int i = 0; i < 4; ++i)
            if (copy_block(S.in[i], ins[i], true, B, T, HN, t0, tb, esz, q->h2d) != cudaSuccess)
                return KLA_ERR_CUDA;
        if (k == 0) {
            if (cudaMemcpyAsync(S.lam0, lambda0, (size_t)C * 4, cudaMemcpyHostToDevice, q->h2d) != cudaSuccess ||
                cudaMemcpyAsync(S.eta0, eta0, (size_t)C * 4, cudaMemcpyHostToDevice, q->h2d) != cudaSuccess)
                return KLA_ERR_CUDA;
        }
        if (cudaEventRecord(q->loaded[s], q->h2d) != cudaSuccess) return KLA_ERR_CUDA;

        // 2. scan on the caller's stream, entering with the state that left block k-1
        if (cudaStreamWaitEvent(cs, q->loaded[s], 0) != cudaSuccess) return KLA_ERR_CUDA;
        if (k >= kSlots && cudaStreamWaitEvent(cs, q->stored[s], 0) != cudaSuccess) return KLA_ERR_CUDA;
        if (k > 0) {
            const Slot &P = slot[1 - s];
            const int64_t tbp = lay.tb;  // every block before the last is full (dense [B, tbp, HN])
            for (int i = 0; i < 2; ++i) {
                float *dst = i == 0 ? S.lam0 : S.eta0;
                const float *src = P.out[i] + (tbp - 1) * HN;  // last row of batch 0
                if (cudaMemcpy2DAsync(dst, (size_t)HN * 4, src, (size_t)(tbp * HN) * 4, (size_t)HN * 4,
                                      (size_t)B, cudaMemcpyDeviceToDevice, cs) != cudaSuccess)
                    return KLA_ERR_CUDA;
            }
        }
        st = kla_scan_forward(S.in[0], S.in[1], S.in[2], S.in[3], in_dtype, S.lam0, S.eta0, S.out[0], S.out[1],
                              mu_out ? S.out[2] : nullptr, var_out ? S.out[3] : nullptr, B, tb, H, N, scan_ws,
                              lay.scan_ws, cs);
        if (st != KLA_OK) return st;
        if (cudaEventRecord(q->scanned[s], cs) != cudaSuccess) return KLA_ERR_CUDA;

        // 3. outputs out
        if (cudaStreamWaitEvent(q->d2h, q->scanned[s], 0) != cudaSuccess) return KLA_ERR_CUDA;
        for (int i = 0; i < 4; ++i)
            if (outs[i] && copy_block(outs[i], S.out[i], false, B, T, HN, t0, tb, 4, q->d2h) != cudaSuccess)
                return KLA_ERR_CUDA;
        if (cudaEventRecord(q->stored[s], q->d2h) != cudaSuccess) return KLA_ERR_CUDA;
    }
    // the caller's stream covers the whole call: wait for the last copies out
    for (int s = 0; s < kSlots && s < nblocks; ++s)
        if (cudaStreamWaitEvent(cs, q->stored[s], 0) != cudaSuccess) return KLA_ERR_CUDA;
    return KLA_OK;
}
