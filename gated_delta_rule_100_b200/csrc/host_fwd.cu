// host_fwd.cu -- kda_chunk_fwd_host: the prefill on HOST buffers (host code only).
//
// The token axis is cut into pieces of P tokens (a multiple of the 64-token
// chunk).  Piece i is copied host -> device into one of two staging slots on
// an upload stream, computed by kda_chunk_fwd on the caller's stream (its h0
// is the state the previous piece left, its hT the same buffer: the
// recurrence is exact across any token boundary, section 3.3 of "Kimi Linear's
// Hybrid Linear Attention Architecture: A Technical Breakdown"), and its
// output copied device -> host on a download stream.  Events order the three:
//   upload(i)   after compute(i - 2)   (slot inputs free)
//   compute(i)  after upload(i), download(i - 2)   (slot output free)
//   download(i) after compute(i)
// so uploads, computes and downloads of neighbouring pieces overlap and the
// call runs at the host link's upload rate (the link is full duplex).  One
// cudaMemcpyAsync per tensor and batch row; nothing else touches the data.
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "kda.h"

namespace {

constexpr int kStageDevices = 16;
constexpr size_t kPieceInputBytes = 256ull << 20;  // input bytes per piece, about
constexpr int kChunk = 64;

struct Stage {
    uint8_t *buf = nullptr;  // [2 slots][q k v g beta out], then the carried state
    size_t bytes = 0;
    cudaStream_t up = nullptr, down = nullptr;
    cudaEvent_t fork = nullptr, done = nullptr;
    cudaEvent_t uploaded[2] = {nullptr, nullptr}, computed[2] = {nullptr, nullptr},
                downloaded[2] = {nullptr, nullptr};
};
Stage g_stage[kStageDevices];
std::mutex g_stage_mu;
std::atomic<int> g_piece_tokens{0};  // test hook: 0 = automatic

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

// Byte sizes of one slot's arrays for pieces of P tokens.
struct SlotPlan {
    size_t q, k, v, g, beta, out, slot;
};
SlotPlan slot_plan(int B, int P, int H, int dk, int dv) {
    const size_t rows = (size_t)B * P * H;
    SlotPlan s;
    s.q = up256(rows * dk * 2);
    s.k = s.q;
    s.v = up256(rows * dv * 2);
    s.g = up256(rows * dk * 4);
    s.beta = up256(rows * 4);
    s.out = up256(rows * dv * 2);
    s.slot = s.q + s.k + s.v + s.g + s.beta + s.out;
    return s;
}

int piece_tokens(int B, int T, int H, int dk, int dv) {
    const int forced = g_piece_tokens.load();
    long long p;
    if (forced > 0) {
        p = forced;
    } else {
        const size_t per_token = (size_t)B * H * (2 * dk * 2 + dv * 2 + dk * 4 + 4);
        p = (long long)(kPieceInputBytes / per_token) / kChunk * kChunk;
        if (p < kChunk) p = kChunk;
    }
    return (int)(p < T ? p : T);
}

int reserve_stage(int dev, size_t bytes, Stage **out) {
    Stage &s = g_stage[dev];
    if (s.bytes < bytes) {
        if (s.buf != nullptr && cudaFree(s.buf) != cudaSuccess) return KDA_ERR_CUDA;
        s.buf = nullptr;
        s.bytes = 0;
        if (cudaMalloc(&s.buf, bytes) != cudaSuccess) return KDA_ERR_CUDA;
        s.bytes = bytes;
    }
    if (s.up == nullptr) {
        if (cudaStreamCreateWithFlags(&s.up, cudaStreamNonBlocking) != cudaSuccess ||
            cudaStreamCreateWithFlags(&s.down, cudaStreamNonBlocking) != cudaSuccess)
            return KDA_ERR_CUDA;
        cudaEvent_t *evs[8] = {&s.fork, &s.done, &s.uploaded[0], &s.uploaded[1], &s.computed[0], &s.computed[1],
                               &s.downloaded[0], &s.downloaded[1]};
        for (cudaEvent_t *e : evs)
            if (cudaEventCreateWithFlags(e, cudaEventDisableTiming) != cudaSuccess) return KDA_ERR_CUDA;
    }
    *out = &s;
    return KDA_OK;
}

// Tokens [t0, t0 + n) of every batch row of a [B][T][row bytes] host tensor,
// into a compact [B][n][row bytes] device array (or back, `down`).
cudaError_t copy_rows(void *dev_arr, const void *host_arr, size_t row_bytes, int B, int T, int t0, int n,
                      cudaStream_t st, bool down, void *host_dst = nullptr) {
    for (int b = 0; b < B; ++b) {
        const size_t hoff = ((size_t)b * T + t0) * row_bytes, doff = (size_t)b * n * row_bytes;
        cudaError_t e = down ? cudaMemcpyAsync(static_cast<uint8_t *>(host_dst) + hoff,
                                               static_cast<const uint8_t *>(dev_arr) + doff, (size_t)n * row_bytes,
                                               cudaMemcpyDeviceToHost, st)
                             : cudaMemcpyAsync(static_cast<uint8_t *>(dev_arr) + doff,
                                               static_cast<const uint8_t *>(host_arr) + hoff, (size_t)n * row_bytes,
                                               cudaMemcpyHostToDevice, st);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace

// Frees the staging of device `dev` (called by kda_release_workspace).
extern "C" int kda_release_host_staging(int dev) {
    if (dev < 0 || dev >= kStageDevices) return KDA_OK;
    std::lock_guard<std::mutex> lk(g_stage_mu);
    Stage &s = g_stage[dev];
    int st = KDA_OK;
    if (s.buf != nullptr && cudaFree(s.buf) != cudaSuccess) st = KDA_ERR_CUDA;
    s.buf = nullptr;
    s.bytes = 0;
    return st;
}

void kda_chunk_fwd_host_debug_piece(int tokens) { g_piece_tokens.store(tokens > 0 ? tokens : 0); }

int kda_chunk_fwd_host(const void *q, const void *k, const void *v, const float *g, const float *beta, float scale,
                       const float *h0, void *out, float *hT, int B, int T, int H, int dk, int dv, void *stream) {
    if (B < 1 || H < 1 || T < 0) return KDA_ERR_INVALID_ARG;
    if (T > 0 && (!q || !k || !v || !g || !beta || !out)) return KDA_ERR_INVALID_ARG;
    if ((dk != 64 && dk != 128) || (dv != 64 && dv != 128)) return KDA_ERR_UNSUPPORTED;
    if ((long long)B * H * 4 > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t state_bytes = (size_t)B * H * dk * dv * sizeof(float);
    if (T == 0) {  // nothing to scan: hT = h0 (or zero), once the stream's earlier work is done
        if (hT == nullptr) return KDA_OK;
        if (cudaStreamSynchronize(s) != cudaSuccess) return KDA_ERR_CUDA;
        if (h0 == nullptr) memset(hT, 0, state_bytes);
        else if (h0 != hT) memmove(hT, h0, state_bytes);
        return KDA_OK;
    }
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return KDA_ERR_CUDA;
    if (dev < 0 || dev >= kStageDevices) return KDA_ERR_UNSUPPORTED;

    const int P = piece_tokens(B, T, H, dk, dv);
    const SlotPlan sp = slot_plan(B, P, H, dk, dv);
    std::lock_guard<std::mutex> lk(g_stage_mu);
    Stage *st = nullptr;
    if (int r = reserve_stage(dev, 2 * sp.slot + up256(state_bytes), &st); r != KDA_OK) return r;
    float *state = reinterpret_cast<float *>(st->buf + 2 * sp.slot);

    // The previous call's staging use is ordered before this one; the copy streams
    // start after the caller's earlier work on `s`.
    if (cudaStreamWaitEvent(s, st->done, 0) != cudaSuccess || cudaEventRecord(st->fork, s) != cudaSuccess ||
        cudaStreamWaitEvent(st->up, st->fork, 0) != cudaSuccess ||
        cudaStreamWaitEvent(st->down, st->fork, 0) != cudaSuccess)
        return KDA_ERR_CUDA;
    int status = KDA_OK;
    if (h0 != nullptr && cudaMemcpyAsync(state, h0, state_bytes, cudaMemcpyHostToDevice, st->up) != cudaSuccess)
        status = KDA_ERR_CUDA;
    int i = 0;
    for (int t0 = 0; t0 < T && status == KDA_OK; t0 += P, ++i) {
        const int n = T - t0 < P ? T - t0 : P;
        const int b = i & 1;
        uint8_t *slot = st->buf + (size_t)b * sp.slot;
        uint8_t *dq = slot, *dk_ = dq + sp.q, *dv_ = dk_ + sp.k, *dg = dv_ + sp.v, *db = dg + sp.g, *dout = db + sp.beta;
        // upload piece i once compute(i - 2) has read the slot
        if (i >= 2 && cudaStreamWaitEvent(st->up, st->computed[b], 0) != cudaSuccess) { status = KDA_ERR_CUDA; break; }
        if (copy_rows(dq, q, (size_t)H * dk * 2, B, T, t0, n, st->up, false) != cudaSuccess ||
            copy_rows(dk_, k, (size_t)H * dk * 2, B, T, t0, n, st->up, false) != cudaSuccess ||
            copy_rows(dv_, v, (size_t)H * dv * 2, B, T, t0, n, st->up, false) != cudaSuccess ||
            copy_rows(dg, g, (size_t)H * dk * 4, B, T, t0, n, st->up, false) != cudaSuccess ||
            copy_rows(db, beta, (size_t)H * 4, B, T, t0, n, st->up, false) != cudaSuccess ||
            cudaEventRecord(st->uploaded[b], st->up) != cudaSuccess) {
            status = KDA_ERR_CUDA;
            break;
        }
        // compute piece i once it is uploaded and download(i - 2) has read the slot's output
        if (cudaStreamWaitEvent(s, st->uploaded[b], 0) != cudaSuccess ||
            (i >= 2 && cudaStreamWaitEvent(s, st->downloaded[b], 0) != cudaSuccess)) {
            status = KDA_ERR_CUDA;
            break;
        }
        const float *start = (i == 0 && h0 == nullptr) ? nullptr : state;
        status = kda_chunk_fwd(dq, dk_, dv_, reinterpret_cast<const float *>(dg), reinterpret_cast<const float *>(db),
                               scale, start, dout, state, B, n, H, dk, dv, s);
        if (status != KDA_OK) break;
        if (cudaEventRecord(st->computed[b], s) != cudaSuccess) { status = KDA_ERR_CUDA; break; }
        // download piece i's output
        if (cudaStreamWaitEvent(st->down, st->computed[b], 0) != cudaSuccess ||
            copy_rows(dout, nullptr, (size_t)H * dv * 2, B, T, t0, n, st->down, true, out) != cudaSuccess ||
            cudaEventRecord(st->downloaded[b], st->down) != cudaSuccess) {
            status = KDA_ERR_CUDA;
            break;
        }
    }
    if (status == KDA_OK && hT != nullptr &&
        cudaMemcpyAsync(hT, state, state_bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess)
        status = KDA_ERR_CUDA;
    // join: the caller's stream follows everything enqueued on the copy streams (on an
    // error path too, so that the next call cannot reuse staging under a copy in flight)
    if (cudaEventRecord(st->uploaded[0], st->up) != cudaSuccess || cudaEventRecord(st->downloaded[0], st->down) != cudaSuccess ||
        cudaStreamWaitEvent(s, st->uploaded[0], 0) != cudaSuccess || cudaStreamWaitEvent(s, st->downloaded[0], 0) != cudaSuccess)
        status = KDA_ERR_CUDA;
    if (cudaEventRecord(st->done, s) != cudaSuccess) status = KDA_ERR_CUDA;
    return status;
}
