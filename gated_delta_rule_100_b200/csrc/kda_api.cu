// kda_api.cu -- the extern "C" boundary of libkda: argument validation,
// TMA descriptor encoding, kernel launch, and the per-device status word.
// Declarations and the contract of every entry point are in include/kda.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include <atomic>
#include <mutex>
#include <utility>
#include <vector>

#include "../../include/kda.h"
#include "kda_device.cuh"

namespace kda {
cudaError_t launch_decode(const void *q, const void *k, const void *v, const float *g,
                          const float *beta, float scale, float *state, void *out, int BH, int dk,
                          int dv, int g_dk, int prologue, float gate_c, cudaStream_t stream);
}

#include "bwd_params.cuh"
#include "chunk_common.cuh"
#include "chunk_params.cuh"

namespace kda {
cudaError_t launch_prep(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tg, const PrepParams &prm,
                        int dk, int max_ctas, cudaStream_t stream, bool prologue);
cudaError_t launch_chain(const CUtensorMap *maps, const ChainParams &prm, int dk, cudaStream_t stream,
                         cudaEvent_t started = nullptr);
cudaError_t launch_exact(const ExactParams &prm, int dk, int ctas, cudaStream_t stream);
cudaError_t launch_parts_fixup(float *start, const float *local, const float *trans, int BH, int dk, int dv,
                               int parts, cudaStream_t stream, unsigned long long *stamp);
cudaError_t launch_bwd(const BwdParams &prm, int dk, int dv, cudaStream_t stream);
size_t bwd_ckpt_bytes(int B, int T, int H, int dk, int dv);
cudaError_t launch_varlen_setup(const int *cu, int N, int T_total, int cmax, int *cu_s, int *cc, int *chunk_seq,
                                const DeviceStatus &st, cudaStream_t stream);
}

// Device-side status word: kernels OR error bits into it (one per device,
// part of this module's image, so nothing is allocated for it).
__device__ uint32_t g_kda_status_word;

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
uint32_t *g_status_ptr[kMaxDevices] = {};
std::atomic<unsigned long long> g_wait_polls{0};
std::atomic<unsigned long long> g_inject_polls{0};
std::atomic<int> g_force_exact{0};
std::atomic<int> g_block_refs{0};  // test hook: prep's block references for every chunk
std::atomic<int> g_parts_override{0};  // test hook: parts of the two-level pass (0 = automatic, 1 = off)
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

int current_status_word(uint32_t **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KDA_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_status_ptr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_kda_status_word) != cudaSuccess) return KDA_ERR_CUDA;
        g_status_ptr[dev] = static_cast<uint32_t *>(p);
    }
    *out = g_status_ptr[dev];
    return KDA_OK;
}

int get_encoder(PFN_cuTensorMapEncodeTiled_v12000 *fn) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_encode == nullptr) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || p == nullptr)
            return KDA_ERR_CUDA;
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    *fn = g_encode;
    return KDA_OK;
}

// Per-device workspace of the prefill: the per-chunk records passed from the
// prep kernel to the chain kernel, the prep kernel's item counters, and a
// state buffer carried between segments.  Grown on demand (cudaFree
// synchronises the device, so no kernel still reads the old buffer) and kept
// for later calls.  Calls on different streams are ordered on it by `done`,
// recorded after each call's last kernel and waited on by the next call's
// stream.
//
// A sequence whose records fit the cap runs as one segment (prep, then chain,
// on the caller's stream).  A longer one runs in segments over two record
// buffers so that the prep kernel of segment i + 1 overlaps the chain kernel
// of segment i: prep on a low-priority internal stream, chain on a
// high-priority one (its few CTAs are placed first, prep fills the other SMs).
constexpr size_t kWorkspaceCap = size_t(2) << 30;  // bytes of records
std::atomic<unsigned long long> g_record_cap{0};   // test hook: a smaller cap (0 = kWorkspaceCap)
size_t record_cap() {
    const unsigned long long c = g_record_cap.load();
    return c ? (size_t)c : kWorkspaceCap;
}
constexpr size_t kTicketBytes = 256;               // per record buffer: item counter, steep-item count
struct Workspace {
    uint8_t *base = nullptr;  // [counters][steep-item list][records]
    size_t base_bytes = 0;
    float *state = nullptr;
    size_t state_bytes = 0;
    float *parts = nullptr;  // the two-level pass: start, local and transition states of every part
    size_t parts_bytes = 0;
    float *ckpt = nullptr;   // the backward pass: state checkpoints
    size_t ckpt_bytes = 0;
    cudaEvent_t done = nullptr;
    cudaStream_t lo = nullptr, hi = nullptr;  // prep and chain streams of the segmented path
    cudaEvent_t fork = nullptr, prep_done[2] = {nullptr, nullptr}, chain_done[2] = {nullptr, nullptr};
    cudaEvent_t chain_go = nullptr;  // every CTA of a segment's first chain launch has begun
};
Workspace g_ws[kMaxDevices];

size_t rec_row_bytes(int B, int H) { return (size_t)B * H * kda::REC_BYTES; }
size_t round256(size_t x) { return (x + 255) & ~size_t(255); }
// The list of steep items of one segment (prep appends, the exact kernel reads):
// room for every item of the segment.
size_t steep_list_bytes(int B, int H, int seg) { return round256((size_t)B * H * seg * sizeof(int)); }

struct SegPlan {
    int nchunks, seg, nbuf;  // chunks, chunks per segment, record buffers
};
SegPlan plan_segments(int B, int T, int H) {
    SegPlan p;
    p.nchunks = (T + kda::CH - 1) / kda::CH;
    const size_t row = rec_row_bytes(B, H);
    const size_t cap = record_cap();
    if ((size_t)p.nchunks * row <= cap) {
        p.seg = p.nchunks;
        p.nbuf = 1;
    } else {
        const size_t fit = cap / (2 * row);
        p.seg = (int)(fit < 1 ? 1 : fit);
        p.nbuf = 2;
    }
    return p;
}

// Packed batches: global chunks bounded by cmax = T_total / 64 + N + 1 (each
// sequence adds at most one partial chunk), run in windows of W chunks.
struct VarlenPlan {
    int cmax, W, nwin;
};
VarlenPlan plan_varlen(int N, int T_total, int H) {
    VarlenPlan p;
    p.cmax = T_total / kda::CH + N + 1;
    const size_t fit = record_cap() / rec_row_bytes(1, H);
    p.W = (int)((size_t)p.cmax < fit ? (size_t)p.cmax : (fit < 1 ? 1 : fit));
    p.nwin = (p.cmax + p.W - 1) / p.W;
    return p;
}
// cu_s and cc ([N + 1] each) and chunk_seq ([cmax]), 256-byte rounded.
size_t varlen_meta_bytes(int N, int cmax) { return round256((size_t)(2 * (N + 1) + cmax) * sizeof(int)); }
size_t varlen_base_bytes(int N, int H, const VarlenPlan &pl) {
    return kTicketBytes + steep_list_bytes(1, H, pl.W) + varlen_meta_bytes(N, pl.cmax) +
           (size_t)pl.W * rec_row_bytes(1, H);
}

// Called with g_mu held.
int reserve_workspace(int dev, size_t base_bytes, size_t state_bytes, bool streams, Workspace **out,
                      size_t parts_bytes = 0) {
    Workspace &w = g_ws[dev];
    if (w.parts_bytes < parts_bytes) {
        if (w.parts != nullptr && cudaFree(w.parts) != cudaSuccess) return KDA_ERR_CUDA;
        w.parts = nullptr;
        w.parts_bytes = 0;
        if (cudaMalloc(&w.parts, parts_bytes) != cudaSuccess) return KDA_ERR_CUDA;
        w.parts_bytes = parts_bytes;
    }
    if (w.base_bytes < base_bytes) {
        if (w.base != nullptr && cudaFree(w.base) != cudaSuccess) return KDA_ERR_CUDA;
        w.base = nullptr;
        w.base_bytes = 0;
        if (cudaMalloc(&w.base, base_bytes) != cudaSuccess) return KDA_ERR_CUDA;
        w.base_bytes = base_bytes;
    }
    if (w.state_bytes < state_bytes) {
        if (w.state != nullptr && cudaFree(w.state) != cudaSuccess) return KDA_ERR_CUDA;
        w.state = nullptr;
        w.state_bytes = 0;
        if (cudaMalloc(&w.state, state_bytes) != cudaSuccess) return KDA_ERR_CUDA;
        w.state_bytes = state_bytes;
    }
    if (w.done == nullptr && cudaEventCreateWithFlags(&w.done, cudaEventDisableTiming) != cudaSuccess)
        return KDA_ERR_CUDA;
    if (streams && w.lo == nullptr) {
        int least = 0, greatest = 0;
        if (cudaDeviceGetStreamPriorityRange(&least, &greatest) != cudaSuccess ||
            cudaStreamCreateWithPriority(&w.lo, cudaStreamNonBlocking, least) != cudaSuccess ||
            cudaStreamCreateWithPriority(&w.hi, cudaStreamNonBlocking, greatest) != cudaSuccess)
            return KDA_ERR_CUDA;
        cudaEvent_t *evs[6] = {&w.fork, &w.prep_done[0], &w.prep_done[1], &w.chain_done[0], &w.chain_done[1],
                               &w.chain_go};
        for (cudaEvent_t *e : evs)
            if (cudaEventCreateWithFlags(e, cudaEventDisableTiming) != cudaSuccess) return KDA_ERR_CUDA;
    }
    *out = &w;
    return KDA_OK;
}

// Per-kernel timing hook (measurement only).  While enabled, every prefill
// kernel launch gets a slot in the device's stamp array, set to all ones on the
// launching stream just before the launch; the kernel's CTAs fold their
// %globaltimer start and end into it (see stamp_start / stamp_end), so a slot
// ends as the launch's busy interval on the device.  The kernels' own stamps
// add two atomics per CTA and nothing to the streams' ordering, unlike events
// around each launch.
constexpr int kMaxStamps = 8192;  // launches timed between two reads, per device
struct TimedLaunch {
    int dev, kind, slot;
};
std::atomic<int> g_timing{0};
std::vector<TimedLaunch> g_timed;  // recorded, not yet read
int g_stamp_next[kMaxDevices] = {};
unsigned long long *g_stamp_ptr[kMaxDevices] = {};

}  // namespace

__device__ unsigned long long g_kda_stamps[2 * kMaxStamps];

namespace {

// Launch `fn(stamp)` on `s`; stamp is the launch's timing slot, or NULL when
// the hook is off (or every slot is taken).  Called with g_mu held.
template <class F>
cudaError_t timed_launch(int dev, int kind, cudaStream_t s, F &&fn) {
    if (!g_timing.load()) return fn(nullptr);
    if (g_stamp_ptr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_kda_stamps) != cudaSuccess) return cudaErrorUnknown;
        g_stamp_ptr[dev] = static_cast<unsigned long long *>(p);
    }
    if (g_stamp_next[dev] >= kMaxStamps) return fn(nullptr);
    const int slot = g_stamp_next[dev]++;
    unsigned long long *st = g_stamp_ptr[dev] + 2 * slot;
    cudaError_t e = cudaMemsetAsync(st, 0xFF, 2 * sizeof(unsigned long long), s);
    if (e != cudaSuccess) return e;
    e = fn(st);
    g_timed.push_back({dev, kind, slot});
    return e;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// 4-D map over a [B][T][H][inner] tensor; box {box_inner, 1, 64, 1}.
int make_map(CUtensorMap *map, PFN_cuTensorMapEncodeTiled_v12000 enc, const void *ptr,
             CUtensorMapDataType dt, int esize, int inner, int H, int T, int B, int box_inner,
             CUtensorMapSwizzle swz) {
    cuuint64_t dims[4] = {(cuuint64_t)inner, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)inner * esize, (cuuint64_t)H * inner * esize,
                             (cuuint64_t)T * H * inner * esize};
    cuuint32_t box[4] = {(cuuint32_t)box_inner, 1u, 64u, 1u};
    cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
    CUresult r = enc(map, dt, 4, const_cast<void *>(ptr), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? KDA_OK : KDA_ERR_CUDA;
}

// Streaming multiprocessors of a device (cached; its own lock, so callers may hold g_mu).
std::mutex g_sms_mu;
int g_num_sms[kMaxDevices] = {};
int num_sms(int dev) {
    std::lock_guard<std::mutex> lk(g_sms_mu);
    if (g_num_sms[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) n = 148;
        g_num_sms[dev] = n;
    }
    return g_num_sms[dev];
}

// Tensor maps over the record parts of `nrec` consecutive records at `rec`
// (layouts in chunk_common.cuh), with the boxes and swizzles of the chain
// kernel's operand tiles.
int make_rec_maps(PFN_cuTensorMapEncodeTiled_v12000 enc, const uint8_t *rec, long long nrec, int dk,
                  CUtensorMap *maps) {
    // WQ, P, K-hat: [blocks][rows][16] 16-bit arrays, one box = one record's part
    // (4-D: token-in-block, row, block, record), 32-byte swizzle
    struct Part { size_t off; CUtensorMapDataType dt; int rows, blocks; };
    const Part parts[3] = {{(size_t)kda::REC_WQ, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, dk, 8},
                           {(size_t)kda::REC_P, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, kda::CH, 4},
                           {(size_t)kda::REC_KH, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 128, 4}};
    cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
    for (int i = 0; i < 3; ++i) {
        const Part &p = parts[i];
        cuuint64_t dims[4] = {(cuuint64_t)kda::SUB, (cuuint64_t)p.rows, (cuuint64_t)p.blocks, (cuuint64_t)nrec};
        cuuint64_t strides[3] = {(cuuint64_t)kda::SUB * 2, (cuuint64_t)kda::SUB * 2 * p.rows, (cuuint64_t)kda::REC_BYTES};
        cuuint32_t box[4] = {(cuuint32_t)kda::SUB, (cuuint32_t)p.rows, (cuuint32_t)p.blocks, 1u};
        CUresult r = enc(&maps[i], p.dt, 4, const_cast<uint8_t *>(rec + p.off), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return KDA_ERR_CUDA;
    }
    // T': fp32 [64][64] row-major, boxes of 32 columns, 128-byte swizzle
    cuuint64_t dims[3] = {(cuuint64_t)kda::CH, (cuuint64_t)kda::CH, (cuuint64_t)nrec};
    cuuint64_t strides[2] = {(cuuint64_t)kda::CH * 4, (cuuint64_t)kda::REC_BYTES};
    cuuint32_t box[3] = {32u, (cuuint32_t)kda::CH, 1u};
    CUresult r = enc(&maps[3], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<uint8_t *>(rec + kda::REC_T), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? KDA_OK : KDA_ERR_CUDA;
}

// Value-column slices per (b, h) in the chain kernel.  Every CTA of a (b, h)
// reads all of that (b, h)'s records, so one 128-column CTA reads them once;
// two 64-column CTAs halve the per-chunk work on the sequential path.  Use the
// narrow slices when they still fit one CTA per SM (few (b, h): latency
// matters), the wide one otherwise (many (b, h): record traffic matters).
int chain_slices(int B, int H, int dv, int sms) { return (dv == 128 && 2LL * B * H <= sms) ? 2 : 1; }

// Parts of the two-level pass for a segment of `cnt` chunks.  The plain pass
// keeps each (b, h)'s chain on one CTA per value slice walking every chunk in
// order; with few (b, h) most SMs idle meanwhile.  The two-level pass runs
// pass A on (parts - 1) x (dv + dk) / 64 CTAs per (b, h) and pass B on
// (parts - 1) x dv / 64, so the sequential walk shrinks to two parts' worth of
// chunks plus the short fix-up.  Parts are chosen so that pass A fits in one
// wave and each part holds at least kMinPartChunks chunks (below that the two
// extra launches and the fix-up cost more than the walk saves: on the B200,
// B1 H4 T2048 took 0.158 ms in 8 parts of 4 chunks against 0.113 ms plain);
// fewer than 3 parts gain nothing, so then the plain pass runs (1 is returned).
constexpr int kMinPartChunks = 16;
int plan_parts(int B, int H, int dk, int dv, int cnt, int sms) {
    const int ov = g_parts_override.load();
    int P;
    if (ov >= 1) {
        P = ov;
    } else {
        const long long per_part = (long long)B * H * ((dv + dk) / 64);
        P = (int)(1 + sms / per_part);
        if (P > cnt / kMinPartChunks) P = cnt / kMinPartChunks;
    }
    if (P > cnt) P = cnt;
    if (P < 3) return 1;
    const int len = (cnt + P - 1) / P;
    return (cnt + len - 1) / len;  // parts actually used at that length
}
size_t parts_bytes(int B, int H, int dk, int dv, int P) {
    return P < 3 ? 0 : (size_t)P * B * H * dk * (2 * dv + dk) * sizeof(float);
}

// Chain launch fields of the plain pass.
void plain_pass(kda::ChainParams &cp, int nslices) {
    cp.nslices = nslices;
    cp.parts = 1;
    cp.part_len = 0;
    cp.part0 = 0;
    cp.nparts = 1;
    cp.slots = nslices;
    cp.pass_a = 0;
    cp.p_start = cp.p_local = cp.p_trans = nullptr;
    cp.stamp = nullptr;
}

// Geometry of a uniform launch: B sequences of T tokens, local chunks [n0, n0 + cnt).
kda::SeqGeom uniform_geom(int B, int T, int n0, int cnt) {
    kda::SeqGeom gm = {};
    gm.cu = nullptr;
    gm.nseqs = B;
    gm.T = T;
    gm.n_begin = n0;
    gm.nseg = cnt;
    return gm;
}

// Parameters of the exact kernel for the items of one prep launch.
kda::ExactParams exact_params(const void *q, const void *k, const float *g, int g_dk, const float *beta,
                              const kda::PrepParams &pp, bool prologue = false) {
    kda::ExactParams xp;
    xp.q = static_cast<const uint16_t *>(q);
    xp.k = static_cast<const uint16_t *>(k);
    xp.g = g;
    xp.g_dk = g_dk;
    xp.beta = beta;
    xp.ws = pp.ws;
    xp.nrec = pp.nrec;
    xp.st = pp.st;
    xp.steep_count = pp.steep_count;
    xp.steep_items = pp.steep_items;
    xp.prologue = prologue ? 1 : 0;
    xp.stamp = nullptr;
    xp.gate_c = pp.gate_c;
    xp.H = pp.H;
    xp.gm = pp.gm;
    return xp;
}

}  // namespace

extern "C" {

int kda_abi_version(void) { return 104; }

const char *kda_status_string(int status) {
    switch (status) {
        case KDA_OK: return "KDA_OK";
        case KDA_ERR_INVALID_ARG: return "KDA_ERR_INVALID_ARG";
        case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED";
        case KDA_ERR_ALIGNMENT: return "KDA_ERR_ALIGNMENT";
        case KDA_ERR_CUDA: return "KDA_ERR_CUDA";
        case KDA_ERR_TIMEOUT: return "KDA_ERR_TIMEOUT";
        case KDA_ERR_SCRATCH_LIMIT: return "KDA_ERR_SCRATCH_LIMIT";
        case KDA_ERR_BOUNDS: return "KDA_ERR_BOUNDS";
        default: return "KDA_ERR_UNKNOWN";
    }
}

void kda_chunk_fwd_debug_wait_limit(unsigned long long polls) { g_wait_polls.store(polls); }

void kda_chunk_fwd_debug_inject_timeout(unsigned long long polls) { g_inject_polls.store(polls); }

void kda_chunk_fwd_debug_force_exact(int enable) { g_force_exact.store(enable != 0); }

void kda_chunk_fwd_debug_block_refs(int enable) { g_block_refs.store(enable != 0); }

void kda_chunk_fwd_debug_record_cap(unsigned long long bytes) { g_record_cap.store(bytes); }

void kda_chunk_fwd_debug_parts(int parts) { g_parts_override.store(parts < 0 ? 0 : parts); }

int kda_stream_status(void *stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return KDA_ERR_CUDA;
    uint32_t *word = nullptr;
    if (current_status_word(&word) != KDA_OK) return KDA_ERR_CUDA;
    uint32_t v = 0;
    if (cudaMemcpy(&v, word, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return KDA_ERR_CUDA;
    if (v != 0) {
        const uint32_t zero = 0;
        if (cudaMemcpy(word, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return KDA_ERR_CUDA;
    }
    if (v & kda::DEV_TIMEOUT) return KDA_ERR_TIMEOUT;
    if (v & kda::DEV_BOUNDS) return KDA_ERR_BOUNDS;
    return (v & kda::DEV_BAD_ARG) ? KDA_ERR_INVALID_ARG : KDA_OK;
}

// The prefill for either gate form: g_dk = dk (g [B, T, H, dk]) or 1 (g [B, T, H]).
// prologue: g, beta, q, k are raw projections (per-channel gate only), g = -gate_c softplus(g).
static int chunk_fwd_impl(const void *q, const void *k, const void *v, const float *g, const float *beta,
                          float scale, const float *h0, void *out, float *hT, int B, int T, int H, int dk,
                          int dv, void *stream, bool scalar_gate, bool prologue = false, float gate_c = 0.f) {
    if (B < 1 || H < 1 || T < 0) return KDA_ERR_INVALID_ARG;
    if (T > 0 && (!q || !k || !v || !g || !beta || !out)) return KDA_ERR_INVALID_ARG;
    if ((dk != 64 && dk != 128) || (dv != 64 && dv != 128)) return KDA_ERR_UNSUPPORTED;
    const int g_dk = scalar_gate ? 1 : dk;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !(scalar_gate ? aligned4(g) : aligned16(g)) ||
        !aligned4(beta) || !aligned16(out) || !aligned16(h0) || !aligned16(hT))
        return KDA_ERR_ALIGNMENT;
    if ((long long)B * H * 4 > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    if (T == 0) {  // nothing to scan: hT = h0 (or zero)
        if (hT == nullptr) return KDA_OK;
        const size_t bytes = (size_t)B * H * dk * dv * sizeof(float);
        cudaError_t e = h0 ? (h0 == hT ? cudaSuccess : cudaMemcpyAsync(hT, h0, bytes, cudaMemcpyDeviceToDevice, s))
                           : cudaMemsetAsync(hT, 0, bytes, s);
        return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
    }

    uint32_t *word = nullptr;
    if (current_status_word(&word) != KDA_OK) return KDA_ERR_CUDA;
    PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
    if (get_encoder(&enc) != KDA_OK) return KDA_ERR_CUDA;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return KDA_ERR_CUDA;

    CUtensorMap tq, tk, tg;  // tg: the per-channel gate, dk channels x 64 tokens per box
    if (make_map(&tq, enc, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, dk, H, T, B, 64,
                 CU_TENSOR_MAP_SWIZZLE_128B) != KDA_OK ||
        make_map(&tk, enc, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, dk, H, T, B, 64,
                 CU_TENSOR_MAP_SWIZZLE_128B) != KDA_OK)
        return KDA_ERR_CUDA;
    if (scalar_gate) tg = tq;  // not read
    else if (make_map(&tg, enc, g, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, dk, H, T, B, dk,
                      CU_TENSOR_MAP_SWIZZLE_NONE) != KDA_OK)
        return KDA_ERR_CUDA;

    const SegPlan pl = plan_segments(B, T, H);
    const int nchunks = pl.nchunks, seg = pl.seg;
    const bool multi = pl.nbuf == 2;
    const size_t row = rec_row_bytes(B, H);
    const size_t state_bytes = (multi && hT == nullptr) ? (size_t)B * H * dk * dv * sizeof(float) : 0;
    const int sms = num_sms(dev);
    const int pmax = plan_parts(B, H, dk, dv, seg, sms);  // parts of a full segment (the most)

    std::lock_guard<std::mutex> lk(g_mu);
    Workspace *w = nullptr;
    const size_t list_bytes = steep_list_bytes(B, H, seg);
    if (int st = reserve_workspace(dev, kTicketBytes + list_bytes + pl.nbuf * seg * row, state_bytes, multi, &w,
                                   parts_bytes(B, H, dk, dv, pmax));
        st != KDA_OK)
        return st;
    if (cudaStreamWaitEvent(s, w->done, 0) != cudaSuccess) return KDA_ERR_CUDA;

    const unsigned long long polls = g_wait_polls.load();
    kda::DeviceStatus dst;
    dst.word = word;
    dst.wait_polls = polls ? polls : ~0ull;
    // State carried between segments: the caller's hT when given, else the workspace's.
    float *carry = hT != nullptr ? hT : w->state;
    // counters [buffer][item counter, steep count]; one steep list: the exact kernel of a
    // segment runs on the prep stream before the next segment's prep refills it
    int *counters = reinterpret_cast<int *>(w->base);
    int *steep_list = reinterpret_cast<int *>(w->base + kTicketBytes);
    uint8_t *rec0 = w->base + kTicketBytes + list_bytes;
    uint8_t *recs[2] = {rec0, rec0 + (size_t)seg * row};
    CUtensorMap rmaps[2][4];
    for (int i = 0; i < pl.nbuf; ++i)
        if (make_rec_maps(enc, recs[i], (long long)B * H * seg, dk, rmaps[i]) != KDA_OK) return KDA_ERR_CUDA;

    // Prep CTAs: two per SM, also beside a chain kernel.  The chain's CTAs are
    // placed first (the next prep waits for them), so the prep CTAs that do not
    // fit on the SMs the chain leaves free wait in the queue and start on the
    // chain's SMs as soon as it ends; they claim items from the same counter, so
    // they take over the segment's tail (long-context call 51.7 -> 49.8 ms
    // against two CTAs per free SM only; lower densities were slower still).
    const int prep_ctas = 2 * sms;
    cudaStream_t sp = s, sc = s;  // prep and chain streams
    if (multi) {
        sp = w->lo;
        sc = w->hi;
        if (cudaEventRecord(w->fork, s) != cudaSuccess || cudaStreamWaitEvent(sp, w->fork, 0) != cudaSuccess ||
            cudaStreamWaitEvent(sc, w->fork, 0) != cudaSuccess)
            return KDA_ERR_CUDA;
    }
    int i = 0;
    for (int n0 = 0; n0 < nchunks; n0 += seg, ++i) {
        const int cnt = nchunks - n0 < seg ? nchunks - n0 : seg;
        const int buf = multi ? (i & 1) : 0;
        // buffer reuse: the chain kernel two segments back has read it
        if (multi && i >= 2 && cudaStreamWaitEvent(sp, w->chain_done[buf], 0) != cudaSuccess) return KDA_ERR_CUDA;
        // and the previous segment's chain CTAs are all placed: a prep kernel placed
        // before them spreads its persistent CTAs over every SM and keeps the chain off
        // until it ends (the first segments; later ones are ordered by the wait above)
        if (multi && i >= 1 && cudaStreamWaitEvent(sp, w->chain_go, 0) != cudaSuccess) return KDA_ERR_CUDA;
        if (cudaMemsetAsync(counters + 2 * buf, 0, 2 * sizeof(int), sp) != cudaSuccess) return KDA_ERR_CUDA;
        kda::PrepParams pp;
        pp.g = g;
        pp.g_dk = g_dk;
        pp.beta = beta;
        pp.ws = recs[buf];
        pp.nrec = (long long)B * H * seg;
        pp.ticket = counters + 2 * buf;
        pp.steep_count = counters + 2 * buf + 1;
        pp.steep_items = steep_list;
        pp.force_exact = g_force_exact.load();
        pp.block_refs = g_block_refs.load();
        pp.gate_c = gate_c;
        pp.H = H;
        pp.gm = uniform_geom(B, T, n0, cnt);
        pp.st = dst;
        const int ctas = prep_ctas;
        cudaError_t e = timed_launch(dev, 0, sp, [&](unsigned long long *t) {
            pp.stamp = t;
            return kda::launch_prep(tq, tk, tg, pp, dk, ctas, sp, prologue);
        });
        if (e != cudaSuccess) return KDA_ERR_CUDA;
        kda::ExactParams xp = exact_params(q, k, g, g_dk, beta, pp, prologue);
        e = timed_launch(dev, 2, sp, [&](unsigned long long *t) {
            xp.stamp = t;
            return kda::launch_exact(xp, dk, sms, sp);
        });
        if (e != cudaSuccess) return KDA_ERR_CUDA;
        if (multi && (cudaEventRecord(w->prep_done[buf], sp) != cudaSuccess ||
                      cudaStreamWaitEvent(sc, w->prep_done[buf], 0) != cudaSuccess))
            return KDA_ERR_CUDA;

        kda::ChainParams cp;
        cp.v = static_cast<const uint16_t *>(v);
        cp.h0 = h0;  // read by the first segment; later ones start from carry
        cp.out = static_cast<uint16_t *>(out);
        cp.hT = hT;  // written by the last segment; earlier ones end in carry
        cp.carry = carry;
        cp.ws = recs[buf];
        cp.nrec = (long long)B * H * seg;
        cp.scale = scale;
        cp.H = H; cp.DV = dv;
        cp.gm = pp.gm;
        cp.st = dst;
        cp.inject_wait_polls = g_inject_polls.load();
        const int P = plan_parts(B, H, dk, dv, cnt, sms);
        cudaEvent_t go = multi ? w->chain_go : nullptr;
        if (P < 3) {
            plain_pass(cp, chain_slices(B, H, dv, sms));
            e = timed_launch(dev, 1, sc, [&](unsigned long long *t) {
                cp.stamp = t;
                return kda::launch_chain(rmaps[buf], cp, dk, sc, go);
            });
            if (e != cudaSuccess) return KDA_ERR_CUDA;
        } else {  // two-level pass: pass A, fix-up, pass B (64-column slices)
            const size_t st_part = (size_t)B * H * dk * dv;
            cp.nslices = dv / 64;
            cp.parts = P;
            cp.part_len = (cnt + P - 1) / P;
            cp.p_start = w->parts;
            cp.p_local = w->parts + (size_t)P * st_part;
            cp.p_trans = w->parts + 2 * (size_t)P * st_part;
            cp.pass_a = 1;
            cp.part0 = 0;
            cp.nparts = P - 1;
            cp.slots = (dv + dk) / 64;
            e = timed_launch(dev, 1, sc, [&](unsigned long long *t) {
                cp.stamp = t;
                return kda::launch_chain(rmaps[buf], cp, dk, sc, go);
            });
            if (e != cudaSuccess) return KDA_ERR_CUDA;
            e = timed_launch(dev, 3, sc, [&](unsigned long long *t) {
                return kda::launch_parts_fixup(cp.p_start, cp.p_local, cp.p_trans, B * H, dk, dv, P, sc, t);
            });
            if (e != cudaSuccess) return KDA_ERR_CUDA;
            cp.pass_a = 0;
            cp.part0 = 1;
            cp.nparts = P - 1;
            cp.slots = dv / 64;
            e = timed_launch(dev, 1, sc, [&](unsigned long long *t) {
                cp.stamp = t;
                return kda::launch_chain(rmaps[buf], cp, dk, sc);
            });
            if (e != cudaSuccess) return KDA_ERR_CUDA;
        }
        if (multi && cudaEventRecord(w->chain_done[buf], sc) != cudaSuccess) return KDA_ERR_CUDA;
    }
    // join: the last chain kernel follows every prep kernel
    if (multi && cudaStreamWaitEvent(s, w->chain_done[(i - 1) & 1], 0) != cudaSuccess) return KDA_ERR_CUDA;
    if (cudaEventRecord(w->done, s) != cudaSuccess) return KDA_ERR_CUDA;
    return KDA_OK;
}

size_t kda_chunk_fwd_workspace_bytes(int B, int T, int H, int dk, int dv) {
    if (B < 1 || H < 1 || T < 0 || (dk != 64 && dk != 128) || (dv != 64 && dv != 128)) return 0;
    if (T == 0) return 0;
    const SegPlan pl = plan_segments(B, T, H);
    const size_t state = pl.nbuf == 2 ? (size_t)B * H * dk * dv * sizeof(float) : 0;
    int dev = 0;
    const int sms = cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < kMaxDevices ? num_sms(dev) : 148;
    return kTicketBytes + steep_list_bytes(B, H, pl.seg) + (size_t)pl.nbuf * pl.seg * rec_row_bytes(B, H) + state +
           parts_bytes(B, H, dk, dv, plan_parts(B, H, dk, dv, pl.seg, sms));
}

void kda_debug_kernel_timing(int enable) { g_timing.store(enable != 0); }

// Every launch timed since the last read, in launch order: (kind, start, end) in
// globaltimer nanoseconds, end < start when the kernel left no stamp.  Forgets them.
struct StampRec {
    int kind;
    unsigned long long start, end;
};
static int collect_stamps(std::vector<StampRec> *out) {
    int st = KDA_OK, cur = 0;
    if (cudaGetDevice(&cur) != cudaSuccess) return KDA_ERR_CUDA;
    std::vector<unsigned long long> host;
    for (int dev = 0; dev < kMaxDevices; ++dev) {
        const int n = g_stamp_next[dev];
        if (n == 0) continue;
        host.assign(2 * (size_t)n, 0ull);
        if (cudaSetDevice(dev) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess ||
            cudaMemcpy(host.data(), g_stamp_ptr[dev], host.size() * sizeof(unsigned long long),
                       cudaMemcpyDeviceToHost) != cudaSuccess)
            st = KDA_ERR_CUDA;
        for (const TimedLaunch &t : g_timed) {
            if (t.dev != dev) continue;
            const unsigned long long a = host[2 * t.slot], e = ~host[2 * t.slot + 1];
            const bool ok = st == KDA_OK && a != ~0ull && e >= a;
            out->push_back({t.kind, ok ? a : 1ull, ok ? e : 0ull});
        }
        g_stamp_next[dev] = 0;
    }
    g_timed.clear();
    if (cudaSetDevice(cur) != cudaSuccess) st = KDA_ERR_CUDA;
    return st;
}

int kda_debug_kernel_times(double *ms, long long *launches, int nkinds) {
    if (ms == nullptr || launches == nullptr || nkinds < 0) return KDA_ERR_INVALID_ARG;
    for (int i = 0; i < nkinds; ++i) { ms[i] = 0.0; launches[i] = 0; }
    std::lock_guard<std::mutex> lk(g_mu);
    std::vector<StampRec> recs;
    const int st = collect_stamps(&recs);
    for (const StampRec &r : recs) {
        if (r.kind < 0 || r.kind >= nkinds) continue;
        if (r.end >= r.start) ms[r.kind] += (double)(r.end - r.start) * 1e-6;
        launches[r.kind] += 1;
    }
    return st;
}

int kda_debug_kernel_launches(int *kind, long long *start_ns, long long *end_ns, int cap, int *count) {
    if (kind == nullptr || start_ns == nullptr || end_ns == nullptr || count == nullptr || cap < 0)
        return KDA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(g_mu);
    std::vector<StampRec> recs;
    const int st = collect_stamps(&recs);
    const int n = (int)recs.size() < cap ? (int)recs.size() : cap;
    for (int i = 0; i < n; ++i) {
        kind[i] = recs[i].kind;
        start_ns[i] = (long long)recs[i].start;
        end_ns[i] = (long long)recs[i].end;
    }
    *count = n;
    return st;
}

extern "C" int kda_release_host_staging(int dev);  // host_fwd.cu

int kda_release_workspace(void) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KDA_ERR_CUDA;
    const int hs = kda_release_host_staging(dev);
    std::lock_guard<std::mutex> lk(g_mu);
    Workspace &w = g_ws[dev];
    int st = KDA_OK;
    if (w.base != nullptr && cudaFree(w.base) != cudaSuccess) st = KDA_ERR_CUDA;
    if (w.state != nullptr && cudaFree(w.state) != cudaSuccess) st = KDA_ERR_CUDA;
    if (w.parts != nullptr && cudaFree(w.parts) != cudaSuccess) st = KDA_ERR_CUDA;
    if (w.ckpt != nullptr && cudaFree(w.ckpt) != cudaSuccess) st = KDA_ERR_CUDA;
    w.ckpt = nullptr; w.ckpt_bytes = 0;
    w.base = nullptr; w.base_bytes = 0;
    w.state = nullptr; w.state_bytes = 0;
    w.parts = nullptr; w.parts_bytes = 0;
    return st != KDA_OK ? st : hs;
}

// The decode step for either gate form: g [B, H, dk] or, scalar_gate, g [B, H].
static int decode_impl(const void *q, const void *k, const void *v, const float *g, const float *beta,
                       float scale, float *state, void *out, int B, int H, int dk, int dv, void *stream,
                       bool scalar_gate, bool prologue = false, float gate_c = 0.f) {
    if (!q || !k || !v || !g || !beta || !state || !out) return KDA_ERR_INVALID_ARG;
    if (B < 1 || H < 1) return KDA_ERR_INVALID_ARG;
    if ((dk != 64 && dk != 128) || (dv != 64 && dv != 128)) return KDA_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !(scalar_gate ? aligned4(g) : aligned16(g)) ||
        !aligned4(beta) || !aligned16(state) || !aligned16(out))
        return KDA_ERR_ALIGNMENT;
    if ((long long)B * H > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
    cudaError_t e = kda::launch_decode(q, k, v, g, beta, scale, state, out, B * H, dk, dv, scalar_gate ? 1 : dk,
                                       prologue ? 1 : 0, gate_c, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

int kda_chunk_fwd(const void *q, const void *k, const void *v, const float *g, const float *beta,
                  float scale, const float *h0, void *out, float *hT, int B, int T, int H, int dk,
                  int dv, void *stream) {
    return chunk_fwd_impl(q, k, v, g, beta, scale, h0, out, hT, B, T, H, dk, dv, stream, false);
}

int kda_gdn_chunk_fwd(const void *q, const void *k, const void *v, const float *g, const float *beta,
                      float scale, const float *h0, void *out, float *hT, int B, int T, int H, int dk,
                      int dv, void *stream) {
    return chunk_fwd_impl(q, k, v, g, beta, scale, h0, out, hT, B, T, H, dk, dv, stream, true);
}

// Packed batch: N sequences along the token axis, cu_seqlens on the device.
// One record buffer; the global chunks run in windows of W chunks (every head),
// prep -> exact -> chain per window on the caller's stream; a sequence whose
// chunks span windows carries its state between them (in hT when given).
int kda_chunk_fwd_varlen(const void *q, const void *k, const void *v, const float *g, const float *beta,
                         float scale, const int *cu_seqlens, int N, const float *h0, void *out, float *hT,
                         int T_total, int H, int dk, int dv, void *stream) {
    if (N < 1 || H < 1 || T_total < 0 || cu_seqlens == nullptr) return KDA_ERR_INVALID_ARG;
    if (T_total > 0 && (!q || !k || !v || !g || !beta || !out)) return KDA_ERR_INVALID_ARG;
    if ((dk != 64 && dk != 128) || (dv != 64 && dv != 128)) return KDA_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(g) || !aligned4(beta) || !aligned16(out) ||
        !aligned16(h0) || !aligned16(hT) || !aligned4(cu_seqlens))
        return KDA_ERR_ALIGNMENT;
    if ((long long)N * H * 4 > 0x7fffffffLL || (long long)T_total + 64LL * (N + 1) > 0x7fffffffLL)
        return KDA_ERR_UNSUPPORTED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (T_total == 0) {  // every sequence is empty: hT = h0 (or zero)
        if (hT == nullptr) return KDA_OK;
        const size_t bytes = (size_t)N * H * dk * dv * sizeof(float);
        cudaError_t e = h0 ? (h0 == hT ? cudaSuccess : cudaMemcpyAsync(hT, h0, bytes, cudaMemcpyDeviceToDevice, s))
                           : cudaMemsetAsync(hT, 0, bytes, s);
        return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
    }
    uint32_t *word = nullptr;
    if (current_status_word(&word) != KDA_OK) return KDA_ERR_CUDA;
    PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
    if (get_encoder(&enc) != KDA_OK) return KDA_ERR_CUDA;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return KDA_ERR_CUDA;
    CUtensorMap tq, tk, tg;  // [1][T_total][H][dk]
    if (make_map(&tq, enc, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, dk, H, T_total, 1, 64,
                 CU_TENSOR_MAP_SWIZZLE_128B) != KDA_OK ||
        make_map(&tk, enc, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, dk, H, T_total, 1, 64,
                 CU_TENSOR_MAP_SWIZZLE_128B) != KDA_OK ||
        make_map(&tg, enc, g, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, dk, H, T_total, 1, dk,
                 CU_TENSOR_MAP_SWIZZLE_NONE) != KDA_OK)
        return KDA_ERR_CUDA;

    const VarlenPlan pl = plan_varlen(N, T_total, H);
    const int W = pl.W;
    const size_t row = rec_row_bytes(1, H);  // one chunk of every head
    const size_t state_bytes = (pl.nwin > 1 && hT == nullptr) ? (size_t)N * H * dk * dv * sizeof(float) : 0;
    const int sms = num_sms(dev);

    std::lock_guard<std::mutex> lk(g_mu);
    Workspace *w = nullptr;
    if (int st = reserve_workspace(dev, varlen_base_bytes(N, H, pl), state_bytes, false, &w); st != KDA_OK)
        return st;
    if (cudaStreamWaitEvent(s, w->done, 0) != cudaSuccess) return KDA_ERR_CUDA;
    const unsigned long long polls = g_wait_polls.load();
    kda::DeviceStatus dst;
    dst.word = word;
    dst.wait_polls = polls ? polls : ~0ull;
    // [counters][steep list][cu_s][cc][chunk_seq][records]
    int *counters = reinterpret_cast<int *>(w->base);
    int *steep_list = reinterpret_cast<int *>(w->base + kTicketBytes);
    int *cu_s = reinterpret_cast<int *>(w->base + kTicketBytes + steep_list_bytes(1, H, W));
    int *cc = cu_s + (N + 1);
    int *chunk_seq = cc + (N + 1);
    uint8_t *recs = w->base + kTicketBytes + steep_list_bytes(1, H, W) + varlen_meta_bytes(N, pl.cmax);
    CUtensorMap rmaps[4];
    if (make_rec_maps(enc, recs, (long long)H * W, dk, rmaps) != KDA_OK) return KDA_ERR_CUDA;
    if (kda::launch_varlen_setup(cu_seqlens, N, T_total, pl.cmax, cu_s, cc, chunk_seq, dst, s) != cudaSuccess)
        return KDA_ERR_CUDA;
    float *carry = hT != nullptr ? hT : w->state;

    for (int win = 0; win < pl.nwin; ++win) {
        kda::SeqGeom gm = {};
        gm.cu = cu_s;
        gm.cc = cc;
        gm.chunk_seq = chunk_seq;
        gm.nseqs = N;
        gm.T = T_total;
        gm.c0 = win * W;
        gm.W = W;
        if (cudaMemsetAsync(counters, 0, 2 * sizeof(int), s) != cudaSuccess) return KDA_ERR_CUDA;
        kda::PrepParams pp;
        pp.g = g;
        pp.g_dk = dk;
        pp.beta = beta;
        pp.ws = recs;
        pp.nrec = (long long)H * W;
        pp.ticket = counters;
        pp.steep_count = counters + 1;
        pp.steep_items = steep_list;
        pp.force_exact = g_force_exact.load();
        pp.block_refs = g_block_refs.load();
        pp.gate_c = 0.f;
        pp.H = H;
        pp.gm = gm;
        pp.st = dst;
        cudaError_t e = timed_launch(dev, 0, s, [&](unsigned long long *t) {
            pp.stamp = t;
            return kda::launch_prep(tq, tk, tg, pp, dk, 2 * sms, s, false);
        });
        if (e != cudaSuccess) return KDA_ERR_CUDA;
        kda::ExactParams xp = exact_params(q, k, g, dk, beta, pp);
        e = timed_launch(dev, 2, s, [&](unsigned long long *t) {
            xp.stamp = t;
            return kda::launch_exact(xp, dk, sms, s);
        });
        if (e != cudaSuccess) return KDA_ERR_CUDA;
        kda::ChainParams cp;
        cp.v = static_cast<const uint16_t *>(v);
        cp.h0 = h0;
        cp.out = static_cast<uint16_t *>(out);
        cp.hT = hT;
        cp.carry = carry;
        cp.ws = recs;
        cp.nrec = (long long)H * W;
        cp.scale = scale;
        cp.H = H; cp.DV = dv;
        cp.gm = gm;
        plain_pass(cp, chain_slices(N, H, dv, sms));
        cp.st = dst;
        cp.inject_wait_polls = g_inject_polls.load();
        e = timed_launch(dev, 1, s, [&](unsigned long long *t) {
            cp.stamp = t;
            return kda::launch_chain(rmaps, cp, dk, s);
        });
        if (e != cudaSuccess) return KDA_ERR_CUDA;
    }
    if (cudaEventRecord(w->done, s) != cudaSuccess) return KDA_ERR_CUDA;
    return KDA_OK;
}

size_t kda_chunk_fwd_varlen_workspace_bytes(int N, int T_total, int H, int dk, int dv) {
    if (N < 1 || H < 1 || T_total < 0 || (dk != 64 && dk != 128) || (dv != 64 && dv != 128)) return 0;
    if (T_total == 0) return 0;
    const VarlenPlan pl = plan_varlen(N, T_total, H);
    const size_t state = pl.nwin > 1 ? (size_t)N * H * dk * dv * sizeof(float) : 0;
    return varlen_base_bytes(N, H, pl) + state;
}

// Backward of the prefill (recurrent form, bwd.cu): checkpoints of the state
// every few tokens in the workspace, then the reverse walk.
int kda_chunk_bwd(const void *q, const void *k, const void *v, const float *g, const float *beta, float scale,
                  const float *h0, const void *dout, const float *dhT, void *dq, void *dk_, void *dv_, float *dg,
                  float *dbeta, float *dh0, int B, int T, int H, int dk, int dv, void *stream) {
    if (B < 1 || H < 1 || T < 0) return KDA_ERR_INVALID_ARG;
    if (T > 0 && (!q || !k || !v || !g || !beta || !dq || !dk_ || !dv_ || !dg || !dbeta)) return KDA_ERR_INVALID_ARG;
    if ((dk != 64 && dk != 128) || (dv != 64 && dv != 128)) return KDA_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(g) || !aligned4(beta) || !aligned16(h0) ||
        !aligned16(dout) || !aligned16(dhT) || !aligned16(dq) || !aligned16(dk_) || !aligned16(dv_) ||
        !aligned16(dg) || !aligned4(dbeta) || !aligned16(dh0))
        return KDA_ERR_ALIGNMENT;
    if ((long long)B * H > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (T == 0) {  // hT = h0, so dh0 = dhT
        if (dh0 == nullptr) return KDA_OK;
        const size_t bytes = (size_t)B * H * dk * dv * sizeof(float);
        cudaError_t e = dhT ? (dhT == dh0 ? cudaSuccess : cudaMemcpyAsync(dh0, dhT, bytes, cudaMemcpyDeviceToDevice, s))
                            : cudaMemsetAsync(dh0, 0, bytes, s);
        return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
    }
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KDA_ERR_CUDA;
    uint32_t *word = nullptr;  // before g_mu: current_status_word takes it too
    if (current_status_word(&word) != KDA_OK) return KDA_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    Workspace *w = nullptr;
    if (int st = reserve_workspace(dev, 0, 0, false, &w); st != KDA_OK) return st;
    const size_t need = kda::bwd_ckpt_bytes(B, T, H, dk, dv);
    if (w->ckpt_bytes < need) {
        if (w->ckpt != nullptr && cudaFree(w->ckpt) != cudaSuccess) return KDA_ERR_CUDA;
        w->ckpt = nullptr;
        w->ckpt_bytes = 0;
        if (cudaMalloc(&w->ckpt, need) != cudaSuccess) return KDA_ERR_CUDA;
        w->ckpt_bytes = need;
    }
    if (cudaStreamWaitEvent(s, w->done, 0) != cudaSuccess) return KDA_ERR_CUDA;
    kda::BwdParams bp;
    bp.q = static_cast<const uint16_t *>(q);
    bp.k = static_cast<const uint16_t *>(k);
    bp.v = static_cast<const uint16_t *>(v);
    bp.g = g;
    bp.beta = beta;
    bp.h0 = h0;
    bp.dout = static_cast<const uint16_t *>(dout);
    bp.dhT = dhT;
    bp.dq = static_cast<uint16_t *>(dq);
    bp.dk = static_cast<uint16_t *>(dk_);
    bp.dv = static_cast<uint16_t *>(dv_);
    bp.dg = dg;
    bp.dbeta = dbeta;
    bp.dh0 = dh0;
    bp.ckpt = w->ckpt;
    bp.ckpt_elems = (long long)(need / sizeof(float));
    bp.scale = scale;
    bp.B = B; bp.T = T; bp.H = H;
    bp.st.word = word;
    bp.st.wait_polls = ~0ull;  // the backward has no bounded waits
    if (timed_launch(dev, 4, s, [&](unsigned long long *t) {
            bp.stamp = t;
            return kda::launch_bwd(bp, dk, dv, s);
        }) != cudaSuccess)
        return KDA_ERR_CUDA;
    if (cudaEventRecord(w->done, s) != cudaSuccess) return KDA_ERR_CUDA;
    return KDA_OK;
}

size_t kda_chunk_bwd_workspace_bytes(int B, int T, int H, int dk, int dv) {
    if (B < 1 || H < 1 || T <= 0 || (dk != 64 && dk != 128) || (dv != 64 && dv != 128)) return 0;
    return kda::bwd_ckpt_bytes(B, T, H, dk, dv);
}

int kda_decode_step(const void *q, const void *k, const void *v, const float *g, const float *beta,
                    float scale, float *state, void *out, int B, int H, int dk, int dv, void *stream) {
    return decode_impl(q, k, v, g, beta, scale, state, out, B, H, dk, dv, stream, false);
}

int kda_gdn_decode_step(const void *q, const void *k, const void *v, const float *g, const float *beta,
                        float scale, float *state, void *out, int B, int H, int dk, int dv, void *stream) {
    return decode_impl(q, k, v, g, beta, scale, state, out, B, H, dk, dv, stream, true);
}

int kda_chunk_fwd_raw(const void *q, const void *k, const void *v, const float *g_raw, const float *beta_raw,
                      float gate_c, float scale, const float *h0, void *out, float *hT, int B, int T, int H,
                      int dk, int dv, void *stream) {
    if (!(gate_c >= 0.f) || gate_c > 3.0e38f) return KDA_ERR_INVALID_ARG;  // also rejects NaN
    return chunk_fwd_impl(q, k, v, g_raw, beta_raw, scale, h0, out, hT, B, T, H, dk, dv, stream, false, true,
                          gate_c);
}

int kda_decode_step_raw(const void *q, const void *k, const void *v, const float *g_raw, const float *beta_raw,
                        float gate_c, float scale, float *state, void *out, int B, int H, int dk, int dv,
                        void *stream) {
    if (!(gate_c >= 0.f) || gate_c > 3.0e38f) return KDA_ERR_INVALID_ARG;
    return decode_impl(q, k, v, g_raw, beta_raw, scale, state, out, B, H, dk, dv, stream, false, true, gate_c);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Fixed-scratch prefill (kda_chunk_fwd_noalloc).
//
// Some callers cannot allocate device memory when they call the prefill: a
// process whose device memory is handed out up front to another allocator (a
// serving stack that reserves nearly all of HBM for its own caching allocator
// leaves cudaMalloc nothing to give), or code that must not pay the
// device-wide synchronisation that freeing a grown workspace costs.  This
// variant runs the same two kernels over chunk records kept in a fixed array
// that is part of the module image, in as many segments as the array holds.
// Of the scratch, only the prep kernel's item counter must start at zero, and
// each call clears it before each launch; the prep kernel writes every record
// byte the chain kernel's results depend on before the chain kernel reads it
// (rows it leaves unwritten feed accumulator lanes that are discarded), and
// the carried state is written before it is read.
namespace {

constexpr size_t kScratchBytes = size_t(64) << 20;  // 64 MiB per device
static __device__ __align__(256) uint8_t g_kda_scratch[kScratchBytes];

uint8_t *g_scratch_ptr[kMaxDevices] = {};

// Once per device, with that device current: the device address of the array.
int scratch_base(int dev, uint8_t **out) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_scratch_ptr[dev] == nullptr) {
        uint8_t *p = nullptr;
        if (cudaGetSymbolAddress((void **)&p, g_kda_scratch) != cudaSuccess || p == nullptr) return KDA_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return KDA_OK;
}

}  // namespace

extern "C" {

int kda_chunk_fwd_noalloc(const void *q, const void *k, const void *v, const float *g, const float *beta,
                          float scale, const float *h0, void *out, float *hT, int B, int T, int H, int dk,
                          int dv, void *stream) {
    if (B < 1 || H < 1 || T < 0) return KDA_ERR_INVALID_ARG;
    if (T > 0 && (!q || !k || !v || !g || !beta || !out)) return KDA_ERR_INVALID_ARG;
    if ((dk != 64 && dk != 128) || (dv != 64 && dv != 128)) return KDA_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(g) || !aligned4(beta) ||
        !aligned16(out) || !aligned16(h0) || !aligned16(hT))
        return KDA_ERR_ALIGNMENT;
    if ((long long)B * H * 4 > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    if (T == 0) {  // nothing to scan: hT = h0 (or zero)
        if (hT == nullptr) return KDA_OK;
        const size_t bytes = (size_t)B * H * dk * dv * sizeof(float);
        cudaError_t e = h0 ? (h0 == hT ? cudaSuccess : cudaMemcpyAsync(hT, h0, bytes, cudaMemcpyDeviceToDevice, s))
                           : cudaMemsetAsync(hT, 0, bytes, s);
        return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
    }

    // Scratch layout: [counters][steep-item list][carried state, when hT is NULL][records of one
    // segment]; a segment of n chunks needs n rows of records and n * B * H list entries.
    const int nchunks = (T + kda::CH - 1) / kda::CH;
    const size_t row = rec_row_bytes(B, H);
    const size_t state_bytes = hT == nullptr ? round256((size_t)B * H * dk * dv * sizeof(float)) : 0;
    const size_t fixed = kTicketBytes + 256 + state_bytes;  // 256: the list's rounding
    const size_t per_chunk = row + (size_t)B * H * sizeof(int);
    if (fixed + per_chunk > kScratchBytes) return KDA_ERR_SCRATCH_LIMIT;
    const size_t fit = (kScratchBytes - fixed) / per_chunk;
    const int seg = fit < (size_t)nchunks ? (int)fit : nchunks;
    const size_t list_bytes = steep_list_bytes(B, H, seg);

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KDA_ERR_CUDA;
    uint8_t *scratch = nullptr;
    if (scratch_base(dev, &scratch) != KDA_OK) return KDA_ERR_CUDA;
    uint32_t *word = nullptr;
    if (current_status_word(&word) != KDA_OK) return KDA_ERR_CUDA;
    PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
    if (get_encoder(&enc) != KDA_OK) return KDA_ERR_CUDA;

    CUtensorMap tq, tk, tg;
    if (make_map(&tq, enc, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, dk, H, T, B, 64,
                 CU_TENSOR_MAP_SWIZZLE_128B) != KDA_OK ||
        make_map(&tk, enc, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, dk, H, T, B, 64,
                 CU_TENSOR_MAP_SWIZZLE_128B) != KDA_OK ||
        make_map(&tg, enc, g, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, dk, H, T, B, dk,
                 CU_TENSOR_MAP_SWIZZLE_NONE) != KDA_OK)
        return KDA_ERR_CUDA;

    const unsigned long long polls = g_wait_polls.load();
    kda::DeviceStatus dst;
    dst.word = word;
    dst.wait_polls = polls ? polls : ~0ull;
    // [item counter, steep count][steep list][carried state, when hT is NULL][records]
    int *ticket = reinterpret_cast<int *>(scratch);
    int *steep_list = reinterpret_cast<int *>(scratch + kTicketBytes);
    float *carry = hT != nullptr ? hT : reinterpret_cast<float *>(scratch + kTicketBytes + list_bytes);
    uint8_t *recs = scratch + kTicketBytes + list_bytes + state_bytes;
    const int sms = num_sms(dev);
    CUtensorMap rmaps[4];
    if (make_rec_maps(enc, recs, (long long)B * H * seg, dk, rmaps) != KDA_OK) return KDA_ERR_CUDA;

    for (int n0 = 0; n0 < nchunks; n0 += seg) {
        const int cnt = nchunks - n0 < seg ? nchunks - n0 : seg;
        kda::PrepParams pp;
        pp.g = g;
        pp.g_dk = dk;
        pp.beta = beta;
        pp.ws = recs;
        pp.nrec = (long long)B * H * seg;
        pp.ticket = ticket;
        pp.steep_count = ticket + 1;
        pp.steep_items = steep_list;
        pp.force_exact = g_force_exact.load();
        pp.block_refs = g_block_refs.load();
        pp.gate_c = 0.f;
        pp.H = H;
        pp.gm = uniform_geom(B, T, n0, cnt);
        pp.st = dst;
        pp.stamp = nullptr;
        if (cudaMemsetAsync(ticket, 0, 2 * sizeof(int), s) != cudaSuccess ||  // the counters start at zero
            kda::launch_prep(tq, tk, tg, pp, dk, 2 * sms, s, false) != cudaSuccess ||
            kda::launch_exact(exact_params(q, k, g, dk, beta, pp), dk, sms, s) != cudaSuccess)
            return KDA_ERR_CUDA;

        kda::ChainParams cp;
        cp.v = static_cast<const uint16_t *>(v);
        cp.h0 = h0;
        cp.out = static_cast<uint16_t *>(out);
        cp.hT = hT;
        cp.carry = carry;
        cp.ws = recs;
        cp.nrec = (long long)B * H * seg;
        cp.scale = scale;
        cp.H = H; cp.DV = dv;
        cp.gm = pp.gm;
        plain_pass(cp, chain_slices(B, H, dv, sms));
        cp.st = dst;
        cp.inject_wait_polls = g_inject_polls.load();
        if (kda::launch_chain(rmaps, cp, dk, s) != cudaSuccess) return KDA_ERR_CUDA;
    }
    return KDA_OK;
}

}  // extern "C"
