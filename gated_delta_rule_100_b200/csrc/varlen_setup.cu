// varlen_setup.cu -- the chunk geometry of a packed batch of sequences, built on
// the device from the caller's cu_seqlens (sm_100a).
//
// A packed batch holds N sequences back to back along the token axis;
// cu_seqlens[n] .. cu_seqlens[n+1] - 1 are the tokens of sequence n.  Chunks of
// 64 tokens never cross a sequence boundary (each sequence starts a new chunk
// and its last chunk may be partial), so sequence n owns
// ceil(len_n / 64) chunks, global chunks cc[n] .. cc[n+1] - 1.  One CTA:
//   cu_s   the offsets made safe to index with: cu_s[0] = 0, each one clamped
//          to [cu_s[n-1], T_total] (a running maximum), so no kernel reads
//          outside the token range whatever the caller passed; any change from
//          the caller's values (cu[0] != 0, a decrease, cu[N] != T_total) sets
//          DEV_BAD_ARG in the status word (kda_stream_status then reports it);
//   cc     chunk offsets, an exclusive scan of the chunk counts;
//   chunk_seq[c] the sequence that owns global chunk c (by binary search over
//          cc), for c < cmax; entries past cc[N] are -1.
#include <cuda_runtime.h>
#include <stdint.h>

#include "chunk_common.cuh"
#include "kda_device.cuh"

namespace kda {

constexpr int SETUP_THREADS = 1024;

// Block-wide inclusive scan of one value per thread with `op`.
template <class Op>
__device__ __forceinline__ int block_scan(int x, int *s_warp, Op op) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, d);
        if (lane >= d) x = op(x, y);
    }
    if (lane == 31) s_warp[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = s_warp[lane];
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, d);
            if (lane >= d) w = op(w, y);
        }
        s_warp[lane] = w;
    }
    __syncthreads();
    if (warp > 0) x = op(x, s_warp[warp - 1]);
    __syncthreads();  // s_warp is reused by the next scan
    return x;
}

__global__ void __launch_bounds__(SETUP_THREADS, 1)
varlen_setup_kernel(const int *cu, int N, int T_total, int cmax, int *cu_s, int *cc, int *chunk_seq,
                    DeviceStatus st) {
    __shared__ int s_warp[32];
    __shared__ int s_off[SETUP_THREADS + 1];  // this tile's offsets, after the previous tile's last
    __shared__ int s_carry[2];  // running maximum of the offsets, running sum of the chunks
    const int tid = threadIdx.x;
    auto imax = [](int a, int b) { return a > b ? a : b; };
    auto iadd = [](int a, int b) { return a + b; };
    if (tid == 0) {
        s_carry[0] = 0;
        s_carry[1] = 0;
        cu_s[0] = 0;
        cc[0] = 0;
        if (cu[0] != 0) report(st, DEV_BAD_ARG);
    }
    __syncthreads();
    bool bad = false;
    for (int base = 1; base <= N; base += SETUP_THREADS) {
        const int n = base + tid;  // offset index 1..N
        const int raw = n <= N ? cu[n] : 0;
        const int x0 = raw < 0 ? 0 : (raw > T_total ? T_total : raw);
        const int prev_max = s_carry[0];
        const int x = imax(block_scan(n <= N ? x0 : 0, s_warp, imax), prev_max);  // non-decreasing
        if (n <= N) {
            cu_s[n] = x;
            bad |= x != raw || (n == N && raw != T_total);
        }
        if (tid == 0) s_off[0] = prev_max;
        s_off[tid + 1] = x;
        __syncthreads();
        const int len = n <= N ? s_off[tid + 1] - s_off[tid] : 0;  // sequence n - 1
        const int prev_sum = s_carry[1];
        const int csum = block_scan((len + CH - 1) / CH, s_warp, iadd) + prev_sum;
        if (n <= N) cc[n] = csum;
        __syncthreads();  // every thread has read s_off and s_carry
        if (tid == SETUP_THREADS - 1) {
            s_carry[0] = x;
            s_carry[1] = csum;
        }
        __syncthreads();
    }
    if (__syncthreads_or(bad) && tid == 0) report(st, DEV_BAD_ARG);
    // chunk -> sequence; the last sequence whose first chunk is <= c (skips empty sequences)
    const int total = cc[N];
    for (int c = tid; c < cmax; c += SETUP_THREADS) {
        int r = -1;
        if (c < total) {
            int lo = 0, hi = N - 1;  // cc[lo] <= c < cc[hi + 1]
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (cc[mid] <= c) lo = mid;
                else hi = mid - 1;
            }
            r = lo;
        }
        chunk_seq[c] = r;
    }
}

cudaError_t launch_varlen_setup(const int *cu, int N, int T_total, int cmax, int *cu_s, int *cc, int *chunk_seq,
                                const DeviceStatus &st, cudaStream_t stream) {
    varlen_setup_kernel<<<1, SETUP_THREADS, 0, stream>>>(cu, N, T_total, cmax, cu_s, cc, chunk_seq, st);
    return cudaGetLastError();
}

}  // namespace kda
