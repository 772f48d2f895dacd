// parts_fixup.cu -- the sequential level of the two-level (segment-parallel)
// state pass (sm_100a, fp32 on CUDA cores).
//
// The chain of one (b, h) is cut into parts.  Each part p >= 1 was run from a
// zero start (its end state `local[p]`) and from the identity (its dk x dk
// transition `trans[p]`: the end state it would reach from start state S is
// trans[p] S + local[p], because the update is linear in the state).  Part 0
// ran from the true start and left start[1].  Here, in order,
//   start[p + 1] = trans[p] start[p] + local[p],   p = 1 .. parts - 2,
// after which every part can produce its outputs independently.  This is the
// "compute chunk-level products in parallel, then combine sequentially" scheme
// of the "Kimi Linear" explainer (math.kryvik.com), blocks "DPLR Chunked
// Parallel" and "The Woodbury Identity Trick", at the level of parts of chunks.
//
// One CTA per (b, h) and block of 32 state columns; per step it stages the
// transition (dk x dk) and the block of start[p] in shared memory.
#include <cuda_runtime.h>
#include <stdint.h>

#include "kda_device.cuh"

namespace kda {

constexpr int FIX_THREADS = 256;
constexpr int FIX_COLS = 32;

template <int DK>
__global__ void __launch_bounds__(FIX_THREADS, 1)
parts_fixup_kernel(float *start, const float *local, const float *trans, int BH, int DV, int parts,
                   unsigned long long *stamp) {
    constexpr int TPR = FIX_THREADS / DK;  // threads per state row
    constexpr int CPT = FIX_COLS / TPR;    // columns per thread
    extern __shared__ float fsm[];
    float *sM = fsm;                       // [DK][DK + 1]
    float *sS = fsm + DK * (DK + 1);       // [DK][FIX_COLS + 1]
    const int nblk = DV / FIX_COLS;
    const int bh = blockIdx.x / nblk, cb = blockIdx.x % nblk;
    const int tid = threadIdx.x;
    const int r = tid / TPR, c0 = (tid % TPR) * CPT;
    const size_t sst = (size_t)BH * DK * DV, mst = (size_t)BH * DK * DK;  // per-part strides
    if (tid == 0) stamp_start(stamp);
    for (int p = 1; p + 1 < parts; ++p) {
        const float *Sp = start + p * sst + (size_t)bh * DK * DV + cb * FIX_COLS;
        const float *Mp = trans + p * mst + (size_t)bh * DK * DK;
        for (int e = tid; e < DK * FIX_COLS; e += FIX_THREADS) {
            const int j = e / FIX_COLS, c = e % FIX_COLS;
            sS[j * (FIX_COLS + 1) + c] = Sp[(size_t)j * DV + c];
        }
        for (int e = tid; e < DK * DK; e += FIX_THREADS) sM[(e / DK) * (DK + 1) + e % DK] = Mp[e];
        __syncthreads();
        const float *Lp = local + p * sst + (size_t)bh * DK * DV + (size_t)r * DV + cb * FIX_COLS + c0;
        float acc[CPT];
#pragma unroll
        for (int c = 0; c < CPT; ++c) acc[c] = Lp[c];
        for (int j = 0; j < DK; ++j) {
            const float m = sM[r * (DK + 1) + j];
#pragma unroll
            for (int c = 0; c < CPT; ++c) acc[c] += m * sS[j * (FIX_COLS + 1) + c0 + c];
        }
        float *Sn = start + (p + 1) * sst + (size_t)bh * DK * DV + (size_t)r * DV + cb * FIX_COLS + c0;
#pragma unroll
        for (int c = 0; c < CPT; ++c) Sn[c] = acc[c];
        __syncthreads();  // the next step restages; its start block is this step's output
    }
    if (tid == 0) stamp_end(stamp);
}

// start/local: [parts][BH][dk][dv], trans: [parts][BH][dk][dk], dv a multiple of 32.
cudaError_t launch_parts_fixup(float *start, const float *local, const float *trans, int BH, int dk, int dv,
                               int parts, cudaStream_t stream, unsigned long long *stamp) {
    const int grid = BH * (dv / FIX_COLS);
    if (dk == 128) {
        const int smem = (128 * 129 + 128 * (FIX_COLS + 1)) * 4;
        cudaError_t e = cudaFuncSetAttribute(parts_fixup_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        parts_fixup_kernel<128><<<grid, FIX_THREADS, smem, stream>>>(start, local, trans, BH, dv, parts, stamp);
    } else {
        const int smem = (64 * 65 + 64 * (FIX_COLS + 1)) * 4;
        cudaError_t e = cudaFuncSetAttribute(parts_fixup_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        parts_fixup_kernel<64><<<grid, FIX_THREADS, smem, stream>>>(start, local, trans, BH, dv, parts, stamp);
    }
    return cudaGetLastError();
}

}  // namespace kda
