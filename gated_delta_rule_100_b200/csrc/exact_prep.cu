// exact_prep.cu -- the intra-chunk pieces of "steep" items, computed without
// split decay factors (sm_100a, CUDA cores, fp32).
//
// The prep kernel (prep_fwd.cu) forms A and P with one tensor-core product by
// splitting every decay factor e^{Gamma_i - Gamma_j} around a mid-block
// reference.  When a key channel loses more than 80 of log-decay inside half
// of a 16-token block, a split factor would leave the fp32 range; prep then
// clamps it (so nothing overflows) and lists the item.  This kernel rewrites
// the listed items' P, T' and W in their records, from
//   A_ij = beta_i sum_c k_ic k_jc e^{Gamma_ic - Gamma_jc}   (i > j)
//   P_ij =        sum_c q_ic k_jc e^{Gamma_ic - Gamma_jc}   (i >= j)
//   T    = (I + A)^{-1}  by forward substitution,   T' = T Diag(beta)
//   W    = T' (K * e^Gamma)
// with each pair's factor formed on its own (an exponent <= 0, so <= 1).  The
// other record parts (Q e^Gamma, K-hat, e^{Gamma_C}) use factors <= 1 in prep
// and are already exact.  These are the intra-chunk terms of the chunkwise
// form (section 4 of "Kimi Linear's Hybrid Linear Attention Architecture: A
// Technical Breakdown"), whose "renormalisation when necessary" this is.
//
// A fixed grid of CTAs walks the list (its length is read on the device; an
// empty list costs one launch that exits at once).
#include <cuda_bf16.h>
#include <stdint.h>

#include "chunk_common.cuh"
#include "chunk_params.cuh"
#include "kda_device.cuh"

namespace kda {

constexpr int EXACT_THREADS = 512;

template <int DK>
struct ExactLayout {
    static constexpr int LD = DK + 1;   // fp32 row stride of the [64][DK] tiles
    static constexpr int LDA = CH + 1;  // fp32 row stride of the [64][64] tiles
    static constexpr int OFF_G = 0;                      // Gamma, running sum of g per channel
    static constexpr int OFF_K = OFF_G + CH * LD * 4;    // k, then k * e^Gamma
    static constexpr int OFF_Q = OFF_K + CH * LD * 4;    // q
    static constexpr int OFF_A = OFF_Q + CH * LD * 4;    // A, then T
    static constexpr int OFF_TP = OFF_A + CH * LDA * 4;  // T'
    static constexpr int OFF_BETA = OFF_TP + CH * LDA * 4;
    static constexpr int SMEM_BYTES = OFF_BETA + CH * 4;
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

template <int DK, bool SG>
__global__ void __launch_bounds__(EXACT_THREADS, 1) exact_prep_kernel(const ExactParams prm) {
    using L = ExactLayout<DK>;
    extern __shared__ __align__(16) uint8_t sm[];
    float *sG = reinterpret_cast<float *>(sm + L::OFF_G);
    float *sK = reinterpret_cast<float *>(sm + L::OFF_K);
    float *sQ = reinterpret_cast<float *>(sm + L::OFF_Q);
    float *sA = reinterpret_cast<float *>(sm + L::OFF_A);
    float *sTp = reinterpret_cast<float *>(sm + L::OFF_TP);
    float *sB = reinterpret_cast<float *>(sm + L::OFF_BETA);
    const int tid = threadIdx.x;
    const int H = prm.H;
    constexpr int gdk = SG ? 1 : DK;
    if (tid == 0) stamp_start(prm.stamp);
    const int count = *prm.steep_count;

    for (int idx = blockIdx.x; idx < count; idx += gridDim.x) {
        const ItemGeo gi = geom_packed(prm.gm) ? item_geo<true>(prm.gm, H, prm.steep_items[idx])
                                               : item_geo<false>(prm.gm, H, prm.steep_items[idx]);
        const int h = gi.h;
        uint8_t *rec = prm.ws + (size_t)gi.rec * REC_BYTES;
        // debug build: the record and rows of the item (a bad one is reported and skipped)
        if (!KDA_CHECK(prm.st, gi.rec >= 0 && gi.rec < prm.nrec && gi.row0 >= 0 &&
                                   gi.row0 + (gi.nvalid < CH ? gi.nvalid : CH) <= geom_rows(prm.gm)))
            continue;

        // ---- inputs (tokens past the sequence's end read as zero, with beta = 0) ----
        for (int e = tid; e < CH * DK; e += EXACT_THREADS) {
            const int t = e / DK, c = e % DK;
            const bool valid = t < gi.nvalid;
            const size_t row = (size_t)(gi.row0 + (valid ? t : 0)) * H + h;
            const float graw = valid ? prm.g[row * gdk + (SG ? 0 : c)] : 0.f;
            sG[t * L::LD + c] = (prm.prologue && valid) ? gate_logdecay(graw, prm.gate_c) : graw;
            sK[t * L::LD + c] = valid ? bf16_bits_to_f32(prm.k[row * DK + c]) : 0.f;
            sQ[t * L::LD + c] = valid ? bf16_bits_to_f32(prm.q[row * DK + c]) : 0.f;
        }
        if (tid < CH) {
            const float braw = tid < gi.nvalid ? prm.beta[(size_t)(gi.row0 + tid) * H + h] : 0.f;
            sB[tid] = (prm.prologue && tid < gi.nvalid) ? gate_sigmoid(braw) : braw;
        }
        __syncthreads();
        if (prm.prologue && tid < 2 * CH) {  // L2-normalise q (rows 0..63) and k (64..127), rounded to bf16
            float *rowp = (tid < CH ? sQ : sK) + (tid % CH) * L::LD;
            float ss = 0.f;
            for (int c = 0; c < DK; ++c) ss += rowp[c] * rowp[c];
            const float r = rsqrtf(fmaxf(ss, 1e-24f));
            for (int c = 0; c < DK; ++c) rowp[c] = bf16_bits_to_f32(to_bf16_bits(rowp[c] * r));
        }
        if (tid < DK) {  // Gamma: inclusive running sum over the chunk's tokens
            float run = 0.f;
            for (int t = 0; t < CH; ++t) {
                run += sG[t * L::LD + tid];
                sG[t * L::LD + tid] = run;
            }
        }
        __syncthreads();

        // ---- A and P: thread owns row i, columns j = jg + 8 r ----
        {
            const int i = tid >> 3, jg = tid & 7;
            float a[8], p[8];
#pragma unroll
            for (int r = 0; r < 8; ++r) { a[r] = 0.f; p[r] = 0.f; }
            for (int c = 0; c < DK; ++c) {
                const float gam = sG[i * L::LD + c], ki = sK[i * L::LD + c], qi = sQ[i * L::LD + c];
#pragma unroll
                for (int r = 0; r < 8; ++r) {
                    const int j = jg + 8 * r;
                    if (j <= i) {
                        const float kf = sK[j * L::LD + c] * __expf(gam - sG[j * L::LD + c]);
                        a[r] += ki * kf;
                        p[r] += qi * kf;
                    }
                }
            }
            const float bi = sB[i];
            uint16_t *prec = reinterpret_cast<uint16_t *>(rec + REC_P);  // [J][i][e] = P[i][16 J + e]
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                const int j = jg + 8 * r;
                sA[i * L::LDA + j] = j < i ? bi * a[r] : 0.f;
                prec[((j >> 4) * CH + i) * SUB + (j & 15)] = f16_bits(j <= i ? p[r] : 0.f);
            }
        }
        __syncthreads();

        // ---- T = (I + A)^{-1}: thread j substitutes column j; T' = T Diag(beta) ----
        if (tid < CH) {
            const int j = tid;
            float *tcol = sTp;  // T[i][j] kept in sTp during the substitution
            for (int i = 0; i < CH; ++i) {
                float x = 0.f;
                if (i == j) {
                    x = 1.f;
                } else if (i > j) {
                    float s0 = 0.f, s1 = 0.f;
                    int m = j;
                    for (; m + 1 < i; m += 2) {
                        s0 += sA[i * L::LDA + m] * tcol[m * L::LDA + j];
                        s1 += sA[i * L::LDA + m + 1] * tcol[(m + 1) * L::LDA + j];
                    }
                    if (m < i) s0 += sA[i * L::LDA + m] * tcol[m * L::LDA + j];
                    x = -(s0 + s1);
                }
                tcol[i * L::LDA + j] = x;
            }
            const float bj = sB[j];
            float *trec = reinterpret_cast<float *>(rec + REC_T);  // fp32 [64][64] row-major
            for (int i = 0; i < CH; ++i) {
                const float tp = tcol[i * L::LDA + j] * bj;
                tcol[i * L::LDA + j] = tp;
                trec[i * CH + j] = tp;
            }
        }
        __syncthreads();

        // ---- W = T' (K e^Gamma) -> record WQ blocks 0..3 (bf16 [4][DK][16]) ----
        for (int e = tid; e < CH * DK; e += EXACT_THREADS) {
            const int t = e / DK, c = e % DK;
            sK[t * L::LD + c] *= __expf(sG[t * L::LD + c]);
        }
        __syncthreads();
        {
            constexpr int RG = EXACT_THREADS / DK;  // row groups
            const int c = tid % DK, ig = tid / DK;
            uint16_t *wrec = reinterpret_cast<uint16_t *>(rec + REC_WQ);
            for (int i = ig; i < CH; i += RG) {
                float acc = 0.f;
                for (int j = 0; j <= i; ++j) acc += sTp[i * L::LDA + j] * sK[j * L::LD + c];
                wrec[((i >> 4) * DK + c) * SUB + (i & 15)] = to_bf16_bits(acc);
            }
        }
        __syncthreads();  // the tiles are reused by the next item
    }
    if (tid == 0) stamp_end(prm.stamp);
}

template <int DK, bool SG>
static cudaError_t launch_exact_t(const ExactParams &prm, int ctas, cudaStream_t stream) {
    using L = ExactLayout<DK>;
    cudaError_t e = cudaFuncSetAttribute(exact_prep_kernel<DK, SG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         L::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    exact_prep_kernel<DK, SG><<<ctas, EXACT_THREADS, L::SMEM_BYTES, stream>>>(prm);
    return cudaGetLastError();
}

// `ctas` CTAs walk the list; prm.g_dk selects the gate form (dk or 1).
cudaError_t launch_exact(const ExactParams &prm, int dk, int ctas, cudaStream_t stream) {
    const bool sg = prm.g_dk == 1;
    if (dk == 128) return sg ? launch_exact_t<128, true>(prm, ctas, stream) : launch_exact_t<128, false>(prm, ctas, stream);
    return sg ? launch_exact_t<64, true>(prm, ctas, stream) : launch_exact_t<64, false>(prm, ctas, stream);
}

}  // namespace kda
