// bwd.cu -- the backward pass of the KDA prefill: gradients of a loss through
// kda_chunk_fwd's outputs (out and hT) with respect to q, k, v, g, beta and h0
// (sm_100a, fp32 on CUDA cores).
//
// Reverse-mode differentiation of the recurrence (per (b, h), state S, dk x dv)
//   S' = Diag(alpha) S_{t-1},  p = S'^T k,  u = beta (v - p),  S_t = S' + k u^T,
//   o_t = scale S_t^T q
// (the combined update of section 3.3 of "Kimi Linear's Hybrid Linear
// Attention Architecture: A Technical Breakdown"), walking the tokens
// backwards with the adjoint dS of the state:
//   dq = scale S_t do,  dS += scale q do^T,  du = dS^T k,  dk = dS u + S' dp,
//   dbeta = du . (v - p),  dv = beta du,  dp = -beta du,  dS' = dS + k dp^T,
//   dg = alpha * rowsum(dS' * S_{t-1}),  dS_{t-1} = Diag(alpha) dS'.
// This is the recurrent form: exact, and every step is column-local except
// for dq, dk, dg and dbeta, which sum over the dv columns.
//
// Layout: one CTA of 512 threads per (b, h).  In pass 2 warp w owns state
// columns w CW .. w CW + CW - 1 and lane l rows l + 32 i, so the column
// reduction du is a warp shuffle and the sums over columns go through
// shared-memory atomics per token; pass 1, which has no sums over columns,
// gives each thread 16 rows and 2 columns (see fwd_step_rows).
//   Pass 1 (bwd_ckpt_kernel): the forward recurrence from h0, storing S every
//          CK1 = 64 tokens (level-1 checkpoints, fp32, in the workspace) and
//          every token's p = S'^T k (fp32 [T][dv] per (b, h)).  Every later
//          forward step re-runs from a state this pass produced, so it finds
//          the same p and reads it instead of reducing over the rows again:
//          one column reduction per token is left (du), not four.
//   Pass 2 (bwd_kernel): chunks of CK1 tokens from the last to the first.  Per
//          chunk, the forward is re-run from its level-1 checkpoint to leave a
//          state every CK = 4 tokens in a per-(b, h) scratch (level 2); then
//          blocks of CK tokens from the last to the first: for token t of a
//          block, the state before t is recomputed from the block's checkpoint
//          (kept in shared memory) or, past the block's second token, from a
//          thread-private copy of the state before its third token (stored on
//          the way to the last token), then the reverse step.  After each block
//          its tokens' dq, dk (bf16), dg and dbeta (fp32) are written; dv per
//          column as it is formed; dh0 at the end.
// Memory: (ceil(T / 64) + 16) dk dv + T dv fp32 per (b, h); forward steps per token:
// one in pass 1, one for level 2, one on average for the per-token states
// (blocks of 8, with 3.5 recomputed steps per token, were slower).
// Inputs are staged in shared memory per block of tokens, loaded into registers
// one block ahead.  Level-2 states go through global memory (the scratch); the
// reverse walk copies each block's state into one of two shared buffers with
// cp.async while the block before it (in walk order) runs.
#include <cuda_bf16.h>
#include <stdint.h>

#include "bwd_params.cuh"
#include "kda_device.cuh"

namespace kda {

constexpr int BWD_THREADS = 512;
constexpr int BWD_CK1 = 64;  // tokens per level-1 checkpoint
constexpr int BWD_CK = 4;    // tokens per level-2 checkpoint (per block)
constexpr int BWD_FT = 32;   // tokens staged at a time in pass 1

// This lane's CW consecutive state columns of row r (CW a multiple of 4, 16-byte aligned).
template <int CW>
__device__ __forceinline__ void load_row(const float *src, float (&x)[CW]) {
#pragma unroll
    for (int c = 0; c < CW; c += 4) {
        const float4 v = *reinterpret_cast<const float4 *>(src + c);
        x[c] = v.x; x[c + 1] = v.y; x[c + 2] = v.z; x[c + 3] = v.w;
    }
}
// 16-byte asynchronous global -> shared copy (L2 only), and its group fences.
__device__ __forceinline__ void cp_async16(float *dst, const float *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)),
                 "l"(reinterpret_cast<uint64_t>(src))
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <int CW>
__device__ __forceinline__ void store_row(float *dst, const float (&x)[CW]) {
#pragma unroll
    for (int c = 0; c < CW; c += 4) *reinterpret_cast<float4 *>(dst + c) = make_float4(x[c], x[c + 1], x[c + 2], x[c + 3]);
}

// Pass 1's layout: thread (rg, cg) of an 8 x 64 grid holds rows 4 rg + 32 i + r
// (i < DK / 32, r < 4) of the state and columns cg CP .. cg CP + CP - 1 (CP = DV / 64),
// so the column reduction p = (Diag(a) S)^T k is DK / 8 products in the thread and a
// three-level shuffle over the 8 row groups (lanes rg of one cg).  Rows in blocks of
// four make each 16-byte read of k or alpha by 8 lanes one conflict-free wavefront.
// One forward step S <- Diag(a) S + k (beta (v - p))^T; the rg == 0 lanes write p to
// p_out (unless NULL).  Per element the operations are those of fwd_step_p, in the
// same order.
template <int DK, int DV>
__device__ __forceinline__ void fwd_step_rows(float (&S)[DK / 8][DV / 64], const float *sk, const float *sa,
                                              const float *sv, float beta, int rg, int c0, float *p_out) {
    constexpr int RP = DK / 8, CP = DV / 64;
    float kr[RP], p[CP];
#pragma unroll
    for (int c = 0; c < CP; ++c) p[c] = 0.f;
#pragma unroll
    for (int i = 0; i < RP / 4; ++i) {
        const float4 k4 = *reinterpret_cast<const float4 *>(sk + 4 * rg + 32 * i);
        const float4 a4 = *reinterpret_cast<const float4 *>(sa + 4 * rg + 32 * i);
        const float kk[4] = {k4.x, k4.y, k4.z, k4.w}, aa[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            kr[4 * i + r] = kk[r];
#pragma unroll
            for (int c = 0; c < CP; ++c) {
                S[4 * i + r][c] *= aa[r];
                p[c] += kk[r] * S[4 * i + r][c];
            }
        }
    }
#pragma unroll
    for (int o = 1; o < 8; o <<= 1)
#pragma unroll
        for (int c = 0; c < CP; ++c) p[c] += __shfl_xor_sync(0xffffffffu, p[c], o);
    if (rg == 0 && p_out != nullptr) {
        if constexpr (CP == 2) *reinterpret_cast<float2 *>(p_out + c0) = make_float2(p[0], p[1]);
        else p_out[c0] = p[0];
    }
#pragma unroll
    for (int c = 0; c < CP; ++c) {
        const float u = beta * (sv[c0 + c] - p[c]);
#pragma unroll
        for (int i = 0; i < RP; ++i) S[i][c] += kr[i] * u;
    }
}

// The same step with p known (sp: the token's p, staged in shared memory): the
// same operations in the same order, so the same state, without the reduction.
template <int RI, int CW>
__device__ __forceinline__ void fwd_step_p(float (&S)[RI][CW], const float *sk, const float *sa, const float *sv,
                                           const float *sp, float beta, int lane, int col0) {
    float kr[RI];
#pragma unroll
    for (int i = 0; i < RI; ++i) kr[i] = sk[lane + 32 * i];
#pragma unroll
    for (int i = 0; i < RI; ++i) {
        const float a = sa[lane + 32 * i];
#pragma unroll
        for (int c = 0; c < CW; ++c) S[i][c] *= a;
    }
#pragma unroll
    for (int c = 0; c < CW; ++c) {
        const float u = beta * (sv[col0 + c] - sp[col0 + c]);
#pragma unroll
        for (int i = 0; i < RI; ++i) S[i][c] += kr[i] * u;
    }
}

template <int DK, int DV>
__global__ void __launch_bounds__(BWD_THREADS, 1) bwd_ckpt_kernel(const BwdParams prm) {
    constexpr int RP = DK / 8, CP = DV / 64;  // rows and columns of the state per thread
    extern __shared__ __align__(16) float fsm[];
    float *sk = fsm;                      // [FT][DK]
    float *sa = sk + BWD_FT * DK;         // [FT][DK] alpha
    float *sv = sa + BWD_FT * DK;         // [FT][DV]
    float *sb = sv + BWD_FT * DV;         // [FT]
    const int bh = blockIdx.x, b = bh / prm.H, h = bh % prm.H;
    const int T = prm.T, H = prm.H;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int rg = lane & 7, c0 = (warp * 4 + (lane >> 3)) * CP;  // row group, first column
    const int nck = (T + BWD_CK1 - 1) / BWD_CK1;
    float *pbuf = prm.ckpt + (size_t)prm.B * H * (nck + BWD_CK1 / BWD_CK) * DK * DV + (size_t)bh * T * DV;
    if (tid == 0) stamp_start(prm.stamp);
    auto row_of = [&](int j) { return 4 * rg + 32 * (j >> 2) + (j & 3); };  // this thread's j-th row
    float S[RP][CP];
#pragma unroll
    for (int j = 0; j < RP; ++j)
#pragma unroll
        for (int c = 0; c < CP; ++c)
            S[j][c] = prm.h0 ? prm.h0[((size_t)bh * DK + row_of(j)) * DV + c0 + c] : 0.f;
    for (int t0 = 0; t0 < T; t0 += BWD_FT) {
        const int nt = T - t0 < BWD_FT ? T - t0 : BWD_FT;
        __syncthreads();  // the previous block's inputs are no longer read
        for (int e = tid; e < nt * DK; e += BWD_THREADS) {
            const int t = e / DK, r = e % DK;
            const size_t row = ((size_t)b * T + t0 + t) * H + h;
            sk[t * DK + r] = bf16_bits_to_f32(prm.k[row * DK + r]);
            sa[t * DK + r] = __expf(prm.g[row * DK + r]);
        }
        for (int e = tid; e < nt * DV; e += BWD_THREADS) {
            const int t = e / DV, c = e % DV;
            sv[t * DV + c] = bf16_bits_to_f32(prm.v[(((size_t)b * T + t0 + t) * H + h) * DV + c]);
        }
        if (tid < nt) sb[tid] = prm.beta[((size_t)b * T + t0 + tid) * H + h];
        __syncthreads();
        for (int t = 0; t < nt; ++t) {
            if ((t0 + t) % BWD_CK1 == 0 &&  // the state before token t0 + t, into the level-1 region
                KDA_CHECK(prm.st, ((long long)bh * nck + (t0 + t) / BWD_CK1 + 1) * DK * DV <=
                                      (long long)prm.B * H * nck * DK * DV)) {
                float *dst = prm.ckpt + ((size_t)bh * nck + (t0 + t) / BWD_CK1) * DK * DV;
#pragma unroll
                for (int j = 0; j < RP; ++j) {
                    float *d = dst + (size_t)row_of(j) * DV + c0;
                    if constexpr (CP == 2) *reinterpret_cast<float2 *>(d) = make_float2(S[j][0], S[j][1]);
                    else d[0] = S[j][0];
                }
            }
            const bool p_in = KDA_CHECK(prm.st, (pbuf - prm.ckpt) + (long long)(t0 + t + 1) * DV <= prm.ckpt_elems);
            fwd_step_rows<DK, DV>(S, sk + t * DK, sa + t * DK, sv + t * DV, sb[t], rg, c0,
                                  p_in ? pbuf + (size_t)(t0 + t) * DV : nullptr);
        }
    }
    if (tid == 0) stamp_end(prm.stamp);
}

template <int DK, int DV>
__global__ void __launch_bounds__(BWD_THREADS, 1) bwd_kernel(const BwdParams prm) {
    constexpr int RI = DK / 32, CW = DV / 16, CK = BWD_CK;
    // Row stride of a checkpoint tile: lanes own rows, and 16-byte reads of a row
    // by 8 lanes at a time cover all 32 banks once.
    constexpr int LD0 = DV + 4;
    extern __shared__ __align__(16) float fsm[];
    float *s0b = fsm;                // [2][DK][LD0] block checkpoints (double buffer)
    float *sk = s0b + 2 * DK * LD0;  // [CK][DK]
    float *sq = sk + CK * DK;        // [CK][DK]
    float *sa = sq + CK * DK;        // [CK][DK] alpha
    float *sv = sa + CK * DK;        // [CK][DV]
    float *sd = sv + CK * DV;        // [CK][DV] dout
    float *sp = sd + CK * DV;        // [CK][DV] p (from pass 1)
    float *sb = sp + CK * DV;        // [CK] beta
    float *acq = sb + CK;            // [CK][DK] sums over columns: dq
    float *ack = acq + CK * DK;      //                             dk
    float *aca = ack + CK * DK;      //                             d alpha
    float *acb = aca + CK * DK;      // [CK]                        dbeta
    float *sst = acb + CK;           // [RI CW][threads] each thread's state before token 2 of the block
    const int bh = blockIdx.x, b = bh / prm.H, h = bh % prm.H;
    const int T = prm.T, H = prm.H;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, col0 = warp * CW;
    const int nck1 = (T + BWD_CK1 - 1) / BWD_CK1;
    const float scale = prm.scale;

    float dS[RI][CW];
#pragma unroll
    for (int i = 0; i < RI; ++i) {
        if (prm.dhT) {
            load_row<CW>(prm.dhT + ((size_t)bh * DK + lane + 32 * i) * DV + col0, dS[i]);
        } else {
#pragma unroll
            for (int c = 0; c < CW; ++c) dS[i][c] = 0.f;
        }
    }

    float *scratch = prm.ckpt + ((size_t)prm.B * H * nck1 + (size_t)bh * (BWD_CK1 / CK)) * DK * DV;
    const float *pbuf = prm.ckpt + (size_t)prm.B * H * (nck1 + BWD_CK1 / CK) * DK * DV + (size_t)bh * T * DV;
    // The reverse walk's inputs for a block of CK tokens: loaded into registers one
    // block ahead (fetch), converted into the shared tiles at the block's start (put).
    constexpr int PK = (CK * DK + BWD_THREADS - 1) / BWD_THREADS, PV = (CK * DV + BWD_THREADS - 1) / BWD_THREADS;
    uint16_t rk[PK], rq[PK], rv[PV], rd[PV];
    float rg[PK], rp[PV], rb = 0.f;
    int pf_t0 = -1;  // first token of the block held in the registers
    auto fetch = [&](int t0, int nt) {
#pragma unroll
        for (int x = 0; x < PK; ++x) {
            const int e = tid + x * BWD_THREADS, t = e / DK, r = e % DK;
            const bool in = t < nt;
            const size_t row = ((size_t)b * T + (in ? t0 + t : 0)) * H + h;
            rk[x] = in ? prm.k[row * DK + r] : (uint16_t)0;
            rq[x] = in ? prm.q[row * DK + r] : (uint16_t)0;
            rg[x] = in ? prm.g[row * DK + r] : 0.f;
        }
#pragma unroll
        for (int x = 0; x < PV; ++x) {
            const int e = tid + x * BWD_THREADS, t = e / DV, c = e % DV;
            const bool in = t < nt;
            const size_t row = ((size_t)b * T + (in ? t0 + t : 0)) * H + h;
            rv[x] = in ? prm.v[row * DV + c] : (uint16_t)0;
            rd[x] = (in && prm.dout) ? prm.dout[row * DV + c] : (uint16_t)0;
            rp[x] = (in && KDA_CHECK(prm.st, (pbuf - prm.ckpt) + (long long)(t0 + t + 1) * DV <= prm.ckpt_elems))
                        ? pbuf[(size_t)(t0 + t) * DV + c] : 0.f;
        }
        rb = tid < nt ? prm.beta[((size_t)b * T + t0 + tid) * H + h] : 0.f;
        pf_t0 = t0;
    };
    auto put = [&](int nt) {
#pragma unroll
        for (int x = 0; x < PK; ++x) {
            const int e = tid + x * BWD_THREADS;
            if (e < nt * DK) {
                sk[e] = bf16_bits_to_f32(rk[x]);
                sq[e] = bf16_bits_to_f32(rq[x]);
                sa[e] = __expf(rg[x]);
            }
        }
#pragma unroll
        for (int x = 0; x < PV; ++x) {
            const int e = tid + x * BWD_THREADS;
            if (e < nt * DV) {
                sv[e] = bf16_bits_to_f32(rv[x]);
                sd[e] = bf16_bits_to_f32(rd[x]);
                sp[e] = rp[x];
            }
        }
        if (tid < nt) sb[tid] = rb;
    };
    // a level-2 state from the scratch into a checkpoint tile (this thread's share)
    [[maybe_unused]] const long long scratch_end = (long long)prm.B * H * (nck1 + BWD_CK1 / CK) * DK * DV;  // floats
    auto copy_state = [&](float *dst, const float *src) {
        if (!KDA_CHECK(prm.st, (src - prm.ckpt) + (long long)DK * DV <= scratch_end)) {
            cp_async_commit();  // an empty group keeps the waits' counts
            return;
        }
#pragma unroll
        for (int x = 0; x < DK * DV / 4 / BWD_THREADS; ++x) {
            const int e = (tid + x * BWD_THREADS) * 4;
            cp_async16(dst + (e / DV) * LD0 + e % DV, src + e);
        }
        cp_async_commit();
    };

    for (int n = nck1 - 1; n >= 0; --n) {
        const int c0 = n * BWD_CK1;
        const int nb = ((T - c0 < BWD_CK1 ? T - c0 : BWD_CK1) + CK - 1) / CK;  // blocks of the chunk
        {  // level 2: run the chunk forward from its level-1 checkpoint, leaving a state per block
            float S[RI][CW];
            const float *ck = prm.ckpt + ((size_t)bh * nck1 + n) * DK * DV;
            const bool ck_in = KDA_CHECK(prm.st, ((long long)bh * nck1 + n + 1) * DK * DV <=
                                                     (long long)prm.B * H * nck1 * DK * DV);
#pragma unroll
            for (int i = 0; i < RI; ++i) {
                if (ck_in) {
                    load_row<CW>(ck + (size_t)(lane + 32 * i) * DV + col0, S[i]);
                } else {
#pragma unroll
                    for (int c = 0; c < CW; ++c) S[i][c] = 0.f;
                }
            }
            for (int jb = 0; jb < nb; ++jb) {
                const int t0 = c0 + jb * CK;
                const int nt = T - t0 < CK ? T - t0 : CK;
                float *dst = scratch + (size_t)jb * DK * DV;
                if (KDA_CHECK(prm.st, (dst - prm.ckpt) + (long long)DK * DV <= scratch_end)) {
#pragma unroll
                    for (int i = 0; i < RI; ++i) store_row<CW>(dst + (size_t)(lane + 32 * i) * DV + col0, S[i]);
                }
                if (jb + 1 == nb) break;  // the last block's state is not needed past its start
                __syncthreads();          // the previous block's inputs are no longer read
                if (pf_t0 != t0) fetch(t0, nt);
                put(nt);
                __syncthreads();
                {  // the next block's inputs (it exists: jb + 1 < nb), in flight during this one
                    const int t1 = t0 + CK;
                    fetch(t1, T - t1 < CK ? T - t1 : CK);
                }
                for (int t = 0; t < nt; ++t)
                    fwd_step_p<RI, CW>(S, sk + t * DK, sa + t * DK, sv + t * DV, sp + t * DV, sb[t], lane, col0);
            }
        }
    for (int j = nb - 1; j >= 0; --j) {
        const int t0 = c0 + j * CK;
        const int nt = T - t0 < CK ? T - t0 : CK;
        __syncthreads();  // the previous block's tiles and sums have been read; level 2 is written
        const float *s0 = s0b + (j & 1) * DK * LD0;
        if (j == nb - 1) copy_state(s0b + (j & 1) * DK * LD0, scratch + (size_t)j * DK * DV);
        if (j > 0) {  // the next block's state, into the other buffer (last read two blocks ago)
            copy_state(s0b + ((j - 1) & 1) * DK * LD0, scratch + (size_t)(j - 1) * DK * DV);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        if (pf_t0 != t0) fetch(t0, nt);  // the first block walked: nothing was prefetched
        put(nt);
        for (int e = tid; e < CK * DK; e += BWD_THREADS) { acq[e] = 0.f; ack[e] = 0.f; aca[e] = 0.f; }
        if (tid < CK) acb[tid] = 0.f;
        __syncthreads();
        // the inputs of the next block walked, or of the previous chunk's first block
        // (its level-2 pass comes next), in flight during this one
        if (j > 0) fetch(t0 - CK, CK);
        else if (c0 > 0) fetch(c0 - BWD_CK1, CK);

        constexpr int SP = 2;  // the stashed state is the one before the block's token SP
        bool stashed = false;
        for (int tt = nt - 1; tt >= 0; --tt) {
            // the state before token t0 + tt, from the stash or the checkpoint
            float S[RI][CW];
            int s = 0;
            if (tt >= SP && stashed) {
#pragma unroll
                for (int i = 0; i < RI; ++i)
#pragma unroll
                    for (int c = 0; c < CW; ++c) S[i][c] = sst[(i * CW + c) * BWD_THREADS + tid];
                s = SP;
            } else {
#pragma unroll
                for (int i = 0; i < RI; ++i) load_row<CW>(s0 + (lane + 32 * i) * LD0 + col0, S[i]);
            }
            for (; s < tt; ++s) {
                fwd_step_p<RI, CW>(S, sk + s * DK, sa + s * DK, sv + s * DV, sp + s * DV, sb[s], lane, col0);
                if (s + 1 == SP && tt > SP) {  // on the way to a later token: keep the state before SP
#pragma unroll
                    for (int i = 0; i < RI; ++i)
#pragma unroll
                        for (int c = 0; c < CW; ++c) sst[(i * CW + c) * BWD_THREADS + tid] = S[i][c];
                    stashed = true;
                }
            }

            const float *kt = sk + tt * DK, *qt = sq + tt * DK, *at = sa + tt * DK;
            const float *vt = sv + tt * DV, *dot = sd + tt * DV;
            const float bt = sb[tt];
            float kr[RI], qr[RI], ar[RI];
#pragma unroll
            for (int i = 0; i < RI; ++i) {
                kr[i] = kt[lane + 32 * i];
                qr[i] = qt[lane + 32 * i];
                ar[i] = at[lane + 32 * i];
            }
            // The readout's share of dS first (it needs no forward quantity), then the one
            // column reduction du = dS^T k; p = (Diag(a) S)^T k is pass 1's.
            float p[CW], du[CW];
#pragma unroll
            for (int c = 0; c < CW; ++c) {
                const float d = scale * dot[col0 + c];
                float ua = 0.f;
#pragma unroll
                for (int i = 0; i < RI; ++i) {
                    dS[i][c] += qr[i] * d;
                    ua += dS[i][c] * kr[i];
                }
                p[c] = sp[tt * DV + col0 + c];
                du[c] = ua;
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
#pragma unroll
                for (int c = 0; c < CW; ++c) du[c] += __shfl_xor_sync(0xffffffffu, du[c], o);
            float dqp[RI], dkp[RI], dap[RI];
#pragma unroll
            for (int i = 0; i < RI; ++i) { dqp[i] = 0.f; dkp[i] = 0.f; dap[i] = 0.f; }
            float dbp = 0.f;
            const size_t row = ((size_t)b * T + t0 + tt) * H + h;
#pragma unroll
            for (int c = 0; c < CW; ++c) {
                const float vmp = vt[col0 + c] - p[c];
                const float u = bt * vmp;                 // u = beta (v - p)
                const float d = scale * dot[col0 + c];
                dbp += du[c] * vmp;
                const float dp = -bt * du[c];
#pragma unroll
                for (int i = 0; i < RI; ++i) {
                    const float sdv = ar[i] * S[i][c];    // S' = Diag(a) S_{t-1}
                    dqp[i] += (sdv + kr[i] * u) * d;      // dq = scale S_t do
                    dkp[i] += dS[i][c] * u + sdv * dp;    // dk = dS u + S' dp
                    const float dsd = dS[i][c] + kr[i] * dp;
                    dap[i] += dsd * S[i][c];
                    dS[i][c] = ar[i] * dsd;
                }
            }
            if (lane == 0) {  // this warp's CW columns of dv = beta du, one 8- or 16-byte store
                uint32_t w[CW / 2];
#pragma unroll
                for (int c = 0; c < CW; c += 2) w[c / 2] = pack_bf16x2(bt * du[c], bt * du[c + 1]);
                if constexpr (CW == 8)
                    *reinterpret_cast<uint4 *>(prm.dv + row * DV + col0) = make_uint4(w[0], w[1], w[2], w[3]);
                else
                    *reinterpret_cast<uint2 *>(prm.dv + row * DV + col0) = make_uint2(w[0], w[1]);
                atomicAdd(&acb[tt], dbp);
            }
#pragma unroll
            for (int i = 0; i < RI; ++i) {
                atomicAdd(&acq[tt * DK + lane + 32 * i], dqp[i]);
                atomicAdd(&ack[tt * DK + lane + 32 * i], dkp[i]);
                atomicAdd(&aca[tt * DK + lane + 32 * i], dap[i]);
            }
        }
        __syncthreads();
        for (int e = tid; e < nt * DK; e += BWD_THREADS) {
            const int t = e / DK, r = e % DK;
            const size_t row = ((size_t)b * T + t0 + t) * H + h;
            prm.dq[row * DK + r] = to_bf16_bits(acq[e]);
            prm.dk[row * DK + r] = to_bf16_bits(ack[e]);
            prm.dg[row * DK + r] = sa[e] * aca[e];
        }
        if (tid < nt) prm.dbeta[((size_t)b * T + t0 + tid) * H + h] = acb[tid];
    }
    }
    if (prm.dh0) {
#pragma unroll
        for (int i = 0; i < RI; ++i) store_row<CW>(prm.dh0 + ((size_t)bh * DK + lane + 32 * i) * DV + col0, dS[i]);
    }
    __syncthreads();
    if (tid == 0) stamp_end(prm.stamp);
}

template <int DK, int DV>
static cudaError_t launch_bwd_t(const BwdParams &prm, cudaStream_t stream) {
    const int BH = prm.B * prm.H;
    const int s1 = (2 * BWD_FT * DK + BWD_FT * DV + BWD_FT) * 4;
    const int s2 = (2 * DK * (DV + 4) + 3 * BWD_CK * DK + 3 * BWD_CK * DV + BWD_CK + 3 * BWD_CK * DK + BWD_CK + DK * DV) * 4;
    cudaError_t e = cudaFuncSetAttribute(bwd_ckpt_kernel<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, s1);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(bwd_kernel<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, s2);
    if (e != cudaSuccess) return e;
    bwd_ckpt_kernel<DK, DV><<<BH, BWD_THREADS, s1, stream>>>(prm);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    bwd_kernel<DK, DV><<<BH, BWD_THREADS, s2, stream>>>(prm);
    return cudaGetLastError();
}

// Level-1 checkpoints [B H][ceil(T / CK1)] and level-2 scratch [B H][CK1 / CK], each dk x dv
// fp32, then every token's p, [B H][T][dv] fp32.
size_t bwd_ckpt_bytes(int B, int T, int H, int dk, int dv) {
    return (size_t)B * H * ((T + BWD_CK1 - 1) / BWD_CK1 + BWD_CK1 / BWD_CK) * dk * dv * sizeof(float) +
           (size_t)B * H * T * dv * sizeof(float);
}

cudaError_t launch_bwd(const BwdParams &prm, int dk, int dv, cudaStream_t stream) {
    if (dk == 128 && dv == 128) return launch_bwd_t<128, 128>(prm, stream);
    if (dk == 128 && dv == 64) return launch_bwd_t<128, 64>(prm, stream);
    if (dk == 64 && dv == 128) return launch_bwd_t<64, 128>(prm, stream);
    return launch_bwd_t<64, 64>(prm, stream);
}

}  // namespace kda
