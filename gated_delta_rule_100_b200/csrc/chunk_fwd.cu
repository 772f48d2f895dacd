// chunk_fwd.cu -- chunkwise KDA prefill on sm_100a (TMA + tcgen05/TMEM).
//
// Math (per head, per slice of VS = 32 value columns; C = 64 tokens per
// chunk, Gamma = inclusive running sum of g inside the chunk, S0 = state at
// the chunk start, every exp factor taken per key channel):
//   A_ij = beta_i sum_c k_ic k_jc e^{Gamma_ic - Gamma_jc}   (i > j, else 0)
//   P_ij =        sum_c q_ic k_jc e^{Gamma_ic - Gamma_jc}   (i >= j, else 0)
//   T    = (I + A)^{-1}                                   (unit lower)
//   W    = T Diag(beta) (K * e^Gamma),   U = T Diag(beta) V
//   Vnew = U - W S0                                       (the corrected writes)
//   O    = scale ((Q * e^Gamma) S0 + P Vnew)
//   S    = Diag(e^{Gamma_C}) S0 + (K * e^{Gamma_C - Gamma})^T Vnew
// This is the chunkwise rewrite of the KDA recurrence: state passing across
// chunks plus a causal (lower-triangular) intra-chunk correction, section 4
// of "Kimi Linear's Hybrid Linear Attention Architecture: A Technical
// Breakdown", with the intra-chunk rank-1 updates packed into W and U (the WY
// form mentioned in the "Kimi Linear" explainer).
//
// Decay factors.  e^{Gamma_i - Gamma_j} is split into two factors, one per
// side of the contraction over key channels.  Rows of 16-token block I use
// the reference m = 16 I + 8: row factor e^{Gamma_i - Gamma_m}, column factor
// e^{Gamma_m - Gamma_j}.  For j in an earlier block both factors are <= 1; in
// the block itself a factor can exceed 1 and is clamped at e^80, so results
// are exact when a channel's log-decay over one aligned 16-token block is
// >= -160.  All factors come from running products of alpha = e^g (one exp
// per input element) plus one reciprocal per factor above 1.
//
// One CTA (256 threads; threads c and c + 128 share key channel c) owns one
// (b, h, 32-column value slice) and walks its chunks in order:
//   E  alpha, running products; bf16 / tf32 operand tiles, written
//      channel-major with 16-byte stores                       (CUDA cores)
//   F  X * Y^(I) for the four row blocks -> A, P                (UMMA bf16)
//   AP A -> fp32 scratch, P -> tf32 tile                        (TMEM -> smem)
//   T  (I + A)^{-1}: 16x16 diagonal blocks by substitution, off-diagonal
//      blocks by block products, fp32                          (CUDA cores)
//   WU W^T = (beta K e^G)^T T^T and U = T (beta V)              (UMMA tf32)
//   1  [W; Q e^G] S0                                            (UMMA bf16)
//   2  Vnew = U - W S0 -> tf32 tile
//   3  K-hat^T Vnew and O += P Vnew                             (UMMA tf32)
//   4  O -> out (bf16); S = e^{Gamma_C} S0 + K-hat^T Vnew (fp32 registers)
// tf32 UMMA operands are all K-major (the MN-major tf32 form returned zeros
// on sm_100a in a single-MMA probe); bf16 operands are channel-major
// (MN-major) where that lets one thread write a whole row.
#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "chunk_params.cuh"
#include "kda_device.cuh"

namespace kda {

constexpr int CH = 64;          // chunk length
constexpr int SUB = 16;         // sub-block of the decay references
constexpr int NSUB = CH / SUB;  // 4
constexpr int VSL = 32;         // value columns per CTA
constexpr int CHUNK_THREADS = 256;  // two threads per key channel
constexpr int VSH = VSL / 2;        // value columns per thread in the state update
constexpr int A_LD = 68;        // fp32 row stride of the A / T scratch
constexpr float EXP_CLAMP_HI = 5.5406223843935098e34f;  // e^80
constexpr float EXP_CLAMP_LO = 1.8048513878454153e-35f; // e^-80

__host__ __device__ constexpr int align1k(int x) { return (x + 1023) & ~1023; }
__host__ __device__ constexpr int cmax(int a, int b) { return a > b ? a : b; }

template <int DK>
struct ChunkLayout {
    static_assert(DK == 64 || DK == 128, "dk");
    // R_in: TMA destinations, dead after phase E
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + CH * DK * 2;
    static constexpr int OFF_V = OFF_K + CH * DK * 2;
    static constexpr int IN_B = align1k(2 * CH * DK * 2 + CH * VSL * 2);
    // R_form: formation operands (E..F), then A, T scratch, T, P, Vnew^T
    static constexpr int OFF_F = IN_B;
    static constexpr int OFF_X = OFF_F;                      // MN-major bf16 [DK][128]
    static constexpr int OFF_Y0 = OFF_X + DK * 256;          // SW32  [DK][16]
    static constexpr int OFF_Y1 = OFF_Y0 + DK * 32;          // SW64  [DK][32]
    static constexpr int OFF_Y2 = OFF_Y1 + DK * 64;          // SW128 [DK][64] (48 used)
    static constexpr int OFF_Y3 = OFF_Y2 + DK * 128;         // SW128 [DK][64]
    static constexpr int FORM_B = DK * (256 + 32 + 64 + 128 + 128);
    static constexpr int OFF_A = OFF_F;                      // fp32 [64][A_LD]
    static constexpr int OFF_TF = OFF_A + 64 * A_LD * 4;     // fp32 [64][A_LD]
    static constexpr int OFF_T = OFF_F + align1k(2 * 64 * A_LD * 4);  // tf32 K-major rows 0..63, K-block stride 8 KB
    static constexpr int OFF_PB = OFF_T + 8192;              // descriptor base of [junk; P]: P rows 64..127
    static constexpr int OFF_VN = OFF_PB + 24576;            // tf32 K-major Vnew^T [32][64]
    static constexpr int OFF_ZS = OFF_VN;                    // T-solve scratch (before Vnew^T exists)
    static constexpr int POST_B = OFF_VN + VSL * 64 * 4 - OFF_F;
    static constexpr int RF_B = align1k(cmax(FORM_B, POST_B));
    // operand tiles that live until the chain
    static constexpr int OFF_BK = OFF_F + RF_B;              // tf32 K-major (beta K e^G)^T [128][64]
    static constexpr int OFF_BV = OFF_BK + 128 * 64 * 4;     // tf32 K-major (beta V)^T [32][64]
    static constexpr int OFF_KH = OFF_BV + VSL * 64 * 4;     // tf32 K-major K-hat^T [128][64]
    static constexpr int OFF_WQ = OFF_KH + 128 * 64 * 4;     // bf16 MN-major [W; Q e^G] [DK][128]
    static constexpr int OFF_S = OFF_WQ + DK * 256;          // bf16 MN-major S0 [DK][32] (SW64)
    static constexpr int OFF_MISC = OFF_S + DK * VSL * 2;    // beta, e^{Gamma_C}, barriers, TMEM address
    static constexpr int TOTAL = OFF_MISC + 1024;
    static constexpr int SMEM_BYTES = TOTAL + 1024;          // slack for the 1 KB base alignment
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
    static_assert(POST_B <= RF_B && FORM_B <= RF_B, "R_form");

    // TMEM columns
    static constexpr uint32_t TM_AP = 0;    // 160: formation products D^(I)
    static constexpr uint32_t TM_W = 160;   // 64: W^T (lane = key channel, column = token)
    static constexpr uint32_t TM_U = 224;   // 32: U (lane = token)
    static constexpr uint32_t TM_D1 = 256;  // 32: [W; Q e^G] S0, then += P Vnew on rows 64..127
    static constexpr uint32_t TM_D3 = 288;  // 32: K-hat^T Vnew (lane = key channel)
    static constexpr uint32_t TM_COLS = 512;
};

// First TMEM column / Y row of block I's formation product: 16 * I (I + 1) / 2.
__device__ __forceinline__ constexpr int yoff(int I) { return SUB * (I * (I + 1) / 2); }

__device__ __forceinline__ float rcp_clamped(float p) {
    return p < EXP_CLAMP_LO ? EXP_CLAMP_HI : __fdividef(1.0f, p);
}

__device__ __forceinline__ uint4 pack8_bf16(const float (&v)[8]) {
    return make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                      pack_bf16x2(v[6], v[7]));
}

__device__ __forceinline__ uint4 pack4_tf32(float a, float b, float c, float d) {
    return make_uint4(to_tf32(a), to_tf32(b), to_tf32(c), to_tf32(d));
}

template <int DK>
__global__ void __launch_bounds__(CHUNK_THREADS, 1)
chunk_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const float *__restrict__ gptr,
                 const ChunkParams prm) {
    using L = ChunkLayout<DK>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(sm);

    float *s_beta = reinterpret_cast<float *>(sm + L::OFF_MISC);        // [64]
    float *s_dec = reinterpret_cast<float *>(sm + L::OFF_MISC + 256);   // [128]: e^{Gamma_C} per key channel
    uint64_t *s_bars = reinterpret_cast<uint64_t *>(sm + L::OFF_MISC + 768);
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(sm + L::OFF_MISC + 800);
    int *s_abort = reinterpret_cast<int *>(sm + L::OFF_MISC + 808);
    const uint32_t bar_in = smem_u32(&s_bars[0]);
    const uint32_t bar_mma = smem_u32(&s_bars[1]);
    const uint32_t bar_never = smem_u32(&s_bars[2]);  // nothing arrives on it (fault-injection hook)

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int ch = tid & 127;        // key channel / TMEM lane of this thread
    const int half = tid >> 7;       // which of the channel's two threads
    const int unit = blockIdx.x;
    const int slice = unit % prm.nslices;
    const int bh = unit / prm.nslices;
    const int h = bh % prm.H, b = bh / prm.H;
    const int T = prm.T, H = prm.H, DV = prm.DV;
    const int col0 = slice * VSL;
    const uint64_t polls = prm.st.wait_polls;

    if (tid == 0) {
        mbar_init(bar_in, 1);
        mbar_init(bar_mma, 1);
        mbar_init(bar_never, 1);
        fence_mbar_init();
        *s_abort = 0;
        prefetch_tmap(&tm_q); prefetch_tmap(&tm_k); prefetch_tmap(&tm_v);
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(s_tmem), L::TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;  // this warp's TMEM lanes

    // ---- state: thread (ch, half) holds S[ch][16 half .. 16 half + 15] in fp32 ----
    float S[VSH];
#pragma unroll
    for (int n = 0; n < VSH; ++n) S[n] = 0.f;
    const int scol = col0 + half * VSH;
    if (ch < DK && prm.h0 != nullptr) {
        const float *src = prm.h0 + (((size_t)b * H + h) * DK + ch) * DV + scol;
#pragma unroll
        for (int n = 0; n < VSH; n += 4) {
            const float4 x = *reinterpret_cast<const float4 *>(src + n);
            S[n] = x.x; S[n + 1] = x.y; S[n + 2] = x.z; S[n + 3] = x.w;
        }
    }
    auto store_state_bf16 = [&]() {
        if (ch < DK) {
#pragma unroll
            for (int n = 0; n < VSH; n += 8) {
                float v8[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) v8[e] = S[n + e];
                *reinterpret_cast<uint4 *>(sm + L::OFF_S + mnmaj<64, 2>(ch, half * VSH + n, DK)) = pack8_bf16(v8);
            }
        }
    };
    store_state_bf16();

    const int nchunks = (T + CH - 1) / CH;
    constexpr uint32_t IN_TX = (uint32_t)(2 * CH * DK * 2 + CH * VSL * 2);
    auto issue_loads = [&](int n) {
        const int t0 = n * CH;
        mbar_expect_tx(bar_in, IN_TX);
#pragma unroll
        for (int kb = 0; kb < DK / 64; ++kb) {
            tma_load_4d(sbase + L::OFF_Q + kb * CH * 128, &tm_q, bar_in, kb * 64, h, t0, b);
            tma_load_4d(sbase + L::OFF_K + kb * CH * 128, &tm_k, bar_in, kb * 64, h, t0, b);
        }
        tma_load_4d(sbase + L::OFF_V, &tm_v, bar_in, col0, h, t0, b);
    };
    // g (fp32) of one chunk for channel tid, straight from global into registers
    float al[CH];
    auto load_g = [&](int n) {
        const int t0 = n * CH;
        const int Lc = min(CH, T - t0);
        const float *gp = gptr + (((size_t)b * T + t0) * H + h) * DK + ch;
#pragma unroll
        for (int t = 0; t < CH; ++t) al[t] = (t < Lc && ch < DK) ? __ldg(gp + (size_t)t * H * DK) : 0.f;
    };
    auto load_beta = [&](int n) -> float {
        const int t0 = n * CH;
        return (tid < CH && t0 + tid < T) ? prm.beta[((size_t)b * T + t0 + tid) * H + h] : 0.f;
    };

    uint32_t ph_in = 0, ph_mma = 0;
    bool tma_pending = false, mma_pending = false, aborted = false;

    // all threads wait; returns false (uniformly) when any thread gave up
    auto wait_all = [&](uint32_t bar, uint32_t &ph, bool &pending) -> bool {
        const bool ok = mbar_wait(bar, ph, polls, prm.st);
        if (!ok) atomicExch(s_abort, 1);
        __syncthreads();
        if (*s_abort) return false;
        ph ^= 1u;
        pending = false;
        tc_fence_after();
        return true;
    };
    auto sync_for_mma = [&]() {  // smem operands written by threads -> visible to UMMA
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    };

    if (nchunks > 0) {
        if (tid == 0) issue_loads(0);
        tma_pending = true;
        load_g(0);
    }
    float beta_next = nchunks > 0 ? load_beta(0) : 0.f;

    if (prm.inject_wait_polls != 0) {
        // Fault-injection hook: wait on a barrier nothing arrives on, so the
        // bounded wait gives up and the kernel takes its error path.
        if (!mbar_wait(bar_never, 0u, prm.inject_wait_polls, prm.st)) atomicExch(s_abort, 1);
        __syncthreads();
        if (*s_abort) aborted = true;
    }

    for (int n = 0; n < nchunks && !aborted; ++n) {
        const int t0 = n * CH;
        const int Lc = min(CH, T - t0);

        // ---------------- inputs ----------------
        if (tid < CH) s_beta[tid] = beta_next;
        if (!wait_all(bar_in, ph_in, tma_pending)) { aborted = true; break; }

        // ---------------- E: decay factors and operand tiles ----------------
        // half 0: e^{Gamma} (Q e^G, (beta K e^G)^T), e^{Gamma_C - Gamma} (K-hat^T), X rows
        // half 1: Y^(I) columns, (beta V)^T
        if (ch < DK) {
            const int c = ch;
            const uint8_t *qs = sm + L::OFF_Q, *ks = sm + L::OFF_K;
            auto kval = [&](int i) { return bf16_bits_to_f32(*reinterpret_cast<const uint16_t *>(ks + kmaj<128, 2>(i, c, CH))); };
            auto qval = [&](int i) { return bf16_bits_to_f32(*reinterpret_cast<const uint16_t *>(qs + kmaj<128, 2>(i, c, CH))); };
#pragma unroll
            for (int t = 0; t < CH; ++t) al[t] = __expf(al[t]);

            if (half == 0) {
                float pre = 1.f;
#pragma unroll
                for (int g8 = 0; g8 < CH / 8; ++g8) {
                    float qv[8], bk[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const int t = g8 * 8 + u;
                        pre *= al[t];
                        qv[u] = qval(t) * pre;
                        bk[u] = s_beta[t] * kval(t) * pre;
                    }
                    *reinterpret_cast<uint4 *>(sm + L::OFF_WQ + mnmaj<128, 2>(c, 64 + g8 * 8, DK)) = pack8_bf16(qv);
                    *reinterpret_cast<uint4 *>(sm + L::OFF_BK + kmaj<128, 4>(c, g8 * 8, 128)) = pack4_tf32(bk[0], bk[1], bk[2], bk[3]);
                    *reinterpret_cast<uint4 *>(sm + L::OFF_BK + kmaj<128, 4>(c, g8 * 8 + 4, 128)) = pack4_tf32(bk[4], bk[5], bk[6], bk[7]);
                }
                s_dec[c] = pre;
                float suf = 1.f;
#pragma unroll
                for (int g4 = CH / 4 - 1; g4 >= 0; --g4) {
                    float kh[4];
#pragma unroll
                    for (int u = 3; u >= 0; --u) {
                        const int t = g4 * 4 + u;
                        kh[u] = kval(t) * suf;
                        suf *= al[t];
                    }
                    *reinterpret_cast<uint4 *>(sm + L::OFF_KH + kmaj<128, 4>(c, g4 * 4, 128)) = pack4_tf32(kh[0], kh[1], kh[2], kh[3]);
                }
                // X rows of block I (reference m = 16 I + 8): F_t = e^{Gamma_t - Gamma_m}
#pragma unroll
                for (int I = 0; I < NSUB; ++I) {
                    const int m = SUB * I + SUB / 2;
                    float xk[8], xq[8];
                    float p = 1.f;
#pragma unroll
                    for (int u = 0; u < 8; ++u) {  // tokens m .. m+7
                        const int t = m + u;
                        if (u > 0) p *= al[t];
                        xk[u] = kval(t) * p;
                        xq[u] = qval(t) * p;
                    }
                    *reinterpret_cast<uint4 *>(sm + L::OFF_X + mnmaj<128, 2>(c, m, DK)) = pack8_bf16(xk);
                    *reinterpret_cast<uint4 *>(sm + L::OFF_X + mnmaj<128, 2>(c, 64 + m, DK)) = pack8_bf16(xq);
                    float y = 1.f;
#pragma unroll
                    for (int u = 7; u >= 0; --u) {  // tokens m-1 down to 16 I
                        const int t = SUB * I + u;
                        y *= al[t + 1];
                        const float r = rcp_clamped(y);
                        xk[u] = kval(t) * r;
                        xq[u] = qval(t) * r;
                    }
                    *reinterpret_cast<uint4 *>(sm + L::OFF_X + mnmaj<128, 2>(c, SUB * I, DK)) = pack8_bf16(xk);
                    *reinterpret_cast<uint4 *>(sm + L::OFF_X + mnmaj<128, 2>(c, 64 + SUB * I, DK)) = pack8_bf16(xq);
                }
            } else {
                // Y^(I) columns j <= 16 I + 15: e^{Gamma_m - Gamma_j}
#pragma unroll
                for (int I = 0; I < NSUB; ++I) {
                    const int m = SUB * I + SUB / 2;
                    const int yofs = I == 0 ? L::OFF_Y0 : I == 1 ? L::OFF_Y1 : I == 2 ? L::OFF_Y2 : L::OFF_Y3;
                    auto yput = [&](int j0, const float (&v)[8]) {
                        uint8_t *dst = sm + yofs;
                        if (I == 0)      *reinterpret_cast<uint4 *>(dst + mnmaj<32, 2>(c, j0, DK)) = pack8_bf16(v);
                        else if (I == 1) *reinterpret_cast<uint4 *>(dst + mnmaj<64, 2>(c, j0, DK)) = pack8_bf16(v);
                        else             *reinterpret_cast<uint4 *>(dst + mnmaj<128, 2>(c, j0, DK)) = pack8_bf16(v);
                    };
                    {
                        float yv[8];
                        float p = 1.f;
#pragma unroll
                        for (int u = 0; u < 8; ++u) {  // tokens m .. m+7: 1 / prod_{s=m+1..t} alpha_s
                            const int t = m + u;
                            if (u > 0) p *= al[t];
                            yv[u] = u == 0 ? kval(t) : kval(t) * rcp_clamped(p);
                        }
                        yput(m, yv);
                    }
                    float y = 1.f;
#pragma unroll
                    for (int g8 = m / 8 - 1; g8 >= 0; --g8) {  // tokens below m: prod_{s=t+1..m} alpha_s
                        float yv[8];
#pragma unroll
                        for (int u = 7; u >= 0; --u) {
                            const int t = g8 * 8 + u;
                            y *= al[t + 1];
                            yv[u] = kval(t) * y;
                        }
                        yput(g8 * 8, yv);
                    }
                }
            }
        }
        if (half == 1 && ch >= DK - VSL && ch < DK) {  // (beta V)^T: row n = value column
            const int nn = ch - (DK - VSL);
            const uint16_t *vs = reinterpret_cast<const uint16_t *>(sm + L::OFF_V);
#pragma unroll
            for (int g4 = 0; g4 < CH / 4; ++g4) {
                float w[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int t = g4 * 4 + u;
                    w[u] = s_beta[t] * bf16_bits_to_f32(vs[t * VSL + nn]);
                }
                *reinterpret_cast<uint4 *>(sm + L::OFF_BV + kmaj<128, 4>(nn, g4 * 4, VSL)) = pack4_tf32(w[0], w[1], w[2], w[3]);
            }
        }
        sync_for_mma();

        // ---------------- F: formation products (bf16) ----------------
        if (tid == 0) {
            if (n + 1 < nchunks) issue_loads(n + 1);  // R_in is consumed: prefetch
#pragma unroll
            for (int I = 0; I < NSUB; ++I) {
                const uint32_t idesc = make_idesc(1, true, true, 128, SUB * (I + 1));
#pragma unroll
                for (int kk = 0; kk < DK / 16; ++kk) {
                    const uint64_t da = desc_mnmaj<128>(sbase + L::OFF_X, DK, kk * 16);
                    uint64_t db;
                    if (I == 0)      db = desc_mnmaj<32>(sbase + L::OFF_Y0, DK, kk * 16);
                    else if (I == 1) db = desc_mnmaj<64>(sbase + L::OFF_Y1, DK, kk * 16);
                    else if (I == 2) db = desc_mnmaj<128>(sbase + L::OFF_Y2, DK, kk * 16);
                    else             db = desc_mnmaj<128>(sbase + L::OFF_Y3, DK, kk * 16);
                    umma<0>(tmem + L::TM_AP + yoff(I), da, db, idesc, kk > 0);
                }
            }
            umma_commit(bar_mma);
        }
        tma_pending = n + 1 < nchunks;
        mma_pending = true;
        beta_next = n + 1 < nchunks ? load_beta(n + 1) : 0.f;
        if (!wait_all(bar_mma, ph_mma, mma_pending)) { aborted = true; break; }

        // ---------------- AP: A -> fp32 scratch, P -> tf32 tile ----------------
        // TMEM lane = row of [k; q]; the two warps of a lane quarter split the
        // four 16-column chunks of each row (half 0: chunks 0-1, half 1: 2-3).
        {
            float *sA = reinterpret_cast<float *>(sm + L::OFF_A);
            const int row = ch;
            const int i = row & 63;
            const int myI = i / SUB;
            const bool is_q = row >= 64;
            const float bi = s_beta[i];
            const int I0 = (((warp & 3) & 1) * 32) / SUB;  // the lane quarter covers blocks I0, I0 + 1
#pragma unroll
            for (int c2 = 0; c2 < 2; ++c2) {
                const int cc = half * 2 + c2;
                float v16[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) v16[e] = 0.f;
#pragma unroll
                for (int dI = 0; dI < 2; ++dI) {
                    const int I = I0 + dI;
                    if (cc <= I) {
                        float t[16];
                        tmem_ld16(tmem + lane_base + L::TM_AP + yoff(I) + cc * 16, t);
                        tmem_wait_ld();
                        if (myI == I) {
#pragma unroll
                            for (int e = 0; e < 16; ++e) v16[e] = t[e];
                        }
                    }
                }
                const int j0 = cc * 16;
                if (!is_q) {
#pragma unroll
                    for (int e = 0; e < 16; e += 4) {
                        float4 w;
                        w.x = (j0 + e + 0 < i) ? bi * v16[e + 0] : 0.f;
                        w.y = (j0 + e + 1 < i) ? bi * v16[e + 1] : 0.f;
                        w.z = (j0 + e + 2 < i) ? bi * v16[e + 2] : 0.f;
                        w.w = (j0 + e + 3 < i) ? bi * v16[e + 3] : 0.f;
                        *reinterpret_cast<float4 *>(sA + i * A_LD + j0 + e) = w;
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 16; e += 4) {
                        uint4 w;
                        w.x = (j0 + e + 0 <= i) ? to_tf32(v16[e + 0]) : 0u;
                        w.y = (j0 + e + 1 <= i) ? to_tf32(v16[e + 1]) : 0u;
                        w.z = (j0 + e + 2 <= i) ? to_tf32(v16[e + 2]) : 0u;
                        w.w = (j0 + e + 3 <= i) ? to_tf32(v16[e + 3]) : 0u;
                        *reinterpret_cast<uint4 *>(sm + L::OFF_PB + kmaj_s<128, 4>(64 + i, j0 + e, 8192)) = w;
                    }
                }
            }
        }
        tc_fence_before();
        __syncthreads();

        // ---------------- T: (I + A)^{-1}, fp32 ----------------
        {
            const float *sA = reinterpret_cast<const float *>(sm + L::OFF_A);
            float *sTf = reinterpret_cast<float *>(sm + L::OFF_TF);
            float *sZ = reinterpret_cast<float *>(sm + L::OFF_ZS);
            // diagonal 16x16 blocks: thread (I, jj) solves column jj of (I + A_II) x = e_jj
            if (tid < 64) {
                const int I = tid >> 4, jj = tid & 15, base = SUB * I;
                float x[SUB];
#pragma unroll
                for (int ii = 0; ii < SUB; ++ii) {
                    float acc = (ii == jj) ? 1.f : 0.f;
#pragma unroll
                    for (int mm = 0; mm < ii; ++mm) acc -= sA[(base + ii) * A_LD + base + mm] * x[mm];
                    x[ii] = (ii < jj) ? 0.f : acc;
                }
#pragma unroll
                for (int ii = 0; ii < SUB; ++ii) sTf[(base + ii) * A_LD + base + jj] = x[ii];
            }
            __syncthreads();
            // off-diagonal blocks by distance d: T_{I,J} = -T_II sum_{K=J}^{I-1} A_IK T_KJ, J = I - d
#pragma unroll
            for (int d = 1; d < NSUB; ++d) {
                const int nt = NSUB - d;
                for (int e = tid; e < nt * 256; e += CHUNK_THREADS) {
                    const int blk = e >> 8, I = d + blk, J = blk, r = (e >> 4) & 15, cc = e & 15;
                    float acc = 0.f;
                    for (int K = J; K < I; ++K) {
                        const float *arow = sA + (SUB * I + r) * A_LD + SUB * K;
#pragma unroll
                        for (int m4 = 0; m4 < SUB; m4 += 4) {
                            const float4 a4 = *reinterpret_cast<const float4 *>(arow + m4);
                            const float *tc = sTf + (SUB * K + m4) * A_LD + SUB * J + cc;
                            acc += a4.x * tc[0] + a4.y * tc[A_LD] + a4.z * tc[2 * A_LD] + a4.w * tc[3 * A_LD];
                        }
                    }
                    sZ[blk * 256 + r * 16 + cc] = acc;
                }
                __syncthreads();
                for (int e = tid; e < nt * 256; e += CHUNK_THREADS) {
                    const int blk = e >> 8, I = d + blk, J = blk, r = (e >> 4) & 15, cc = e & 15;
                    const float *trow = sTf + (SUB * I + r) * A_LD + SUB * I;
                    float acc = 0.f;
#pragma unroll
                    for (int m4 = 0; m4 < SUB; m4 += 4) {
                        const float4 t4 = *reinterpret_cast<const float4 *>(trow + m4);  // zero above the diagonal
                        const float *z = sZ + blk * 256 + m4 * 16 + cc;
                        acc += t4.x * z[0] + t4.y * z[16] + t4.z * z[32] + t4.w * z[48];
                    }
                    sTf[(SUB * I + r) * A_LD + SUB * J + cc] = -acc;
                }
                __syncthreads();
            }
            // T -> tf32 K-major tile (rows 0..63, K-block stride 8 KB), zeros above the diagonal
            for (int e = tid; e < 64 * 16; e += CHUNK_THREADS) {
                const int i = e >> 4, j = (e & 15) * 4;
                const float *src = sTf + i * A_LD + j;
                *reinterpret_cast<uint4 *>(sm + L::OFF_T + kmaj_s<128, 4>(i, j, 8192)) =
                    pack4_tf32(j + 0 <= i ? src[0] : 0.f, j + 1 <= i ? src[1] : 0.f,
                               j + 2 <= i ? src[2] : 0.f, j + 3 <= i ? src[3] : 0.f);
            }
        }
        sync_for_mma();

        // ---------------- WU: W^T = (beta K e^G)^T T^T,  U = T (beta V)  (tf32) ----------------
        if (tid == 0) {
            const uint32_t id_w = make_idesc(2, false, false, 128, 64);
            const uint32_t id_u = make_idesc(2, false, false, 128, VSL);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                umma<1>(tmem + L::TM_W, desc_kmaj_s<128, 4>(sbase + L::OFF_BK, 128 * 128, kk * 8),
                        desc_kmaj_s<128, 4>(sbase + L::OFF_T, 8192, kk * 8), id_w, kk > 0);
                umma<1>(tmem + L::TM_U, desc_kmaj_s<128, 4>(sbase + L::OFF_T, 8192, kk * 8),
                        desc_kmaj_s<128, 4>(sbase + L::OFF_BV, VSL * 128, kk * 8), id_u, kk > 0);
            }
            umma_commit(bar_mma);
        }
        mma_pending = true;
        if (!wait_all(bar_mma, ph_mma, mma_pending)) { aborted = true; break; }
        if (n + 1 < nchunks) load_g(n + 1);  // consumed at the next chunk's phase E
        if (ch < DK) {  // W^T row ch -> W columns of [W; Q e^G]; half h takes tokens 32 h .. 32 h + 31
#pragma unroll
            for (int i0 = half * 32; i0 < half * 32 + 32; i0 += 16) {
                float t[16];
                tmem_ld16(tmem + lane_base + L::TM_W + i0, t);
                tmem_wait_ld();
                float a8[8], b8[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) { a8[e] = t[e]; b8[e] = t[8 + e]; }
                *reinterpret_cast<uint4 *>(sm + L::OFF_WQ + mnmaj<128, 2>(ch, i0, DK)) = pack8_bf16(a8);
                *reinterpret_cast<uint4 *>(sm + L::OFF_WQ + mnmaj<128, 2>(ch, i0 + 8, DK)) = pack8_bf16(b8);
            }
        }
        sync_for_mma();

        // ---------------- 1: [W; Q e^G] S0 (bf16) ----------------
        if (tid == 0) {
            const uint32_t idesc = make_idesc(1, true, true, 128, VSL);
#pragma unroll
            for (int kk = 0; kk < DK / 16; ++kk)
                umma<0>(tmem + L::TM_D1, desc_mnmaj<128>(sbase + L::OFF_WQ, DK, kk * 16),
                        desc_mnmaj<64>(sbase + L::OFF_S, DK, kk * 16), idesc, kk > 0);
            umma_commit(bar_mma);
        }
        mma_pending = true;
        if (!wait_all(bar_mma, ph_mma, mma_pending)) { aborted = true; break; }

        // ---------------- 2: Vnew = U - W S0 -> Vnew^T tile (tf32) ----------------
        if ((warp & 3) < 2) {  // lanes 0..63 = tokens; half picks 16 of the 32 columns
            const int i = ch;
            const int n0 = half * VSH;
            float u[16], ws[16];
            tmem_ld16(tmem + lane_base + L::TM_U + n0, u);
            tmem_ld16(tmem + lane_base + L::TM_D1 + n0, ws);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e)
                *reinterpret_cast<uint32_t *>(sm + L::OFF_VN + kmaj_s<128, 4>(n0 + e, i, VSL * 128)) = to_tf32(u[e] - ws[e]);
        }
        sync_for_mma();

        // ---------------- 3: K-hat^T Vnew;  O += P Vnew  (tf32) ----------------
        if (tid == 0) {
            const uint32_t idesc = make_idesc(2, false, false, 128, VSL);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint64_t bvn = desc_kmaj_s<128, 4>(sbase + L::OFF_VN, VSL * 128, kk * 8);
                umma<1>(tmem + L::TM_D3, desc_kmaj_s<128, 4>(sbase + L::OFF_KH, 128 * 128, kk * 8), bvn, idesc, kk > 0);
                umma<1>(tmem + L::TM_D1, desc_kmaj_s<128, 4>(sbase + L::OFF_PB, 8192, kk * 8), bvn, idesc, 1u);
            }
            umma_commit(bar_mma);
        }
        mma_pending = true;
        if (!wait_all(bar_mma, ph_mma, mma_pending)) { aborted = true; break; }

        // ---------------- 4: output and state update ----------------
        if ((warp & 3) >= 2) {  // lanes 64..127 = output rows
            const int i = ch - 64;
            const int n0 = half * VSH;
            float t[16];
            tmem_ld16(tmem + lane_base + L::TM_D1 + n0, t);
            tmem_wait_ld();
            if (i < Lc) {
                uint16_t *dst = prm.out + (((size_t)b * T + t0 + i) * H + h) * DV + col0 + n0;
                float a8[8], b8[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) { a8[e] = prm.scale * t[e]; b8[e] = prm.scale * t[8 + e]; }
                reinterpret_cast<uint4 *>(dst)[0] = pack8_bf16(a8);
                reinterpret_cast<uint4 *>(dst)[1] = pack8_bf16(b8);
            }
        }
        if ((warp & 3) < DK / 32) {
            float t[16];
            tmem_ld16(tmem + lane_base + L::TM_D3 + half * VSH, t);
            tmem_wait_ld();
            const float dc = s_dec[ch];
#pragma unroll
            for (int e = 0; e < VSH; ++e) S[e] = dc * S[e] + t[e];
        }
        store_state_bf16();
        tc_fence_before();
        __syncthreads();
    }

    if (aborted) {
        // Leave nothing in flight that targets this CTA's smem or TMEM.
        if (tid == 0) {
            if (tma_pending) mbar_wait(bar_in, ph_in, ~0ull, prm.st);
            if (mma_pending) mbar_wait(bar_mma, ph_mma, ~0ull, prm.st);
        }
        tc_fence_before();
        __syncthreads();
    } else if (prm.hT != nullptr && ch < DK) {
        float *dst = prm.hT + (((size_t)b * H + h) * DK + ch) * DV + scol;
#pragma unroll
        for (int n = 0; n < VSH; n += 4)
            *reinterpret_cast<float4 *>(dst + n) = make_float4(S[n], S[n + 1], S[n + 2], S[n + 3]);
    }
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, L::TM_COLS);
}

// ------------------------------------------------------------------- host ----
template <int DK>
static cudaError_t launch_chunk_t(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                  const float *g, const ChunkParams &prm, int units, cudaStream_t stream) {
    using L = ChunkLayout<DK>;
    cudaError_t e = cudaFuncSetAttribute(chunk_fwd_kernel<DK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         L::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    chunk_fwd_kernel<DK><<<units, CHUNK_THREADS, L::SMEM_BYTES, stream>>>(tq, tk, tv, g, prm);
    return cudaGetLastError();
}

int chunk_value_slice() { return VSL; }

cudaError_t launch_chunk(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv, const float *g,
                         const ChunkParams &prm, int dk, cudaStream_t stream) {
    const int units = prm.B * prm.H * prm.nslices;
    if (dk == 128) return launch_chunk_t<128>(tq, tk, tv, g, prm, units, stream);
    return launch_chunk_t<64>(tq, tk, tv, g, prm, units, stream);
}

}  // namespace kda
