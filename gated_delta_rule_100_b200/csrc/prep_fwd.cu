// prep_fwd.cu -- the intra-chunk half of the chunkwise KDA prefill (sm_100a).
//
// Per chunk of C = 64 tokens of one head (Gamma = inclusive running sum of g
// inside the chunk, every exp factor per key channel):
//   A_ij = beta_i sum_c k_ic k_jc e^{Gamma_ic - Gamma_jc}   (i > j, else 0)
//   P_ij =        sum_c q_ic k_jc e^{Gamma_ic - Gamma_jc}   (i >= j, else 0)
//   T    = (I + A)^{-1}                                   (unit lower)
//   T'   = T Diag(beta),   W = T' (K * e^Gamma)
//   plus Q * e^Gamma, K-hat = K * e^{Gamma_C - Gamma} and e^{Gamma_C}.
// These are the intra-chunk pieces of the chunkwise rewrite of the KDA
// recurrence (section 4 of "Kimi Linear's Hybrid Linear Attention
// Architecture: A Technical Breakdown"), with the chunk's rank-1 updates
// packed in the WY form (W, and U = T' V in the chain kernel).
// None of them depends on the state, so chunks are independent work items;
// each result goes to a per-chunk record (layout in chunk_common.cuh).
//
// Decay factors.  e^{Gamma_i - Gamma_j} is split into two factors, one per
// side of the contraction over key channels.  In a mild chunk (every key
// channel keeps e^{Gamma_C} >= e^-40, which covers ordinary gates) the chunk's
// start is the reference: row factor e^{Gamma_i}, column factor e^{-Gamma_j},
// both within [e^-40, e^40], so the formation operands X = [K e^G; Q e^G] and
// Y = K e^{-G} are products the record needs anyway and one 64-column product
// forms A and P.  Otherwise rows of 16-token block I use
// the reference m = 16 I + 8: row factor e^{Gamma_i - Gamma_m}, column factor
// e^{Gamma_m - Gamma_j}.  For j in an earlier block both factors are <= 1; in
// the block itself a factor can exceed 1.  It stays below e^80 unless some key
// channel loses more than 80 of log-decay over tokens 16 I + 1 .. 16 I + 8 or
// 16 I + 9 .. 16 I + 15.  Such a "steep" item is flagged in phase E (its
// factors are clamped at e^80 meanwhile, so nothing overflows) and appended to
// a list; the exact kernel (exact_prep.cu) then rewrites its P, T' and W from
// pairwise factors e^{Gamma_i - Gamma_j} <= 1 before the chain reads them.  So
// results are exact up to rounding for any finite g <= 0, and only items with
// extreme decay pay for the slow path.  All factors of this kernel come from
// running products of alpha = e^g (one exp per input element) plus one
// reciprocal per factor above 1.
//
// Persistent CTAs (two per SM, 512 threads) claim items from a counter; while
// one item is processed the next one's q, k and g are prefetched into L2.  In the
// elementwise phase thread (c, I) owns key channel c and tokens 16 I .. 16 I +
// 15 (a two-level scan: products inside the block, then the four block
// totals through shared memory); its key and query values are held as bf16
// pairs, so the phase fits in 64 registers.  Phases per item:
//   E  alpha, running products; operand tiles X, Y^(I) (bf16, smem) for the
//      formation; Q e^G, K-hat (record); (K e^G)^T (tf32, smem)
//   F  X Y^(I)^T -> A, P                    (UMMA bf16, overlapped with E's tail;
//      a mild chunk: X Y^T after all of E)
//   AP A -> fp32 scratch, P -> record (fp16)
//   T  (I + A)^{-1}: 16x16 diagonal blocks by substitution, off-diagonal blocks
//      from N = D A_off as T = (I - N + N^2 - N^3) D, fp32 on CUDA cores
//   W  T' = T Diag(beta) -> record;  W^T = (K e^G)^T T'^T  (UMMA tf32) -> record
// Each warp writes its record parts as contiguous 1 KB runs (the block layout
// of chunk_common.cuh); the chain kernel's tensor loads apply the operand swizzle.
#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "chunk_common.cuh"
#include "chunk_params.cuh"
#include "kda_device.cuh"

namespace kda {

constexpr int PREP_THREADS = 512;

template <int DK>
struct PrepLayout {
    static_assert(DK == 64 || DK == 128, "dk");
    // R_form: formation operands (E..F), then A, T scratch, T, the N/M scratch
    static constexpr int OFF_F = 0;
    static constexpr int OFF_XCH = OFF_F;                    // block products exchange (E only)
    static constexpr int OFF_X = OFF_F;                      // MN-major bf16 [DK][128]
    // [Y^(0) | Y^(1) | Y^(2) | Y^(3)]: MN-major bf16 [DK][160], 64B swizzle (32-column
    // blocks); Y^(I) starts at column yoff(I), so one 160-wide product forms all four
    static constexpr int OFF_Y = OFF_X + DK * 256;
    static constexpr int FORM_B = DK * (256 + 320);
    static constexpr int OFF_A = OFF_F;                      // fp32 [64][A_LD]
    static constexpr int OFF_TF = OFF_A + 64 * A_LD * 4;     // fp32 [64][A_LD]
    static constexpr int OFF_T = OFF_F + align1k(2 * 64 * A_LD * 4);  // tf32 K-major [64][64], 8 KB K-blocks
    static constexpr int OFF_ZS = OFF_T + 16384;             // N / M scratch, 7 x 1 KB
    static constexpr int POST_B = OFF_ZS + 7 * 1024 - OFF_F;
    static constexpr int RF_B = align1k(cmax(FORM_B, POST_B));
    // (K e^G)^T: tf32 K-major [128][64]; holds the q, k TMA tiles during E
    static constexpr int OFF_BK = OFF_F + RF_B;
    static constexpr int OFF_QIN = OFF_BK;                   // bf16 [64][DK], 128B swizzle
    static constexpr int OFF_KIN = OFF_BK + CH * DK * 2;
    static constexpr int OFF_MISC = OFF_BK + 128 * 64 * 4;   // beta, barriers, TMEM address
    // g (per key channel) by TMA during the inputs: fp32 [64 tokens][DK channels], after
    // the block-products exchange in R_form (free until phase E writes X)
    static constexpr int OFF_GIN = OFF_F + 4096;
    static_assert(OFF_GIN + CH * DK * 4 <= OFF_F + RF_B, "g tile fits in R_form");
    static constexpr int TOTAL = OFF_MISC + 1024;
    static constexpr int SMEM_BYTES = TOTAL + 1024;          // slack for the 1 KB base alignment
    static_assert(SMEM_BYTES <= 113 * 1024, "two CTAs per SM");
    static_assert(POST_B <= RF_B && FORM_B <= RF_B, "R_form");

    static constexpr uint32_t TM_AP = 0;    // 160: formation products D^(I)
    static constexpr uint32_t TM_W = 160;   // 64: W^T (lane = key channel, column = token)
    static constexpr uint32_t TM_COLS = 256;
};

__device__ __forceinline__ void prefetch_tensor_4d(const CUtensorMap *map, int c0, int c1, int c2, int c3) {
    asm volatile("cp.async.bulk.prefetch.tensor.4d.L2.global.tile [%0, {%1, %2, %3, %4}];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(c0), "r"(c1), "r"(c2), "r"(c3)
                 : "memory");
}

// Prefetch the 128-byte line holding `p` into L2.
__device__ __forceinline__ void prefetch_line_l2(const void *p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<uint64_t>(p)) : "memory");
}

// SG: scalar gate, g [B, T, H] (else g [B, T, H, DK]).  PRO: the gate prologue --
// g, beta, q and k are raw projections: g = -c softplus(g_raw), beta =
// sigmoid(beta_raw), and q, k are L2-normalised per token (the norms come from
// the staged tiles; the normalised values are rounded to bf16 again, as an
// unfused caller would store them).  PACKED: the packed-batch geometry (see
// SeqGeom), else uniform.
template <int DK, bool SG, bool PRO, bool PACKED>
__global__ void __launch_bounds__(PREP_THREADS, 2)
prep_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
            const __grid_constant__ CUtensorMap tm_g, const PrepParams prm) {
    using L = PrepLayout<DK>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(sm);

    float *s_beta = reinterpret_cast<float *>(sm + L::OFF_MISC);        // [64]
    float *s_xch = reinterpret_cast<float *>(sm + L::OFF_XCH);          // [2][4][128]
    uint64_t *s_bars = reinterpret_cast<uint64_t *>(sm + L::OFF_MISC + 768);
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(sm + L::OFF_MISC + 800);
    int *s_next = reinterpret_cast<int *>(sm + L::OFF_MISC + 808);  // the item claimed next
    const uint32_t bar_in = smem_u32(&s_bars[0]);
    const uint32_t bar_mma = smem_u32(&s_bars[1]);

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int ch = tid & 127;        // key channel / TMEM lane of this thread
    const int qb = tid >> 7;         // 16-token block (phase E) / 16-column quarter (elsewhere)
    const int H = prm.H;
    const int nitems = geom_items<PACKED>(prm.gm, H);
    const uint64_t polls = prm.st.wait_polls;

    if (tid == 0) {
        stamp_start(prm.stamp);
        mbar_init(bar_in, 1);
        mbar_init(bar_mma, 1);
        fence_mbar_init();
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        if (!SG) prefetch_tmap(&tm_g);
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(s_tmem), L::TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;

    bool tma_pending = false, mma_pending = false, aborted = false;
    uint32_t ph_in = 0;   // phase of bar_in the TMA in flight completes
    uint32_t ph_mma = 0;  // phase of bar_mma the MMAs in flight complete
    auto wait_all = [&](uint32_t bar, uint32_t ph, bool &pending) -> bool {
        const bool ok = mbar_wait(bar, ph, polls, prm.st);
        if (__syncthreads_or(!ok)) return false;
        pending = false;
        tc_fence_after();
        return true;
    };
    auto sync_for_mma = [&]() {
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    };
    const int c = ch, I = qb, tb = SUB * I;
    const bool active = c < DK;

    if (tid == 0) *s_next = atomicAdd(prm.ticket, 1);
    __syncthreads();
    int claim = 0;  // thread 0: the item claimed for after this one (result needed mid-item)
    for (int item = *s_next; item < nitems && !aborted;) {
        if (tid == 0) claim = atomicAdd(prm.ticket, 1);
        const ItemGeo gi = item_geo<PACKED>(prm.gm, H, item);
        const int h = gi.h;
        uint8_t *rec = prm.ws + (size_t)gi.rec * REC_BYTES;
        // debug build: the record and the token rows this item touches
        const bool rec_in = KDA_CHECK(prm.st, gi.rec >= 0 && gi.rec < prm.nrec);
        const long long rows = geom_rows(prm.gm);
        (void)KDA_CHECK(prm.st, h < H && gi.tok0 >= 0 && gi.row0 >= 0);

        // ---------------- inputs: q, k (thread 0) and g (thread 32) by TMA; beta by plain loads.
        // Thread 0's arrival carries every byte of the phase, so the phase cannot complete
        // before it even if thread 32's load lands first (the count of pending bytes may dip
        // below zero meanwhile); a TMA issue can hold its thread for a while, hence two issuers.
        if (tid == 0) {
            mbar_expect_tx(bar_in, (uint32_t)(2 * CH * DK * 2 + (SG ? 0 : CH * DK * 4)));
#pragma unroll
            for (int kb = 0; kb < DK / 64; ++kb) {
                tma_load_4d(sbase + L::OFF_QIN + kb * CH * 128, &tm_q, bar_in, kb * 64, h, gi.tok0, gi.bcoord);
                tma_load_4d(sbase + L::OFF_KIN + kb * CH * 128, &tm_k, bar_in, kb * 64, h, gi.tok0, gi.bcoord);
            }
        }
        if (!SG && tid == 32) tma_load_4d(sbase + L::OFF_GIN, &tm_g, bar_in, 0, h, gi.tok0, gi.bcoord);
        tma_pending = true;
        float al[SUB];
        // SG: one gate per (token, head), shared by all channels: threads 64..127 stage
        // the chunk's 64 gates in shared memory (the prologue's norm slots, unused here)
        float *s_gsc = reinterpret_cast<float *>(sm + L::OFF_MISC + 256);
        if (SG && tid >= CH && tid < 2 * CH) {
            const int t = tid - CH;
            s_gsc[t] = (t < gi.nvalid && KDA_CHECK(prm.st, gi.row0 + t < rows))
                           ? __ldg(prm.g + (size_t)(gi.row0 + t) * H + h) : 0.f;
        }
        if (tid < CH) {
            const float braw = (tid < gi.nvalid && KDA_CHECK(prm.st, gi.row0 + tid < rows))
                                   ? prm.beta[(size_t)(gi.row0 + tid) * H + h] : 0.f;
            s_beta[tid] = (PRO && tid < gi.nvalid) ? gate_sigmoid(braw) : braw;
        }
        if (!wait_all(bar_in, ph_in, tma_pending)) { aborted = true; break; }
        ph_in ^= 1u;
        if constexpr (!SG) {  // one gate per key channel, from the g tile (TMA; zero past the tensor)
            const float *gs = reinterpret_cast<const float *>(sm + L::OFF_GIN) + tb * DK + c;
#pragma unroll
            for (int u = 0; u < SUB; ++u) al[u] = (tb + u < gi.nvalid && active) ? gs[u * DK] : 0.f;
        } else {
#pragma unroll
            for (int u = 0; u < SUB; ++u) al[u] = (tb + u < gi.nvalid && active) ? s_gsc[tb + u] : 0.f;
        }
        float *s_rn = reinterpret_cast<float *>(sm + L::OFF_MISC + 256);  // PRO: 1 / |q_t|, then 1 / |k_t|
        if constexpr (PRO) {
#pragma unroll
            for (int u = 0; u < SUB; ++u) al[u] = (tb + u < gi.nvalid && active) ? gate_logdecay(al[u], prm.gate_c) : 0.f;
            // 1 / |row| of the 128 rows of [q; k]: warp w takes rows 8 w .. 8 w + 7, each row
            // on DK / 8 lanes that load one 16-byte chunk (8 values) apiece; the tile's
            // swizzle only permutes the chunks of a 128-byte row, which a sum ignores
            constexpr int CPR = DK / 8, RPI = 32 / CPR;  // chunks per row, rows per pass
            const int sub = lane / CPR, chunk = lane % CPR;
#pragma unroll
            for (int it = 0; it < 8 / RPI; ++it) {
                const int row = warp * 8 + it * RPI + sub;
                const uint8_t *tile = sm + (row < CH ? L::OFF_QIN : L::OFF_KIN);
                const uint4 w = *reinterpret_cast<const uint4 *>(tile + (chunk >> 3) * CH * 128 +
                                                                 (row & (CH - 1)) * 128 + (chunk & 7) * 16);
                const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
                float ss = 0.f;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float lo = __uint_as_float(wv[j] << 16), hi = __uint_as_float(wv[j] & 0xFFFF0000u);
                    ss += lo * lo;
                    ss += hi * hi;
                }
#pragma unroll
                for (int o = CPR / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
                if (chunk == 0) s_rn[row] = rsqrtf(fmaxf(ss, 1e-24f));
            }
            __syncthreads();
        }

        // ---------------- E: decay factors and operand tiles ----------------
        // This thread's 16 key and query values, kept as bf16 pairs (tokens 2e, 2e + 1).
        uint32_t kp[SUB / 2], qp[SUB / 2];
        {
            const uint8_t *qs = sm + L::OFF_QIN, *ks = sm + L::OFF_KIN;
#pragma unroll
            for (int e = 0; e < SUB / 2; ++e) {
                uint32_t k0 = *reinterpret_cast<const uint16_t *>(ks + kmaj<128, 2>(tb + 2 * e, c, CH));
                uint32_t k1 = *reinterpret_cast<const uint16_t *>(ks + kmaj<128, 2>(tb + 2 * e + 1, c, CH));
                uint32_t q0 = *reinterpret_cast<const uint16_t *>(qs + kmaj<128, 2>(tb + 2 * e, c, CH));
                uint32_t q1 = *reinterpret_cast<const uint16_t *>(qs + kmaj<128, 2>(tb + 2 * e + 1, c, CH));
                if constexpr (PRO) {  // normalised, rounded to bf16 again, two at a time
                    const int t = tb + 2 * e;
                    const float2 nk = *reinterpret_cast<const float2 *>(s_rn + CH + t);
                    const float2 nq = *reinterpret_cast<const float2 *>(s_rn + t);
                    kp[e] = pack_bf16x2(bf16_bits_to_f32((uint16_t)k0) * nk.x, bf16_bits_to_f32((uint16_t)k1) * nk.y);
                    qp[e] = pack_bf16x2(bf16_bits_to_f32((uint16_t)q0) * nq.x, bf16_bits_to_f32((uint16_t)q1) * nq.y);
                } else {
                    kp[e] = k0 | (k1 << 16);
                    qp[e] = q0 | (q1 << 16);
                }
            }
        }
        auto unpack = [](const uint32_t (&pr)[SUB / 2], int u) {
            return __uint_as_float((u & 1) ? (pr[u >> 1] & 0xFFFF0000u) : (pr[u >> 1] << 16));
        };
        auto kval = [&](int u) { return unpack(kp, u); };
        auto qval = [&](int u) { return unpack(qp, u); };
#pragma unroll
        for (int u = 0; u < SUB; ++u) al[u] = __expf(al[u]);
        {
            float p = 1.f, p8 = 1.f;
#pragma unroll
            for (int u = 0; u < SUB; ++u) { p *= al[u]; if (u == SUB / 2) p8 = p; }
            if (active) { s_xch[I * 128 + c] = p; s_xch[512 + I * 128 + c] = p8; }
        }
        __syncthreads();  // also: every thread holds its q, k values, so their tiles' space is free
        // From the block totals bt_J and the products l8_J through each block's
        // reference token: preB = prod_{J<I} bt_J, postB = prod_{J>I} bt_J, and
        // sc[I'] = prod_{J=I+1..I'-1} bt_J * l8_{I'} for the later blocks I' > I.
        float preB = 1.f, postB = 1.f, dec = 1.f, sc[NSUB];
        {
            float mid = 1.f;
#pragma unroll
            for (int J = 0; J < NSUB; ++J) {
                const float btJ = s_xch[J * 128 + c], l8J = s_xch[512 + J * 128 + c];
                sc[J] = mid * l8J;
                if (J > I) mid *= btJ;
                if (J < I) preB *= btJ;
                if (J > I) postB *= btJ;
                dec *= btJ;
            }
        }
        // Mild chunk: no key channel loses more than 40 of log-decay over the chunk.  Then
        // the chunk's own start is a usable reference for every token (factors e^{Gamma_t}
        // and e^{-Gamma_t} within [e^-40, e^40]): X = [K e^G; Q e^G], Y = K e^{-G}, one
        // 64-column formation product.  Otherwise the 16-token block references below.
        const bool mild = __syncthreads_and(!active || dec >= MILD_DEC_LO) && !prm.block_refs;  // X's area is free

        auto yput4 = [&](int Iy, int j0, uint4 w) {
            const uint32_t off = mnmaj<64, 2>(c, yoff(Iy) + j0, DK);
            if (KDA_CHECK(prm.st, off + 16 <= (uint32_t)(DK * 320)))
                *reinterpret_cast<uint4 *>(sm + L::OFF_Y + off) = w;
        };
        auto xput4 = [&](int col, uint4 w) {
            const uint32_t off = mnmaj<128, 2>(c, col, DK);
            if (KDA_CHECK(prm.st, off + 16 <= (uint32_t)(DK * 256)))
                *reinterpret_cast<uint4 *>(sm + L::OFF_X + off) = w;
        };
        auto yput = [&](int Iy, int j0, const float (&v8)[8]) { yput4(Iy, j0, pack8_bf16(v8)); };
        auto xput = [&](int col, const float (&v8)[8]) { xput4(col, pack8_bf16(v8)); };
        bool steep = false;  // a split factor of this thread's block would pass e^80
        if (active && mild) {
            // One pass over this thread's 16 tokens.  From the last token down, r =
            // e^{Gamma_C - Gamma_t}: K-hat (record) and Y = K-hat / e^{Gamma_C} = K e^{-G}.
            // From the first token up, p = e^{Gamma_t}: Q e^G (record, and the query rows
            // of X), K e^G (the key rows of X, and (K e^G)^T).  Values are packed in pairs
            // as they are formed.
            if (I == 0 && rec_in && KDA_CHECK(prm.st, REC_DEC + 4 * c + 4 <= REC_BYTES))
                reinterpret_cast<float *>(rec + REC_DEC)[c] = dec;
            const float inv_dec = __fdividef(1.0f, dec);
            {
                uint16_t *khr = reinterpret_cast<uint16_t *>(rec + REC_KH) + (I * 128 + c) * SUB;
                const bool kh_in = rec_in && KDA_CHECK(prm.st, ((I * 128 + c) * SUB + 16) * 2 <= REC_T - REC_KH);
                float r = postB;
#pragma unroll
                for (int hh = 1; hh >= 0; --hh) {
                    uint32_t hk[4], yk[4];
#pragma unroll
                    for (int e = 7; e >= 1; e -= 2) {  // tokens e - 1, e of the half
                        const float hi = kval(hh * 8 + e) * r;
                        r *= al[hh * 8 + e];
                        const float lo = kval(hh * 8 + e - 1) * r;
                        r *= al[hh * 8 + e - 1];
                        hk[e / 2] = pack_f16x2(lo, hi);
                        yk[e / 2] = pack_bf16x2(lo * inv_dec, hi * inv_dec);
                    }
                    if (kh_in) *reinterpret_cast<uint4 *>(khr + hh * 8) = make_uint4(hk[0], hk[1], hk[2], hk[3]);
                    yput4(0, tb + hh * 8, make_uint4(yk[0], yk[1], yk[2], yk[3]));
                }
            }
            {
                uint16_t *qer = reinterpret_cast<uint16_t *>(rec + REC_WQ) + ((NSUB + I) * DK + c) * SUB;
                const bool qe_in = rec_in && KDA_CHECK(prm.st, (((NSUB + I) * DK + c) * SUB + 16) * 2 <= REC_P - REC_WQ);
                float p = preB;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    uint32_t qk[4], xk[4];
#pragma unroll
                    for (int e4 = 0; e4 < 2; ++e4) {
                        float b[4];
#pragma unroll
                        for (int ep = 0; ep < 2; ++ep) {
                            const int u = hh * 8 + e4 * 4 + 2 * ep;
                            p *= al[u];
                            const float q0 = qval(u) * p, k0 = kval(u) * p;
                            p *= al[u + 1];
                            const float q1 = qval(u + 1) * p, k1 = kval(u + 1) * p;
                            qk[e4 * 2 + ep] = pack_bf16x2(q0, q1);
                            xk[e4 * 2 + ep] = pack_bf16x2(k0, k1);
                            b[2 * ep] = k0;
                            b[2 * ep + 1] = k1;
                        }
                        const uint32_t o = kmaj<128, 4>(c, tb + hh * 8 + e4 * 4, 128);
                        if (KDA_CHECK(prm.st, o + 16 <= 128 * 64 * 4))
                            *reinterpret_cast<uint4 *>(sm + L::OFF_BK + o) = pack4_tf32(b[0], b[1], b[2], b[3]);
                    }
                    const uint4 qw = make_uint4(qk[0], qk[1], qk[2], qk[3]);
                    if (qe_in) *reinterpret_cast<uint4 *>(qer + hh * 8) = qw;
                    xput4(tb + hh * 8, make_uint4(xk[0], xk[1], xk[2], xk[3]));
                    xput4(CH + tb + hh * 8, qw);
                }
            }
        } else if (active) {
            // Own block, reference m = tb + 8:
            //   u >= 8: f_u = prod_{s=9..u} alpha     X = k f,   Y^(I) = k / f
            //   u <  8: y_u = prod_{s=u+1..8} alpha   X = k / y, Y^(I) = k y
            {
                float f[8], v8[8];
                float ff = 1.f;
#pragma unroll
                for (int e = 0; e < 8; ++e) { if (e > 0) ff *= al[8 + e]; f[e] = ff; }
                steep = f[7] < EXP_CLAMP_LO;  // prod of alpha over tokens 9..15, the smallest f
#pragma unroll
                for (int e = 0; e < 8; ++e) v8[e] = kval(8 + e) * f[e];
                xput(tb + 8, v8);
#pragma unroll
                for (int e = 0; e < 8; ++e) v8[e] = qval(8 + e) * f[e];
                xput(64 + tb + 8, v8);
#pragma unroll
                for (int e = 0; e < 8; ++e) v8[e] = e == 0 ? kval(8) : kval(8 + e) * rcp_clamped(f[e]);
                yput(I, tb + 8, v8);
            }
            {
                float y[8], v8[8];
                float yy = 1.f;
#pragma unroll
                for (int e = 7; e >= 0; --e) { yy *= al[e + 1]; y[e] = yy; }
                steep = steep || y[0] < EXP_CLAMP_LO;  // prod over tokens 1..8, the smallest y
#pragma unroll
                for (int e = 0; e < 8; ++e) v8[e] = kval(e) * y[e];
                yput(I, tb, v8);
#pragma unroll
                for (int e = 0; e < 8; ++e) y[e] = rcp_clamped(y[e]);
#pragma unroll
                for (int e = 0; e < 8; ++e) v8[e] = kval(e) * y[e];
                xput(tb, v8);
#pragma unroll
                for (int e = 0; e < 8; ++e) v8[e] = qval(e) * y[e];
                xput(64 + tb, v8);
            }
            // Later blocks I' > I see this block through e^{Gamma_{m'} - Gamma_j}
            //   = ls_u * prod_{J = I+1 .. I'-1} bt_J * l8_{I'},  ls_u = prod_{s=u+1..15} alpha_s
            // (all factors <= 1).  Half by half, from the top token down.
#pragma unroll
            for (int hh = 1; hh >= 0; --hh) {
                float ls[8];
                float r = 1.f;
                if (hh == 0) {
#pragma unroll
                    for (int s = 8; s < SUB; ++s) r *= al[s];
                }
#pragma unroll
                for (int e = 7; e >= 0; --e) { ls[e] = r; r *= al[hh * 8 + e]; }
                float kk[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) kk[e] = kval(hh * 8 + e) * ls[e];
#pragma unroll
                for (int Ip = 1; Ip < NSUB; ++Ip) {
                    if (Ip > I) {
                        float v8[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) v8[e] = kk[e] * sc[Ip];
                        yput(Ip, tb + hh * 8, v8);
                    }
                }
            }
        }
        fence_async_smem();
        tc_fence_before();
        const bool exact_item = __syncthreads_or(steep) || prm.force_exact;
        tc_fence_after();
        if (exact_item && tid == 0) {
            const int pos = atomicAdd(prm.steep_count, 1);
            if (KDA_CHECK(prm.st, pos < nitems)) prm.steep_items[pos] = item;
        }

        // ---------------- F: formation products (bf16), overlapped with the rest of E ----------------
        // Block references: X [Y^(0) | .. | Y^(3)]^T, 128 x 160, column block I' = D^(I').
        // Mild chunk: X Y^T, 128 x 64 (E is complete).
        if (tid == 0) {
            const uint32_t idesc = make_idesc(1, true, true, 128, mild ? CH : yoff(NSUB));
#pragma unroll
            for (int kk = 0; kk < DK / 16; ++kk)
                umma<0>(tmem + L::TM_AP, desc_mnmaj<128>(sbase + L::OFF_X, DK, kk * 16),
                        desc_mnmaj<64>(sbase + L::OFF_Y, DK, kk * 16), idesc, kk > 0);
            umma_commit(bar_mma);
        }
        mma_pending = true;

        // e^{Gamma_C - Gamma_t}: K-hat^T (record);  e^{Gamma_t}: Q e^G (record) and (K e^G)^T (smem)
        if (active && !mild) {
            if (I == 0 && rec_in && KDA_CHECK(prm.st, REC_DEC + 4 * c + 4 <= REC_BYTES))
                reinterpret_cast<float *>(rec + REC_DEC)[c] = dec;
            uint16_t *khr = reinterpret_cast<uint16_t *>(rec + REC_KH) + (I * 128 + c) * SUB;
            const bool kh_in = rec_in && KDA_CHECK(prm.st, ((I * 128 + c) * SUB + 16) * 2 <= REC_T - REC_KH);
            float r = postB;
#pragma unroll
            for (int hh = 1; hh >= 0; --hh) {
                float kh[8];
#pragma unroll
                for (int e = 7; e >= 0; --e) { kh[e] = kval(hh * 8 + e) * r; r *= al[hh * 8 + e]; }
                if (kh_in) *reinterpret_cast<uint4 *>(khr + hh * 8) = pack8_f16(kh);
            }
            uint16_t *qer = reinterpret_cast<uint16_t *>(rec + REC_WQ) + ((NSUB + I) * DK + c) * SUB;
            const bool qe_in = rec_in && KDA_CHECK(prm.st, (((NSUB + I) * DK + c) * SUB + 16) * 2 <= REC_P - REC_WQ);
            float p = preB;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                float qe[8], bk[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    p *= al[hh * 8 + e];
                    qe[e] = qval(hh * 8 + e) * p;
                    bk[e] = kval(hh * 8 + e) * p;
                }
                if (qe_in) *reinterpret_cast<uint4 *>(qer + hh * 8) = pack8_bf16(qe);
                const uint32_t o0 = kmaj<128, 4>(c, tb + hh * 8, 128), o1 = kmaj<128, 4>(c, tb + hh * 8 + 4, 128);
                if (KDA_CHECK(prm.st, o0 + 16 <= 128 * 64 * 4 && o1 + 16 <= 128 * 64 * 4)) {
                    *reinterpret_cast<uint4 *>(sm + L::OFF_BK + o0) = pack4_tf32(bk[0], bk[1], bk[2], bk[3]);
                    *reinterpret_cast<uint4 *>(sm + L::OFF_BK + o1) = pack4_tf32(bk[4], bk[5], bk[6], bk[7]);
                }
            }
        }
        if (tid == 0) *s_next = claim;  // read by every thread after the barrier below
        if (!wait_all(bar_mma, ph_mma, mma_pending)) { aborted = true; break; }
        ph_mma ^= 1u;
        const int next = *s_next;
        // the next item's q, k and g into L2 while this one finishes
        if (next < nitems) {
            const ItemGeo ng = item_geo<PACKED>(prm.gm, H, next);
            if (tid == 0) {
#pragma unroll
                for (int kb = 0; kb < DK / 64; ++kb) {
                    prefetch_tensor_4d(&tm_q, kb * 64, ng.h, ng.tok0, ng.bcoord);
                    prefetch_tensor_4d(&tm_k, kb * 64, ng.h, ng.tok0, ng.bcoord);
                }
            } else if (!SG && tid == 32) {
                prefetch_tensor_4d(&tm_g, 0, ng.h, ng.tok0, ng.bcoord);
            } else if (SG && tid >= 64 && tid < 64 + CH && tid - 64 < ng.nvalid) {
                prefetch_line_l2(prm.g + (size_t)(ng.row0 + tid - 64) * H + ng.h);
            }
        }

        // ---------------- AP: A -> fp32 scratch, P -> record ----------------
        // TMEM lane = row of [k; q]; the four warps of a lane quarter take one
        // 16-column chunk each (chunk = qb).
        {
            float *sA = reinterpret_cast<float *>(sm + L::OFF_A);
            const int i = ch & 63;
            const int myI = i / SUB;
            const bool is_q = ch >= 64;
            const float bi = s_beta[i];
            const int I0 = ((warp & 1) * 32) / SUB;  // the lane quarter covers blocks I0, I0 + 1
            const int cc = qb;
            float v16[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) v16[e] = 0.f;
            if (mild) {  // column j of the product is token j
                if (cc <= I0 + 1) {  // warp-uniform: some row of the quarter reaches this chunk
                    tmem_ld16(tmem + lane_base + L::TM_AP + cc * 16, v16);
                    tmem_wait_ld();
                }
            } else {
#pragma unroll
                for (int dI = 0; dI < 2; ++dI) {
                    const int Ib = I0 + dI;
                    if (cc <= Ib) {  // warp-uniform
                        float t[16];
                        tmem_ld16(tmem + lane_base + L::TM_AP + yoff(Ib) + cc * 16, t);
                        tmem_wait_ld();
                        if (myI == Ib) {
#pragma unroll
                            for (int e = 0; e < 16; ++e) v16[e] = t[e];
                        }
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
                uint16_t *pr = reinterpret_cast<uint16_t *>(rec + REC_P) + (cc * CH + i) * SUB;
                const bool p_in = rec_in && KDA_CHECK(prm.st, ((cc * CH + i) * SUB + 16) * 2 <= REC_KH - REC_P);
#pragma unroll
                for (int e8 = 0; e8 < 16; e8 += 8) {
                    float p8[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) p8[e] = (j0 + e8 + e <= i) ? v16[e8 + e] : 0.f;
                    if (p_in) *reinterpret_cast<uint4 *>(pr + e8) = pack8_f16(p8);
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
                const int Ib = tid >> 4, jj = tid & 15, base = SUB * Ib;
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
            // Off-diagonal blocks.  With D = diag(T_II) and N = D A_offdiag (strictly block
            // lower, N^4 = 0):  T = (I - N + N^2 - N^3) D, i.e. T_IJ = M_IJ T_JJ with
            //   M_{I,I-1} = -N_{I,I-1},  M_20 = -N_20 + N_21 N_10,  M_31 = -N_31 + N_32 N_21,
            //   M_30 = -N_30 + N_31 N_10 - N_32 M_20.
            // Scratch slots (16x16, row stride 16): 0 N10, 1 N20, 2 N21, 3 N30, 4 N31, 5 N32, 6 M31.
            // One warp per 16x16 product; lane (r = lane / 2, c0 = 8 (lane % 2)) owns 8 outputs.
            {
                const int r = lane >> 1, c0 = (lane & 1) * 8;
                auto rowblk = [&](const float *arow, const float *bblk, int bld, float (&o)[8]) {
#pragma unroll
                    for (int m4 = 0; m4 < SUB; m4 += 4) {
                        const float4 a4 = *reinterpret_cast<const float4 *>(arow + m4);
                        const float av[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
                        for (int mm = 0; mm < 4; ++mm) {
                            const float *brow = bblk + (m4 + mm) * bld + c0;
                            const float4 b0 = *reinterpret_cast<const float4 *>(brow);
                            const float4 b1 = *reinterpret_cast<const float4 *>(brow + 4);
                            o[0] += av[mm] * b0.x; o[1] += av[mm] * b0.y; o[2] += av[mm] * b0.z; o[3] += av[mm] * b0.w;
                            o[4] += av[mm] * b1.x; o[5] += av[mm] * b1.y; o[6] += av[mm] * b1.z; o[7] += av[mm] * b1.w;
                        }
                    }
                };
                auto store8 = [&](float *dst, const float (&o)[8], float sgn) {
                    *reinterpret_cast<float4 *>(dst) = make_float4(sgn * o[0], sgn * o[1], sgn * o[2], sgn * o[3]);
                    *reinterpret_cast<float4 *>(dst + 4) = make_float4(sgn * o[4], sgn * o[5], sgn * o[6], sgn * o[7]);
                };
                const int BI = warp == 0 ? 1 : (warp < 3 ? 2 : 3);            // block pair of warp < 6:
                const int BJ = warp == 0 ? 0 : (warp < 3 ? warp - 1 : warp - 3);  // (1,0) (2,0) (2,1) (3,0) (3,1) (3,2)
                if (warp < 6) {  // N_IJ = T_II A_IJ
                    float o[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                    rowblk(sTf + (SUB * BI + r) * A_LD + SUB * BI, sA + (SUB * BI) * A_LD + SUB * BJ, A_LD, o);
                    store8(sZ + warp * 256 + r * 16 + c0, o, 1.f);
                }
                __syncthreads();
                if (warp < 2) {  // M20 = -N20 + N21 N10 (slot 1);  M31 = -N31 + N32 N21 (slot 6)
                    const int so = warp == 0 ? 1 : 4, sa = warp == 0 ? 2 : 5, sb = warp == 0 ? 0 : 2;
                    float o[8];
                    const float *own = sZ + so * 256 + r * 16 + c0;
#pragma unroll
                    for (int e = 0; e < 8; ++e) o[e] = -own[e];
                    rowblk(sZ + sa * 256 + r * 16, sZ + sb * 256, 16, o);
                    store8(sZ + (warp == 0 ? 1 : 6) * 256 + r * 16 + c0, o, 1.f);
                }
                __syncthreads();
                if (warp == 0) {  // M30 = -N30 + N31 N10 - N32 M20 (slot 3)
                    float o[8], o2[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                    const float *own = sZ + 3 * 256 + r * 16 + c0;
#pragma unroll
                    for (int e = 0; e < 8; ++e) o[e] = -own[e];
                    rowblk(sZ + 4 * 256 + r * 16, sZ + 0 * 256, 16, o);
                    rowblk(sZ + 5 * 256 + r * 16, sZ + 1 * 256, 16, o2);
#pragma unroll
                    for (int e = 0; e < 8; ++e) o[e] -= o2[e];
                    store8(sZ + 3 * 256 + r * 16 + c0, o, 1.f);
                }
                __syncthreads();
                if (warp < 6) {  // T_IJ = M_IJ T_JJ; adjacent blocks carry M = -N
                    const int msl = warp == 4 ? 6 : warp;
                    const float sgn = (warp == 0 || warp == 2 || warp == 5) ? -1.f : 1.f;
                    float o[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                    rowblk(sZ + msl * 256 + r * 16, sTf + (SUB * BJ) * A_LD + SUB * BJ, A_LD, o);
                    store8(sTf + (SUB * BI + r) * A_LD + SUB * BJ + c0, o, sgn);
                }
                __syncthreads();
            }
            // T' = T Diag(beta) -> tf32 K-major tile (smem operand of W) and the record,
            // zeros above the diagonal
            for (int e = tid; e < 64 * 16; e += PREP_THREADS) {
                const int i = e >> 4, j = (e & 15) * 4;
                const float *src = sTf + i * A_LD + j;
                const float4 bj = *reinterpret_cast<const float4 *>(s_beta + j);
                const float4 w = make_float4(j + 0 <= i ? src[0] * bj.x : 0.f, j + 1 <= i ? src[1] * bj.y : 0.f,
                                             j + 2 <= i ? src[2] * bj.z : 0.f, j + 3 <= i ? src[3] * bj.w : 0.f);
                const uint32_t ot = kmaj_s<128, 4>(i, j, 8192);
                if (KDA_CHECK(prm.st, ot + 16 <= 16384))
                    *reinterpret_cast<uint4 *>(sm + L::OFF_T + ot) = pack4_tf32(w.x, w.y, w.z, w.w);
                if (rec_in && KDA_CHECK(prm.st, (i * CH + j) * 4 + 16 <= REC_DEC - REC_T))
                    *reinterpret_cast<float4 *>(rec + REC_T + (i * CH + j) * 4) = w;
            }
        }
        sync_for_mma();

        // ---------------- W: W^T = (K e^G)^T T'^T  (tf32) ----------------
        if (tid == 0) {
            const uint32_t id_w = make_idesc(2, false, false, 128, 64);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                umma<1>(tmem + L::TM_W, desc_kmaj_s<128, 4>(sbase + L::OFF_BK, 128 * 128, kk * 8),
                        desc_kmaj_s<128, 4>(sbase + L::OFF_T, 8192, kk * 8), id_w, kk > 0);
            umma_commit(bar_mma);
        }
        mma_pending = true;
        if (!wait_all(bar_mma, ph_mma, mma_pending)) { aborted = true; break; }
        ph_mma ^= 1u;
        if ((warp & 3) < DK / 32) {  // W^T row ch, tokens 16 qb .. -> WQ block qb
            const int i0 = qb * 16;
            float t[16];
            tmem_ld16(tmem + lane_base + L::TM_W + i0, t);
            tmem_wait_ld();
            float a8[8], b8[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) { a8[e] = t[e]; b8[e] = t[8 + e]; }
            uint16_t *wr = reinterpret_cast<uint16_t *>(rec + REC_WQ) + (qb * DK + ch) * SUB;
            if (rec_in && KDA_CHECK(prm.st, ((qb * DK + ch) * SUB + 16) * 2 <= NSUB * DK * SUB * 2)) {
                *reinterpret_cast<uint4 *>(wr) = pack8_bf16(a8);
                *reinterpret_cast<uint4 *>(wr + 8) = pack8_bf16(b8);
            }
        }
        // This item's shared memory and TMEM are free for the next one.  No tcgen05
        // fences: the W rows' TMEM loads completed (wait::ld), and the next tcgen05
        // operation (the formation product) follows its own fenced barrier.
        __syncthreads();
        item = next;
    }

    if (aborted && tid == 0) {
        // Leave nothing in flight that targets this CTA's smem or TMEM.
        if (tma_pending) mbar_wait(bar_in, ph_in, ~0ull, prm.st);
        if (mma_pending) mbar_wait(bar_mma, ph_mma, ~0ull, prm.st);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, L::TM_COLS);
    if (tid == 0) stamp_end(prm.stamp);
}

template <int DK, bool SG, bool PRO, bool PACKED = false>
static cudaError_t launch_prep_t(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tg,
                                 const PrepParams &prm, int max_ctas, cudaStream_t stream) {
    using L = PrepLayout<DK>;
    cudaError_t e = cudaFuncSetAttribute(prep_kernel<DK, SG, PRO, PACKED>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         L::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    // items of the launch (packed: an upper bound, the kernel reads the exact count)
    const long long items = prm.gm.cu == nullptr ? (long long)prm.gm.nseqs * prm.H * prm.gm.nseg
                                                 : (long long)prm.gm.W * prm.H;
    const int grid = (int)(items < max_ctas ? items : max_ctas);
    prep_kernel<DK, SG, PRO, PACKED><<<grid, PREP_THREADS, L::SMEM_BYTES, stream>>>(tq, tk, tg, prm);
    return cudaGetLastError();
}

// At most max_ctas persistent CTAs (two fit on an SM), at most one per item;
// prm.g_dk selects the gate form (dk: per key channel, read through tg; 1:
// scalar, tg unused); `prologue` the raw-input form (per key channel only).
cudaError_t launch_prep(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tg, const PrepParams &prm,
                        int dk, int max_ctas, cudaStream_t stream, bool prologue) {
    const bool sg = prm.g_dk == 1;
    if (prm.gm.cu != nullptr) {  // packed batches: per-channel gate, inputs as given
        if (sg || prologue) return cudaErrorInvalidValue;
        return dk == 128 ? launch_prep_t<128, false, false, true>(tq, tk, tg, prm, max_ctas, stream)
                         : launch_prep_t<64, false, false, true>(tq, tk, tg, prm, max_ctas, stream);
    }
    if (prologue) {
        if (sg) return cudaErrorInvalidValue;
        return dk == 128 ? launch_prep_t<128, false, true>(tq, tk, tg, prm, max_ctas, stream)
                         : launch_prep_t<64, false, true>(tq, tk, tg, prm, max_ctas, stream);
    }
    if (dk == 128) return sg ? launch_prep_t<128, true, false>(tq, tk, tg, prm, max_ctas, stream)
                             : launch_prep_t<128, false, false>(tq, tk, tg, prm, max_ctas, stream);
    return sg ? launch_prep_t<64, true, false>(tq, tk, tg, prm, max_ctas, stream)
              : launch_prep_t<64, false, false>(tq, tk, tg, prm, max_ctas, stream);
}

}  // namespace kda
