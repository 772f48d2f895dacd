// chain_fwd.cu -- the inter-chunk (state-passing) half of the chunkwise KDA
// prefill (sm_100a).
//
// One CTA owns one (b, h, slice of 64 value columns) and walks the chunks of a
// segment in order, reading the per-chunk records of the prep kernel
// (prep_fwd.cu; layout in chunk_common.cuh).  Per chunk, S0 = state at the
// chunk start:
//   U    = T' V                      T' = T Diag(beta), V the chunk's values
//   Vnew = U - W S0                  the delta-rule corrected writes
//   O    = scale ((Q e^Gamma) S0 + P Vnew)
//   S    = Diag(e^{Gamma_C}) S0 + K-hat^T Vnew
// (state passing across chunks with the causal intra-chunk correction,
// section 4 of "Kimi Linear's Hybrid Linear Attention Architecture: A
// Technical Breakdown").  The state lives in fp32 registers (thread (c, g)
// holds row c, 16 columns); a bf16 copy in shared memory feeds the tensor
// core.  All products are 128-row UMMAs with TMEM accumulators:
//   1   D1 = [W; Q e^G] S0            bf16, A = record WQ (MN-major)
//   U   U  = T' V                      tf32, A = record T' (rows 64..127 unused)
//   3a  D3 = K-hat^T Vnew              tf32
//   3b  D1 += [.; P] Vnew              tf32, rows 64..127 = the output block
// Only 1 and 3a lie on the state's critical path.  The tensor pipe executes
// in issue order, so the other two are issued where they fill its idle time:
// for chunk n the order is 1(n), 3b(n-1), 3a(n), U(n+1) -- 3b(n-1) runs while
// the threads form Vnew(n), U(n+1) while they update the state.  That needs
// two output accumulators, two Vnew tiles and two buffers of P and of T'.
// Record parts arrive by tensor loads (which apply the operand swizzle), each
// part reloaded for a later chunk as soon as its last reader is done; the
// values V are read with plain coalesced loads one chunk ahead.
#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "chunk_common.cuh"
#include "chunk_params.cuh"
#include "kda_device.cuh"

namespace kda {

constexpr int CHAIN_THREADS = 512;
constexpr int CHAIN_VS = 64;       // value columns per CTA
constexpr int CHAIN_PREFETCH = 4;  // chunks between the L2 prefetch of a record and its use

template <int DK>
struct ChainLayout {
    static_assert(DK == 64 || DK == 128, "dk");
    static constexpr int VS = CHAIN_VS;
    static constexpr int OFF_WQ = 0;          // bf16 MN-major [DK][128]: [W; Q e^G]
    static constexpr int OFF_P = 32768;       // two tf32 K-major [64][64] buffers (8 KB K-blocks)
    static constexpr int OFF_KH = 65536;      // tf32 K-major [128][64] (16 KB K-blocks)
    static constexpr int OFF_T = 98304;       // two tf32 K-major [64][64] buffers (8 KB K-blocks)
    static constexpr int OFF_DEC = 131072;    // two 512-byte slots of e^{Gamma_C}
    static constexpr int OFF_S0 = 132096;     // bf16 MN-major S0 [DK][64], 128B swizzle
    static constexpr int OFF_VT = align1k(OFF_S0 + DK * VS * 2);  // tf32 K-major V^T [64][64]
    static constexpr int OFF_VN = OFF_VT + VS * 256;              // two tf32 K-major Vnew^T [64][64]
    static constexpr int OFF_MISC = OFF_VN + 2 * VS * 256;        // barriers, TMEM address
    static constexpr int TOTAL = OFF_MISC + 1024;
    static constexpr int SMEM_BYTES = TOTAL + 1024;  // slack for the 1 KB base alignment
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
    // The 128-row views read 8 KB before P's buffers (rows 0..63, discarded)
    // and 8 KB past T's second buffer (rows 64..127, discarded).
    static_assert(OFF_P >= 8192 && OFF_T + 2 * 16384 + 8192 <= TOTAL, "operand views stay in bounds");

    static constexpr uint32_t TM_U = 0;          // U (lane = token)
    static constexpr uint32_t TM_D1 = VS;        // two: [W; Q e^G] S0, then += P Vnew on lanes 64..127
    static constexpr uint32_t TM_D3 = 3 * VS;    // K-hat^T Vnew (lane = key channel)
    static constexpr uint32_t TM_COLS = 256;
};

template <int DK>
__global__ void __launch_bounds__(CHAIN_THREADS, 1)
chain_kernel(const __grid_constant__ CUtensorMap tm_wq, const __grid_constant__ CUtensorMap tm_p,
             const __grid_constant__ CUtensorMap tm_kh, const __grid_constant__ CUtensorMap tm_t,
             const ChainParams prm) {
    using L = ChainLayout<DK>;
    constexpr int VS = L::VS;
    constexpr int CPT = VS / 4;            // value columns per thread (state, Vnew, output)
    constexpr int NP = VS / 2;             // value column pairs (V loads)
    constexpr int TG = CHAIN_THREADS / NP; // token groups (V loads)
    constexpr int TPT = CH / TG;           // tokens per thread (V loads)
    static_assert(TPT % 4 == 0 && CPT == 16, "thread mapping");
    constexpr uint32_t TX_T = 16384 + 512, TX_W = DK * 256, TX_P = 16384, TX_K = 32768;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(sm);
    // One mbarrier per buffer: a barrier tracks one phase at a time, so a
    // buffer's next load is issued only after its previous one was waited for.
    uint64_t *s_bars = reinterpret_cast<uint64_t *>(sm + L::OFF_MISC);
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(sm + L::OFF_MISC + 128);
    constexpr int NBARS = 10;
    const uint32_t bar_t0 = smem_u32(&s_bars[0]);  // T'(n), e^{Gamma_C}(n) arrived, n even
    const uint32_t bar_p0 = smem_u32(&s_bars[2]);  // P(n) arrived, n even (odd n: the next barrier)
    const uint32_t bar_w = smem_u32(&s_bars[4]);   // WQ(n) arrived
    const uint32_t bar_k = smem_u32(&s_bars[5]);   // K-hat(n) arrived
    const uint32_t bar_m1 = smem_u32(&s_bars[6]);  // U(n) and product 1(n) done
    const uint32_t bar_mb = smem_u32(&s_bars[7]);  // 3b(n) done
    const uint32_t bar_m3 = smem_u32(&s_bars[8]);  // 3a(n) done
    const uint32_t bar_never = smem_u32(&s_bars[9]);  // nothing arrives on it (fault-injection hook)
    auto bar_t = [&](int n) { return bar_t0 + 8u * (uint32_t)(n & 1); };
    auto bar_p = [&](int n) { return bar_p0 + 8u * (uint32_t)(n & 1); };
    auto par2 = [](int n) { return (uint32_t)((n >> 1) & 1); };  // phase parity of a two-buffer barrier

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lq = warp & 3;              // TMEM lane quarter of this warp
    const int cg = warp >> 2;             // value-column group of this warp
    const int ch = lq * 32 + (tid & 31);  // TMEM lane of this thread
    const int slice = blockIdx.x % prm.nslices;
    const int bh = blockIdx.x / prm.nslices;
    const int h = bh % prm.H, b = bh / prm.H;
    const int T = prm.T, H = prm.H, DV = prm.DV;
    const int col0 = slice * VS;
    const int nseg = prm.nseg;
    const uint8_t *recs = prm.ws + (size_t)bh * nseg * REC_BYTES;
    const int rec0 = bh * nseg;  // index of this (b, h)'s first record in the tensor maps
    const uint64_t polls = prm.st.wait_polls;

    if (tid == 0) {
        for (int i = 0; i < NBARS; ++i) mbar_init(smem_u32(&s_bars[i]), 1);
        fence_mbar_init();
        prefetch_tmap(&tm_wq); prefetch_tmap(&tm_p); prefetch_tmap(&tm_kh); prefetch_tmap(&tm_t);
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(s_tmem), L::TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const uint32_t lane_base = (uint32_t)(lq * 32) << 16;

    // ---- record loads (issued by thread 0); each barrier completes once per chunk, in order ----
    auto issue_t = [&](int n) {  // T'(n), e^{Gamma_C}(n) -> buffer n & 1
        const int s = n & 1;
        const uint32_t bar = bar_t(n);
        mbar_expect_tx(bar, TX_T);
#pragma unroll
        for (int kb = 0; kb < 2; ++kb)
            tma_load_3d(sbase + L::OFF_T + s * 16384 + kb * 8192, &tm_t, bar, kb * 32, 0, rec0 + n);
        bulk_load(sbase + L::OFF_DEC + s * 512, recs + (size_t)n * REC_BYTES + REC_DEC, 512, bar);
    };
    auto issue_w = [&](int n) {
        mbar_expect_tx(bar_w, TX_W);
#pragma unroll
        for (int nb = 0; nb < 2; ++nb)
            tma_load_3d(sbase + L::OFF_WQ + nb * DK * 128, &tm_wq, bar_w, nb * 64, 0, rec0 + n);
    };
    auto issue_p = [&](int n) {  // -> buffer n & 1
        const uint32_t bar = bar_p(n);
        mbar_expect_tx(bar, TX_P);
#pragma unroll
        for (int kb = 0; kb < 2; ++kb)
            tma_load_3d(sbase + L::OFF_P + (n & 1) * 16384 + kb * 8192, &tm_p, bar, kb * 32, 0, rec0 + n);
    };
    auto issue_k = [&](int n) {
        mbar_expect_tx(bar_k, TX_K);
#pragma unroll
        for (int kb = 0; kb < 2; ++kb)
            tma_load_3d(sbase + L::OFF_KH + kb * 16384, &tm_kh, bar_k, kb * 32, 0, rec0 + n);
    };

    // ---- products (issued by thread 0) ----
    const uint32_t id_tf = make_idesc(2, false, false, 128, VS);
    const uint32_t id_bf = make_idesc(1, true, true, 128, VS);
    auto mma_u = [&](int n) {  // U = T'(n) V(n)
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
            umma<1>(tmem + L::TM_U, desc_kmaj_s<128, 4>(sbase + L::OFF_T + (n & 1) * 16384, 8192, kk * 8),
                    desc_kmaj_s<128, 4>(sbase + L::OFF_VT, VS * 128, kk * 8), id_tf, kk > 0);
    };
    auto mma_1 = [&](int n) {  // D1[n & 1] = [W; Q e^G](n) S0
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk)
            umma<0>(tmem + L::TM_D1 + (n & 1) * VS, desc_mnmaj<128>(sbase + L::OFF_WQ, DK, kk * 16),
                    desc_mnmaj<128>(sbase + L::OFF_S0, DK, kk * 16), id_bf, kk > 0);
    };
    auto mma_3a = [&](int n) {  // D3 = K-hat(n)^T Vnew(n)
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
            umma<1>(tmem + L::TM_D3, desc_kmaj_s<128, 4>(sbase + L::OFF_KH, 128 * 128, kk * 8),
                    desc_kmaj_s<128, 4>(sbase + L::OFF_VN + (n & 1) * VS * 256, VS * 128, kk * 8), id_tf, kk > 0);
    };
    auto mma_3b = [&](int n) {  // D1[n & 1] rows 64..127 += P(n) Vnew(n)
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
            umma<1>(tmem + L::TM_D1 + (n & 1) * VS,
                    desc_kmaj_s<128, 4>(sbase + L::OFF_P + (n & 1) * 16384 - 8192, 8192, kk * 8),
                    desc_kmaj_s<128, 4>(sbase + L::OFF_VN + (n & 1) * VS * 256, VS * 128, kk * 8), id_tf, 1u);
    };

    // ---- state: thread (ch, cg) holds S[ch][cg CPT .. cg CPT + CPT - 1] in fp32 ----
    float S[CPT];
#pragma unroll
    for (int e = 0; e < CPT; ++e) S[e] = 0.f;
    const int scol = col0 + cg * CPT;
    if (ch < DK && prm.h0 != nullptr) {
        const float4 *src = reinterpret_cast<const float4 *>(prm.h0 + (((size_t)b * H + h) * DK + ch) * DV + scol);
#pragma unroll
        for (int e = 0; e < CPT / 4; ++e) {
            const float4 x = src[e];
            S[4 * e] = x.x; S[4 * e + 1] = x.y; S[4 * e + 2] = x.z; S[4 * e + 3] = x.w;
        }
    }
    auto store_state_bf16 = [&]() {
        if (ch < DK) {
#pragma unroll
            for (int e8 = 0; e8 < CPT / 8; ++e8) {
                float v8[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) v8[e] = S[e8 * 8 + e];
                *reinterpret_cast<uint4 *>(sm + L::OFF_S0 + mnmaj<128, 2>(ch, cg * CPT + e8 * 8, DK)) = pack8_bf16(v8);
            }
        }
    };

    // ---- values: thread (p, tg) loads columns 2p, 2p + 1 of tokens tg TPT .. ----
    const int vp = tid % NP, vtg = tid / NP;
    uint32_t vr[TPT];
    auto load_v = [&](int n) {
        const int t0 = (prm.n_begin + n) * CH + vtg * TPT;
        const uint32_t *src = reinterpret_cast<const uint32_t *>(prm.v + (((size_t)b * T + t0) * H + h) * DV + col0) + vp;
#pragma unroll
        for (int u = 0; u < TPT; ++u) vr[u] = (t0 + u < T) ? __ldg(src + (size_t)u * H * DV / 2) : 0u;
    };
    auto build_vt = [&]() {  // V^T tile: row = value column, K = token
        // a bf16 value is the top half of its fp32 (and tf32) bit pattern
#pragma unroll
        for (int u4 = 0; u4 < TPT / 4; ++u4) {
            const uint32_t *x = vr + u4 * 4;
            const uint4 lo = make_uint4(x[0] << 16, x[1] << 16, x[2] << 16, x[3] << 16);
            const uint4 hi = make_uint4(x[0] & 0xFFFF0000u, x[1] & 0xFFFF0000u, x[2] & 0xFFFF0000u, x[3] & 0xFFFF0000u);
            *reinterpret_cast<uint4 *>(sm + L::OFF_VT + kmaj_s<128, 4>(2 * vp, vtg * TPT + u4 * 4, VS * 128)) = lo;
            *reinterpret_cast<uint4 *>(sm + L::OFF_VT + kmaj_s<128, 4>(2 * vp + 1, vtg * TPT + u4 * 4, VS * 128)) = hi;
        }
    };
    // output rows of chunk n from D1[n & 1] (warps of lane quarters 2, 3; the
    // TMEM load is warp-collective, only the stores are guarded)
    auto write_output = [&](int n) {
        const int i = ch - 64;
        const int t = (prm.n_begin + n) * CH + i;
        float o[16];
        tmem_ld16(tmem + lane_base + L::TM_D1 + (n & 1) * VS + cg * CPT, o);
        tmem_wait_ld();
        if (t < T) {
            uint16_t *dst = prm.out + (((size_t)b * T + t) * H + h) * DV + scol;
            float a8[8], b8[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) { a8[e] = prm.scale * o[e]; b8[e] = prm.scale * o[8 + e]; }
            *reinterpret_cast<uint4 *>(dst) = pack8_bf16(a8);
            *reinterpret_cast<uint4 *>(dst + 8) = pack8_bf16(b8);
        }
    };

    // Work in flight, for the error path: completions issued on each barrier
    // (thread 0 issues everything) and completions waited for (every thread
    // keeps the same counts).
    int issued_t[2] = {0, 0}, issued_p[2] = {0, 0}, waited_t[2] = {0, 0}, waited_p[2] = {0, 0};
    int issued_w = 0, issued_k = 0, issued_m1 = 0, issued_mb = 0, issued_m3 = 0;
    int waited_w = 0, waited_k = 0, waited_m1 = 0, waited_mb = 0, waited_m3 = 0;
    bool aborted = false;

    // All threads wait; false (uniformly) when any thread gave up.  ok_in: the
    // result of a bounded wait this thread already made.
    auto wait_all = [&](uint32_t bar, uint32_t ph, bool ok_in) -> bool {
        const bool ok = ok_in && mbar_wait(bar, ph, polls, prm.st);
        if (__syncthreads_or(!ok)) return false;
        tc_fence_after();
        return true;
    };
    auto before_sync = [&]() {  // smem written by threads -> visible to the tensor core
        fence_async_smem();
        tc_fence_before();
    };

    store_state_bf16();
    if (tid == 32) {
        for (int n = 0; n < CHAIN_PREFETCH && n < nseg; ++n) prefetch_l2(recs + (size_t)n * REC_BYTES, REC_BYTES);
    }
    if (nseg > 0) {
        if (tid == 0) {
            issue_t(0); issue_w(0); issue_p(0); issue_k(0);
            if (nseg > 1) { issue_t(1); issue_p(1); }
        }
        issued_t[0] = issued_p[0] = issued_w = issued_k = 1;
        if (nseg > 1) issued_t[1] = issued_p[1] = 1;
        load_v(0);
    }
    if (prm.inject_wait_polls != 0) {
        // Fault-injection hook: wait on a barrier nothing arrives on, so the
        // bounded wait gives up and the kernel takes its error path.
        const bool ok = mbar_wait(bar_never, 0u, prm.inject_wait_polls, prm.st);
        if (__syncthreads_or(!ok)) aborted = true;
    }
    if (nseg > 0 && !aborted) {
        build_vt();
        before_sync();
        if (!wait_all(bar_t(0), par2(0), true)) aborted = true;
        else { ++waited_t[0]; if (tid == 0) mma_u(0); }
        if (!aborted) {
            before_sync();  // S0
            if (!wait_all(bar_w, 0u, true)) aborted = true;
            else ++waited_w;
        }
    }

    for (int n = 0; n < nseg && !aborted; ++n) {
        const uint32_t par = (uint32_t)(n & 1);
        const bool more = n + 1 < nseg;

        // ---- 1(n), then 3b(n-1) behind it ----
        if (tid == 0) {
            mma_1(n);
            umma_commit(bar_m1);
            if (n >= 1) { mma_3b(n - 1); umma_commit(bar_mb); }
            if (more && n >= 1) issue_t(n + 1);  // its buffer's last reader U(n-1) is done
        }
        ++issued_m1;
        if (n >= 1) ++issued_mb;
        if (more && n >= 1) ++issued_t[(n + 1) & 1];
        if (tid == 32 && n + CHAIN_PREFETCH < nseg)
            prefetch_l2(recs + (size_t)(n + CHAIN_PREFETCH) * REC_BYTES, REC_BYTES);
        if (more) load_v(n + 1);
        if (!wait_all(bar_m1, par, true)) { aborted = true; break; }
        ++waited_m1;
        if (tid == 0 && more) issue_w(n + 1);  // WQ(n) is consumed
        if (more) ++issued_w;

        // ---- Vnew(n) = U - W S0 -> Vnew^T tile n & 1 (lane quarters 0, 1) ----
        if (lq < 2) {
            float u[16], w[16];
            tmem_ld16(tmem + lane_base + L::TM_U + cg * CPT, u);
            tmem_ld16(tmem + lane_base + L::TM_D1 + (n & 1) * VS + cg * CPT, w);
            tmem_wait_ld();
            uint8_t *vn = sm + L::OFF_VN + (n & 1) * VS * 256;
#pragma unroll
            for (int e = 0; e < 16; ++e)
                *reinterpret_cast<uint32_t *>(vn + kmaj_s<128, 4>(cg * CPT + e, ch, VS * 128)) = tf32_bits(u[e] - w[e]);
        }
        before_sync();
        if (!wait_all(bar_k, par, true)) { aborted = true; break; }
        ++waited_k;

        // ---- 3a(n), then U(n+1) behind it; meanwhile the output of chunk n-1 ----
        if (tid == 0) { mma_3a(n); umma_commit(bar_m3); }
        ++issued_m3;
        bool ok_mb = true;
        if (lq >= 2 && n >= 1) {  // output of chunk n-1 once 3b(n-1) is done
            ok_mb = mbar_wait(bar_mb, (uint32_t)((n - 1) & 1), polls, prm.st);
            if (ok_mb) { tc_fence_after(); write_output(n - 1); }
        }
        if (more) {
            build_vt();  // V^T is free: U(n) completed before product 1(n)
            before_sync();
            if (!wait_all(bar_t(n + 1), par2(n + 1), ok_mb)) { aborted = true; break; }
            ++waited_t[(n + 1) & 1];
            if (tid == 0) mma_u(n + 1);  // U is free: Vnew(n) has read it
        } else {
            tc_fence_before();
            if (__syncthreads_or(!ok_mb)) { aborted = true; break; }
        }
        if (n >= 1) ++waited_mb;

        // ---- state update, S = e^{Gamma_C} S0 + K-hat^T Vnew ----
        if (!wait_all(bar_m3, par, true)) { aborted = true; break; }
        ++waited_m3;
        if (tid == 0 && more) {
            issue_k(n + 1);                  // K-hat(n) is consumed
            if (n >= 1) issue_p(n + 1);      // P(n-1)'s buffer: 3b(n-1) completed before 3a(n)
        }
        if (more) {
            ++issued_k;
            if (n >= 1) ++issued_p[(n + 1) & 1];
        }
        if (ch < DK) {  // warp-uniform
            const float dc = reinterpret_cast<const float *>(sm + L::OFF_DEC + (n & 1) * 512)[ch];
            float t[16];
            tmem_ld16(tmem + lane_base + L::TM_D3 + cg * CPT, t);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) S[e] = dc * S[e] + t[e];
        }
        store_state_bf16();  // S0 is free: product 1(n) completed
        // P(n) (read by 3b(n) behind the next product 1) and WQ(n+1)
        before_sync();
        {
            const bool ok = mbar_wait(bar_p(n), par2(n), polls, prm.st) &&
                            (!more || mbar_wait(bar_w, par ^ 1u, polls, prm.st));
            if (__syncthreads_or(!ok)) { aborted = true; break; }
            tc_fence_after();
        }
        ++waited_p[n & 1];
        if (more) ++waited_w;
    }

    // ---- the last chunk's output: 3b(N-1) ----
    if (!aborted && nseg > 0) {
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (tid == 0) { mma_3b(nseg - 1); umma_commit(bar_mb); }
        ++issued_mb;
        bool ok = true;
        if (lq >= 2) {
            ok = mbar_wait(bar_mb, (uint32_t)((nseg - 1) & 1), polls, prm.st);
            if (ok) { tc_fence_after(); write_output(nseg - 1); }
        }
        if (__syncthreads_or(!ok)) aborted = true;
        else ++waited_mb;
    }

    if (aborted) {
        // Leave nothing in flight that targets this CTA's shared memory or TMEM:
        // wait, in order, for every completion issued and not yet waited for
        // (phases complete in order; each wait is bounded).
        if (tid == 0) {
            auto drain = [&](uint32_t bar, int waited, int issued) {
                for (int j = waited; j < issued; ++j) mbar_wait(bar, (uint32_t)(j & 1), ~0ull, prm.st);
            };
            drain(bar_m1, waited_m1, issued_m1);
            drain(bar_mb, waited_mb, issued_mb);
            drain(bar_m3, waited_m3, issued_m3);
            for (int s2 = 0; s2 < 2; ++s2) {
                drain(bar_t(s2), waited_t[s2], issued_t[s2]);
                drain(bar_p(s2), waited_p[s2], issued_p[s2]);
            }
            drain(bar_w, waited_w, issued_w);
            drain(bar_k, waited_k, issued_k);
        }
    } else if (prm.hT != nullptr && ch < DK) {
        float4 *dst = reinterpret_cast<float4 *>(prm.hT + (((size_t)b * H + h) * DK + ch) * DV + scol);
#pragma unroll
        for (int e = 0; e < CPT / 4; ++e) dst[e] = make_float4(S[4 * e], S[4 * e + 1], S[4 * e + 2], S[4 * e + 3]);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, L::TM_COLS);
}

template <int DK>
static cudaError_t launch_chain_t(const CUtensorMap *maps, const ChainParams &prm, cudaStream_t stream) {
    using L = ChainLayout<DK>;
    cudaError_t e = cudaFuncSetAttribute(chain_kernel<DK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         L::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    chain_kernel<DK><<<prm.B * prm.H * prm.nslices, CHAIN_THREADS, L::SMEM_BYTES, stream>>>(
        maps[0], maps[1], maps[2], maps[3], prm);
    return cudaGetLastError();
}

int chain_value_slice() { return CHAIN_VS; }

// maps: the record parts WQ, P, K-hat, T' (see chunk_common.cuh)
cudaError_t launch_chain(const CUtensorMap *maps, const ChainParams &prm, int dk, cudaStream_t stream) {
    if (dk == 128) return launch_chain_t<128>(maps, prm, stream);
    return launch_chain_t<64>(maps, prm, stream);
}

}  // namespace kda
