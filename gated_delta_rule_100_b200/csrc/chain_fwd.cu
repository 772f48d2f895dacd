// chain_fwd.cu -- the inter-chunk (state-passing) half of the chunkwise KDA
// prefill (sm_100a).
//
// One CTA owns one (b, h, slice of VS value columns) and walks the chunks of a
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
// holds row c, VS/4 columns); a bf16 copy in shared memory feeds the tensor
// core.  All products run as 128-row UMMAs with TMEM accumulators:
//   1   D1 = [W; Q e^G] S0            bf16, A = record WQ (MN-major)
//   U   U  = T' V                      tf32, A = record T' (rows 64..127 unused)
//   3a  D3 = K-hat^T Vnew              tf32
//   3b  D1 += [.; P] Vnew              tf32, rows 64..127 = the output block
// Records arrive by 1-D bulk copies in two groups, each reloaded for the next
// chunk as soon as its last reader of this chunk is done: group A (WQ, T',
// e^{Gamma_C}) after product 1, group B (P, K-hat) after product 3b.  The
// values V are read with plain coalesced loads one chunk ahead.
#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "chunk_common.cuh"
#include "chunk_params.cuh"
#include "kda_device.cuh"

namespace kda {

constexpr int CHAIN_THREADS = 512;
constexpr int CHAIN_PREFETCH = 4;  // chunks between the L2 prefetch of a record and its use

template <int DK, int VS>
struct ChainLayout {
    static_assert(DK == 64 || DK == 128, "dk");
    static_assert(VS == 64 || VS == 128, "value slice");
    // record image at offset 0 (same offsets as in global memory)
    static constexpr int OFF_PB = REC_P - 8192;              // 128-row view whose rows 64..127 are P
    static constexpr int OFF_DEC = REC_BYTES;                // two 512-byte slots of e^{Gamma_C}
    static constexpr int OFF_S0 = align1k(OFF_DEC + 1024);   // bf16 MN-major S0 [DK][VS], 128B swizzle
    static constexpr int OFF_VT = OFF_S0 + DK * VS * 2;      // tf32 K-major V^T [VS][64]
    static constexpr int OFF_VN = OFF_VT + VS * 256;         // tf32 K-major Vnew^T [VS][64]
    static constexpr int OFF_MISC = OFF_VN + VS * 256;       // barriers, TMEM address, abort flag
    static constexpr int TOTAL = OFF_MISC + 1024;
    static constexpr int SMEM_BYTES = TOTAL + 1024;          // slack for the 1 KB base alignment
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
    static_assert(REC_T + 24576 <= TOTAL, "the 128-row view of T' reads 8 KB past it");

    static constexpr uint32_t TM_U = 0;     // U (lane = token)
    static constexpr uint32_t TM_D1 = 128;  // [W; Q e^G] S0, then += P Vnew on lanes 64..127
    static constexpr uint32_t TM_D3 = 256;  // K-hat^T Vnew (lane = key channel)
    static constexpr uint32_t TM_COLS = 512;
};

template <int DK, int VS>
__global__ void __launch_bounds__(CHAIN_THREADS, 1)
chain_kernel(const __grid_constant__ CUtensorMap tm_wq, const __grid_constant__ CUtensorMap tm_p,
             const __grid_constant__ CUtensorMap tm_kh, const __grid_constant__ CUtensorMap tm_t,
             const ChainParams prm) {
    using L = ChainLayout<DK, VS>;
    constexpr int CPT = VS / 4;            // value columns per thread (state, Vnew, output)
    constexpr int NP = VS / 2;             // value column pairs (V loads)
    constexpr int TG = CHAIN_THREADS / NP; // token groups (V loads)
    constexpr int TPT = CH / TG;           // tokens per thread (V loads)
    static_assert(TPT % 4 == 0, "V^T tile stores take four tokens");
    constexpr uint32_t TX_A = (uint32_t)(DK * 256 + 16384 + 512);
    constexpr uint32_t TX_B = (uint32_t)(16384 + 32768);

    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(sm);
    uint64_t *s_bars = reinterpret_cast<uint64_t *>(sm + L::OFF_MISC);
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(sm + L::OFF_MISC + 64);
    const uint32_t bar_a = smem_u32(&s_bars[0]);
    const uint32_t bar_b = smem_u32(&s_bars[1]);
    const uint32_t bar_m1 = smem_u32(&s_bars[2]);
    const uint32_t bar_3 = smem_u32(&s_bars[3]);
    const uint32_t bar_m3 = smem_u32(&s_bars[4]);
    const uint32_t bar_never = smem_u32(&s_bars[5]);  // nothing arrives on it (fault-injection hook)

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lq = warp & 3;            // TMEM lane quarter of this warp
    const int cg = warp >> 2;           // value-column group of this warp
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
        for (int i = 0; i < 6; ++i) mbar_init(smem_u32(&s_bars[i]), 1);
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

    // Record parts are plain row-major in global memory; the tensor loads
    // write them in the swizzled operand layouts.
    auto issue_a = [&](int n) {
        const uint8_t *r = recs + (size_t)n * REC_BYTES;
        mbar_expect_tx(bar_a, TX_A);
#pragma unroll
        for (int nb = 0; nb < 2; ++nb) tma_load_3d(sbase + REC_WQ + nb * DK * 128, &tm_wq, bar_a, nb * 64, 0, rec0 + n);
#pragma unroll
        for (int kb = 0; kb < 2; ++kb) tma_load_3d(sbase + REC_T + kb * 8192, &tm_t, bar_a, kb * 32, 0, rec0 + n);
        bulk_load(sbase + L::OFF_DEC + (n & 1) * 512, r + REC_DEC, 512, bar_a);
    };
    auto issue_b = [&](int n) {
        mbar_expect_tx(bar_b, TX_B);
#pragma unroll
        for (int kb = 0; kb < 2; ++kb) {
            tma_load_3d(sbase + REC_P + kb * 8192, &tm_p, bar_b, kb * 32, 0, rec0 + n);
            tma_load_3d(sbase + REC_KH + kb * 16384, &tm_kh, bar_b, kb * 32, 0, rec0 + n);
        }
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

    bool pend_a = false, pend_b = false, pend_mma = false, aborted = false;
    uint32_t ph_mma_last = 0;  // parity of the MMA barrier last committed (bar_m3 or bar_m1)
    uint32_t bar_mma_last = bar_m1;

    // all threads wait; returns false (uniformly) when any thread gave up
    auto wait_all = [&](uint32_t bar, uint32_t ph) -> bool {
        const bool ok = mbar_wait(bar, ph, polls, prm.st);
        if (__syncthreads_or(!ok)) return false;
        tc_fence_after();
        return true;
    };
    auto sync_for_mma = [&]() {
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    };

    const uint32_t id_u = make_idesc(2, false, false, 128, VS);
    const uint32_t id_1 = make_idesc(1, true, true, 128, VS);
    const uint32_t id_3 = make_idesc(2, false, false, 128, VS);
    auto issue_u = [&]() {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
            umma<1>(tmem + L::TM_U, desc_kmaj_s<128, 4>(sbase + REC_T, 8192, kk * 8),
                    desc_kmaj_s<128, 4>(sbase + L::OFF_VT, VS * 128, kk * 8), id_u, kk > 0);
    };

    store_state_bf16();
    if (tid == 32) {
        for (int n = 1; n < CHAIN_PREFETCH && n < nseg; ++n) prefetch_l2(recs + (size_t)n * REC_BYTES, REC_BYTES);
    }
    if (nseg > 0) {
        if (tid == 0) { issue_a(0); issue_b(0); }
        pend_a = pend_b = true;
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
        if (!wait_all(bar_a, 0)) aborted = true;
        else {
            pend_a = false;
            sync_for_mma();
            if (tid == 0) issue_u();
        }
    }

    for (int n = 0; n < nseg && !aborted; ++n) {
        const uint32_t par = (uint32_t)(n & 1);
        const bool more = n + 1 < nseg;
        const int t0 = (prm.n_begin + n) * CH;

        // ---- 1: D1 = [W; Q e^G] S0 (U of this chunk is already queued ahead of it) ----
        if (tid == 32 && n + CHAIN_PREFETCH < nseg)  // records a few chunks ahead -> L2
            prefetch_l2(recs + (size_t)(n + CHAIN_PREFETCH) * REC_BYTES, REC_BYTES);
        if (tid == 0) {
#pragma unroll
            for (int kk = 0; kk < DK / 16; ++kk)
                umma<0>(tmem + L::TM_D1, desc_mnmaj<128>(sbase + REC_WQ, DK, kk * 16),
                        desc_mnmaj<128>(sbase + L::OFF_S0, DK, kk * 16), id_1, kk > 0);
            umma_commit(bar_m1);
        }
        pend_mma = true; bar_mma_last = bar_m1; ph_mma_last = par;
        if (more) load_v(n + 1);
        if (!wait_all(bar_m1, par)) { aborted = true; break; }
        pend_mma = false;
        if (tid == 0 && more) issue_a(n + 1);
        pend_a = more;

        // ---- 2: Vnew = U - W S0 -> Vnew^T tile (tf32) ----
        if (lq < 2) {
#pragma unroll
            for (int c16 = 0; c16 < CPT; c16 += 16) {
                float u[16], w[16];
                tmem_ld16(tmem + lane_base + L::TM_U + cg * CPT + c16, u);
                tmem_ld16(tmem + lane_base + L::TM_D1 + cg * CPT + c16, w);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    *reinterpret_cast<uint32_t *>(sm + L::OFF_VN + kmaj_s<128, 4>(cg * CPT + c16 + e, ch, VS * 128)) =
                        tf32_bits(u[e] - w[e]);
            }
        }
        if (!wait_all(bar_b, par)) { aborted = true; break; }
        pend_b = false;
        sync_for_mma();

        // ---- 3a: D3 = K-hat^T Vnew;  3b: D1 += P Vnew ----
        if (tid == 0) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                umma<1>(tmem + L::TM_D3, desc_kmaj_s<128, 4>(sbase + REC_KH, 128 * 128, kk * 8),
                        desc_kmaj_s<128, 4>(sbase + L::OFF_VN, VS * 128, kk * 8), id_3, kk > 0);
            umma_commit(bar_3);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                umma<1>(tmem + L::TM_D1, desc_kmaj_s<128, 4>(sbase + L::OFF_PB, 8192, kk * 8),
                        desc_kmaj_s<128, 4>(sbase + L::OFF_VN, VS * 128, kk * 8), id_3, 1u);
            umma_commit(bar_m3);
        }
        pend_mma = true; bar_mma_last = bar_m3; ph_mma_last = par;
        if (more) build_vt();  // V^T is free: U of this chunk completed before product 1

        // ---- 4: state update, S = e^{Gamma_C} S0 + K-hat^T Vnew ----
        if (!wait_all(bar_3, par)) { aborted = true; break; }
        if (ch < DK) {
            const float dc = reinterpret_cast<const float *>(sm + L::OFF_DEC + (n & 1) * 512)[ch];
#pragma unroll
            for (int c16 = 0; c16 < CPT; c16 += 16) {
                float t[16];
                tmem_ld16(tmem + lane_base + L::TM_D3 + cg * CPT + c16, t);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e) S[c16 + e] = dc * S[c16 + e] + t[e];
            }
        }
        store_state_bf16();  // S0 is free: product 1 completed

        // ---- 5: output rows, O = scale (Q e^G S0 + P Vnew) ----
        if (!wait_all(bar_m3, par)) { aborted = true; break; }
        pend_mma = false;
        if (tid == 0 && more) issue_b(n + 1);
        pend_b = more;
        if (lq >= 2) {  // warp-uniform: the TMEM loads are warp-collective; only the stores are guarded
            const int i = ch - 64;
            const bool valid = t0 + i < T;
            uint16_t *dst = prm.out + (((size_t)b * T + t0 + i) * H + h) * DV + col0 + cg * CPT;
#pragma unroll
            for (int c16 = 0; c16 < CPT; c16 += 16) {
                float t[16];
                tmem_ld16(tmem + lane_base + L::TM_D1 + cg * CPT + c16, t);
                tmem_wait_ld();
                if (valid) {
                    float a8[8], b8[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) { a8[e] = prm.scale * t[e]; b8[e] = prm.scale * t[8 + e]; }
                    *reinterpret_cast<uint4 *>(dst + c16) = pack8_bf16(a8);
                    *reinterpret_cast<uint4 *>(dst + c16 + 8) = pack8_bf16(b8);
                }
            }
        }
        if (more) {
            if (!wait_all(bar_a, par ^ 1u)) { aborted = true; break; }
            pend_a = false;
            sync_for_mma();
            if (tid == 0) issue_u();
        }
    }

    if (aborted) {
        // Leave nothing in flight that targets this CTA's shared memory or TMEM.
        // A copy in flight completes the current phase of its barrier: waiting on
        // both parities waits for exactly that phase.
        if (tid == 0) {
            if (pend_mma) mbar_wait(bar_mma_last, ph_mma_last, ~0ull, prm.st);
            if (pend_a) { mbar_wait(bar_a, 0u, ~0ull, prm.st); mbar_wait(bar_a, 1u, ~0ull, prm.st); }
            if (pend_b) { mbar_wait(bar_b, 0u, ~0ull, prm.st); mbar_wait(bar_b, 1u, ~0ull, prm.st); }
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

template <int DK, int VS>
static cudaError_t launch_chain_t(const CUtensorMap *maps, const ChainParams &prm, cudaStream_t stream) {
    using L = ChainLayout<DK, VS>;
    cudaError_t e = cudaFuncSetAttribute(chain_kernel<DK, VS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         L::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    chain_kernel<DK, VS><<<prm.B * prm.H * prm.nslices, CHAIN_THREADS, L::SMEM_BYTES, stream>>>(
        maps[0], maps[1], maps[2], maps[3], prm);
    return cudaGetLastError();
}

// maps: the record parts WQ, P, K-hat, T' (see chunk_common.cuh)
cudaError_t launch_chain(const CUtensorMap *maps, const ChainParams &prm, int dk, cudaStream_t stream) {
    const int vs = prm.DV / prm.nslices;
    if (dk == 128)
        return vs == 128 ? launch_chain_t<128, 128>(maps, prm, stream) : launch_chain_t<128, 64>(maps, prm, stream);
    return vs == 128 ? launch_chain_t<64, 128>(maps, prm, stream) : launch_chain_t<64, 64>(maps, prm, stream);
}

}  // namespace kda
