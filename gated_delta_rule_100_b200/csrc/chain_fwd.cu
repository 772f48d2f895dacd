// chain_fwd.cu -- the inter-chunk (state-passing) half of the chunkwise KDA
// prefill (sm_100a).
//
// One CTA owns one (b, h, slice of 64 or 128 value columns) and walks the chunks of a
// segment in order, reading the per-chunk records of the prep kernel
// (prep_fwd.cu; layout in chunk_common.cuh).  Per chunk, S0 = state at the
// chunk start:
//   U    = T' V                      T' = T Diag(beta), V the chunk's values
//   Vnew = U - W S0                  the delta-rule corrected writes
//   O    = scale ((Q e^Gamma) S0 + P Vnew)
//   S    = Diag(e^{Gamma_C}) S0 + K-hat^T Vnew
// (state passing across chunks with the causal intra-chunk correction,
// section 4 of "Kimi Linear's Hybrid Linear Attention Architecture: A
// Technical Breakdown").  All products are 128-row UMMAs with TMEM
// accumulators:
//   1   D1 = [W; Q e^G] S0            bf16, A = record WQ (MN-major)
//   U   U  = T' V                      tf32, A = record T' (rows 64..127 unused)
//   3a  D3 = K-hat^T Vnew              fp16
//   3b  D1 += [.; P] Vnew              fp16, rows 64..127 = the output block
// (fp16 keeps tf32's 10-bit mantissa; K-hat, P and Vnew are bounded in
// magnitude, T' is kept in tf32 for its range).
//
// Warp roles.  One loader warp (its lane 0) issues every record load, one
// issuer warp (its lane 0) issues every product, and sixteen compute warps move
// data between TMEM, registers and shared memory.  They never meet at a
// CTA-wide barrier inside the loop: each hand-off is an mbarrier -- a full/empty
// pair per record buffer between the loader and its readers, product commits
// and the compute warps' arrivals (Vnew written, an output block read, V^T
// written, S0 written) between the issuer and the compute warps -- so the
// tensor pipe, which executes in issue order, is fed as soon as each operand is
// ready.  A TMA issue can hold its thread for hundreds of cycles while the
// SM's copy engine is busy, which is why no load sits in the issuer's path.
// Per chunk n it runs 1(n), 3b(n-1), 3a(n), U(n+1): only 1 and 3a lie on the
// state's critical path, the other two fill the pipe while the compute warps
// form Vnew(n) and update the state.  Buffers: two output accumulators and two
// each of the Vnew tiles, WQ (at 64 columns), P, K-hat and T'; one V^T and one
// S0.
//
// The state lives in fp32 registers (compute thread (c, g) holds row c and
// VS / 4 columns); a bf16 copy in shared memory feeds the tensor core.  The
// values V are read with plain coalesced loads one chunk before their V^T tile
// is built, issued after the state update: global loads in flight delay the
// compute warps' TMEM loads.
#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "chunk_common.cuh"
#include "chunk_params.cuh"
#include "kda_device.cuh"

namespace kda {

constexpr int CHAIN_WORKERS = 512;                   // sixteen compute warps
constexpr int CHAIN_THREADS = CHAIN_WORKERS + 64;    // plus the issuer and loader warps

// VS value columns per CTA (64 or 128).  Every CTA of a (b, h) reads that
// (b, h)'s whole records, so fewer, wider slices read fewer record bytes; the
// 128-column layout has room for one WQ buffer, the 64-column one for two.
template <int DK, int VS_>
struct ChainLayout {
    static_assert(DK == 64 || DK == 128, "dk");
    static_assert(VS_ == 64 || VS_ == 128, "value slice");
    static constexpr int VS = VS_;
    static constexpr int WS = VS == 64 ? 2 : 1;          // WQ buffers
    // Record tiles (32B swizzle, 32-byte rows of 16 tokens; 32 KB WQ slots):
    static constexpr int OFF_WQ = 0;                     // bf16 MN-major [8][DK][16]: [W; Q e^G]
    static constexpr int OFF_P = WS * 32768;             // two fp16 K-major [4][64][16] (8 KB)
    static constexpr int OFF_KH = OFF_P + 16384;         // two fp16 K-major [4][128][16] (16 KB)
    static constexpr int OFF_T = OFF_KH + 32768;         // two tf32 K-major [64][64] (8 KB K-blocks)
    static constexpr int OFF_DEC = OFF_T + 32768;        // two 512-byte slots of e^{Gamma_C} (with K-hat)
    static constexpr int OFF_S0 = OFF_DEC + 1024;        // bf16 MN-major S0 [DK][VS], 128B swizzle
    static constexpr int OFF_VT = OFF_S0 + DK * VS * 2;  // tf32 K-major V^T [VS][64]
    static constexpr int OFF_VN = OFF_VT + VS * 256;     // two fp16 MN-major Vnew [64][VS], 128B swizzle
    static constexpr int OFF_MISC = OFF_VN + 2 * VS * 128;  // barriers, TMEM address, abort flag
    static constexpr int TOTAL = OFF_MISC + 1024;
    static constexpr int SMEM_BYTES = TOTAL + 1024;  // slack for the 1 KB base alignment
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
    static_assert(OFF_S0 % 1024 == 0 && OFF_VT % 1024 == 0 && OFF_VN % 1024 == 0, "1 KB aligned tiles");
    // The 128-row views read 2 KB before each 2 KB block of P (rows 0..63,
    // discarded) and 8 KB past T's second buffer (rows 64..127, discarded).
    static_assert(OFF_P >= 2048 && OFF_T + 2 * 16384 + 8192 <= TOTAL, "operand views stay in bounds");

    static constexpr uint32_t TM_U = 0;          // U (lane = token)
    static constexpr uint32_t TM_D1 = VS;        // two: [W; Q e^G] S0, then += P Vnew on lanes 64..127
    static constexpr uint32_t TM_D3 = 3 * VS;    // K-hat^T Vnew (lane = key channel)
    static constexpr uint32_t TM_COLS = 4 * VS;
};

template <int DK, int VS_>
__global__ void __launch_bounds__(CHAIN_THREADS, 1)
chain_kernel(const __grid_constant__ CUtensorMap tm_wq, const __grid_constant__ CUtensorMap tm_p,
             const __grid_constant__ CUtensorMap tm_kh, const __grid_constant__ CUtensorMap tm_t,
             const ChainParams prm) {
    using L = ChainLayout<DK, VS_>;
    constexpr int VS = L::VS, WS = L::WS;
    constexpr int CPT = VS / 4;             // value columns per compute thread
    constexpr int NP = VS / 2;              // value column pairs (V loads)
    constexpr int TG = CHAIN_WORKERS / NP;  // token groups (V loads)
    constexpr int TPT = CH / TG;            // tokens per compute thread (V loads)
    static_assert(TPT % 4 == 0 && CPT % 16 == 0, "thread mapping");
    constexpr uint32_t TX_T = 16384, TX_W = DK * 256, TX_P = 8192, TX_K = 16384 + 512;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(sm);
    uint64_t *s_bars = reinterpret_cast<uint64_t *>(sm + L::OFF_MISC);
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(sm + L::OFF_MISC + 256);
    volatile int *s_abort = reinterpret_cast<volatile int *>(sm + L::OFF_MISC + 260);

    // mbarriers (each tracks one phase at a time; the protocol never arms a
    // barrier again before its previous phase was waited for)
    enum { B_W0, B_W1, B_P0, B_P1, B_K0, B_K1, B_T0, B_T1,       // record buffers full (loader, count 1)
           B_M1, B_MB, B_M3, B_WE0, B_WE1, B_TE0, B_TE1, B_PE0, B_PE1,  // product commits (count 1)
           B_S0, B_VT, B_VN0, B_VN1, B_OUT0, B_OUT1, B_KE0, B_KE1,  // compute-warp arrivals
           B_NEVER, NBARS };
    auto bar = [&](int i) { return smem_u32(&s_bars[i]); };
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const bool issuer = warp == CHAIN_WORKERS / 32;
    const bool loader = warp == CHAIN_WORKERS / 32 + 1;
    const int slot = blockIdx.x % prm.slots;
    const int rest = blockIdx.x / prm.slots;
    const int part = prm.part0 + rest % prm.nparts;
    const int bh = rest / prm.nparts;
    const int h = bh % prm.H, seq = bh / prm.H;
    const int H = prm.H, DV = prm.DV;
    const int nvs = DV / VS;                       // value slices
    const bool trans = prm.pass_a && part > 0;     // a transition of the two-level pass
    const bool ident = trans && slot >= nvs;       // columns of the identity instead of values
    if (!trans && slot >= nvs) return;             // pass A's part 0 needs value slices only
    const int col0 = (ident ? slot - nvs : slot) * VS;
    const ChainGeo geo = chain_geo(prm.gm, H, seq, h, part, prm.parts, prm.part_len);
    const int nseg = geo.nch;  // chunks of this (sequence, head, part) in this launch
    const uint8_t *recs = prm.ws + (size_t)geo.rec0 * REC_BYTES;
    const int rec0 = (int)geo.rec0;  // index of its first record in the tensor maps
    // Where the state comes from and goes to (row stride ld, this slice's column 0 at col0):
    // the sequence's h0/hT (or the carry between segments), or the two-level pass's buffers.
    const size_t BHn = (size_t)prm.gm.nseqs * H;
    const float *s_in = nullptr;  // NULL: zero (or, ident, the identity)
    float *s_out = nullptr;       // NULL: not written
    int s_ld = DV;
    if (trans) {
        if (ident) {
            s_out = prm.p_trans + ((size_t)part * BHn + bh) * DK * DK;
            s_ld = DK;
        } else {
            s_out = prm.p_local + ((size_t)part * BHn + bh) * DK * DV;
        }
    } else {
        const float *h0p = geo.first ? prm.h0 : prm.carry;
        float *hTp = geo.last ? prm.hT : prm.carry;
        s_in = part == 0 ? (h0p ? h0p + ((size_t)seq * H + h) * DK * DV : nullptr)
                         : prm.p_start + ((size_t)part * BHn + bh) * DK * DV;
        if (part == prm.parts - 1) s_out = hTp ? hTp + ((size_t)seq * H + h) * DK * DV : nullptr;
        else if (prm.pass_a) s_out = prm.p_start + ((size_t)(part + 1) * BHn + bh) * DK * DV;
    }
    const uint64_t polls = prm.st.wait_polls;
    const long long rows = geom_rows(prm.gm);  // token rows of v and out (debug-build checks)

    if (tid == 0) {
        stamp_start(prm.stamp);
        for (int i = 0; i < NBARS; ++i) {
            const bool group = i >= B_S0 && i <= B_KE1;
            const bool all16 = i == B_S0 || i == B_VT || i == B_KE0 || i == B_KE1;
            const uint32_t cnt = !group ? 1u : all16 ? 16u : 8u;  // warps that arrive
            mbar_init(bar(i), cnt);
        }
        *s_abort = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(s_tmem), L::TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;

    // Bounded wait agreed by the whole warp; false once this CTA aborts.
    // Bounded wait of the single thread that runs the loader or the issuer.
    auto wait1 = [&](int i, uint32_t par) -> bool {
        if (mbar_wait(bar(i), par, polls, prm.st)) return true;
        *s_abort = 1;
        return false;
    };
    // Bounded wait agreed by the whole warp (a compute warp).
    auto wait_warp = [&](int i, uint32_t par) -> bool {
        const bool ok = __all_sync(0xffffffffu, mbar_wait(bar(i), par, polls, prm.st));
        if (!ok) *s_abort = 1;
        return ok;
    };
    auto arrive = [&](int i) {  // one arrival per warp, after all its lanes' prior work
        __syncwarp();
        if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar(i)) : "memory");
    };

    if (prm.inject_wait_polls != 0) {
        // Fault-injection hook: wait on a barrier nothing arrives on, so the
        // bounded wait gives up and the kernel takes its error path.
        if (!mbar_wait(bar(B_NEVER), 0u, prm.inject_wait_polls, prm.st)) *s_abort = 1;
        __syncthreads();
    }

    if (loader && lane == 0) {
        // ====================== loader warp (lane 0; the rest idle) ======================
        // Chunk j's records go to buffer j % WS (WQ) or j & 1 (the rest), each
        // once its empty barrier says the readers of chunk j - WS (j - 2) are done.
        uint32_t armed = 0, parity = 0;  // per full barrier: ever armed, count of armed completions mod 2
        auto load_w = [&](int n) {  // WQ(n)
            const int s = n % WS, bi = B_W0 + s;
            mbar_expect_tx(bar(bi), TX_W);
            tma_load_4d(sbase + L::OFF_WQ + s * 32768, &tm_wq, bar(bi), 0, 0, 0, rec0 + n);
            armed |= 1u << bi; parity ^= 1u << bi;
        };
        auto load_p = [&](int n) {  // P(n)
            const int s = n & 1, bi = B_P0 + s;
            mbar_expect_tx(bar(bi), TX_P);
            tma_load_4d(sbase + L::OFF_P + s * 8192, &tm_p, bar(bi), 0, 0, 0, rec0 + n);
            armed |= 1u << bi; parity ^= 1u << bi;
        };
        auto load_k = [&](int n) {  // K-hat(n) and e^{Gamma_C}(n)
            const int s = n & 1, bi = B_K0 + s;
            mbar_expect_tx(bar(bi), TX_K);
            tma_load_4d(sbase + L::OFF_KH + s * 16384, &tm_kh, bar(bi), 0, 0, 0, rec0 + n);
            // debug build: a record past the tensor maps' extent is reported, and the
            // plain bulk copy then reads record 0 instead (the barrier still completes)
            const bool in = KDA_CHECK(prm.st, rec0 + n < prm.nrec);
            bulk_load(sbase + L::OFF_DEC + s * 512, (in ? recs + (size_t)n * REC_BYTES : prm.ws) + REC_DEC, 512, bar(bi));
            armed |= 1u << bi; parity ^= 1u << bi;
        };
        auto load_t = [&](int n) {  // T'(n)
            const int s = n & 1, bi = B_T0 + s;
            mbar_expect_tx(bar(bi), TX_T);
            for (int kb = 0; kb < 2; ++kb)
                tma_load_3d(sbase + L::OFF_T + s * 16384 + kb * 8192, &tm_t, bar(bi), kb * 32, 0, rec0 + n);
            armed |= 1u << bi; parity ^= 1u << bi;
        };
        bool ok = *s_abort == 0 && nseg > 0;
        if (ok) {
            prefetch_tmap(&tm_wq); prefetch_tmap(&tm_p); prefetch_tmap(&tm_kh); prefetch_tmap(&tm_t);
        }
        // In the order their buffers free up: T' (product U(j-2)), K-hat and
        // e^{Gamma_C} (product 3a(j-2) and the state update of chunk j-2), WQ
        // (product 1(j-WS)), P (product 3b(j-2)).
        for (int j = 0; ok && j < nseg; ++j) {
            const uint32_t ph = (uint32_t)(((j - 2) >> 1) & 1);
            if (j >= 2 && !(ok = wait1(B_TE0 + (j & 1), ph))) break;
            load_t(j);
            if (j >= 2 && !(ok = wait1(B_KE0 + (j & 1), ph))) break;
            load_k(j);
            if (j >= WS && !(ok = wait1(B_WE0 + j % WS, (uint32_t)(((j - WS) / WS) & 1)))) break;
            load_w(j);
            if (j >= 2 && !(ok = wait1(B_PE0 + (j & 1), ph))) break;
            load_p(j);
        }
        if (*s_abort) {
            // Leave no copy in flight into this CTA's shared memory.  At most one
            // phase of each barrier is in flight, so waiting for the parity of the
            // last armed completion waits for everything on it.
            for (int i = 0; i <= B_T1; ++i)
                if ((armed >> i) & 1) mbar_wait(bar(i), ((parity >> i) & 1) ^ 1u, ~0ull, prm.st);
        }
    } else if (issuer && lane == 0) {
        // ====================== issuer warp (lane 0; the rest idle) ======================
        const uint32_t id_tf = make_idesc(2, false, false, 128, VS);
        const uint32_t id_bf = make_idesc(1, true, true, 128, VS);
        const uint32_t id_h = make_idesc(0, false, true, 128, VS);  // B = Vnew, MN-major
        uint32_t armed = 0, parity = 0;  // per commit barrier: ever committed, count of commits mod 2
        auto commit = [&](int bi) {
            umma_commit(bar(bi));
            armed |= 1u << bi; parity ^= 1u << bi;
        };
        // debug build: an operand view [lo, hi) (bytes from the tile base) inside the layout;
        // a view that is not skips its instructions (the commits still arrive)
        auto views_ok = [&](int alo, int ahi, int blo, int bhi) {
            return KDA_CHECK(prm.st, alo >= 0 && ahi <= L::TOTAL && blo >= 0 && bhi <= L::TOTAL);
        };
        auto mma_u = [&](int n) {  // U = T'(n) V(n)
            tc_fence_after();
            const int ta = L::OFF_T + (n & 1) * 16384;
            if (views_ok(ta, ta + 8192 + 16384, L::OFF_VT, L::OFF_VT + VS * 256))
            for (int kk = 0; kk < 8; ++kk)
                umma<1>(tmem + L::TM_U, desc_kmaj_s<128, 4>(sbase + L::OFF_T + (n & 1) * 16384, 8192, kk * 8),
                        desc_kmaj_s<128, 4>(sbase + L::OFF_VT, VS * 128, kk * 8), id_tf, kk > 0);
            if (n + 2 < nseg) commit(B_TE0 + (n & 1));  // T'(n) read: its buffer takes T'(n+2)
        };
        auto mma_1 = [&](int n) {  // D1[n & 1] = [W; Q e^G](n) S0
            tc_fence_after();
            const int wa = L::OFF_WQ + (n % WS) * 32768;
            if (views_ok(wa, wa + DK * 256, L::OFF_S0, L::OFF_S0 + DK * VS * 2))
            for (int kk = 0; kk < DK / 16; ++kk)
                umma<0>(tmem + L::TM_D1 + (n & 1) * VS, desc_mnmaj<32>(sbase + L::OFF_WQ + (n % WS) * 32768, DK, kk * 16),
                        desc_mnmaj<128>(sbase + L::OFF_S0, DK, kk * 16), id_bf, kk > 0);
            commit(B_M1);
            if (n + WS < nseg) commit(B_WE0 + n % WS);  // WQ(n) read
        };
        auto mma_3a = [&](int n) {  // D3 = K-hat(n)^T Vnew(n)
            tc_fence_after();
            const int ka = L::OFF_KH + (n & 1) * 16384, vb = L::OFF_VN + (n & 1) * VS * 128;
            if (views_ok(ka, ka + 16384, vb, vb + VS * 128))
            for (int kk = 0; kk < 4; ++kk)
                umma<0>(tmem + L::TM_D3, desc_kmaj<32, 2>(sbase + L::OFF_KH + (n & 1) * 16384, 128, kk * 16),
                        desc_mnmaj<128>(sbase + L::OFF_VN + (n & 1) * VS * 128, CH, kk * 16), id_h, kk > 0);
            commit(B_M3);
        };
        auto mma_3b = [&](int n) {  // D1[n & 1] rows 64..127 += P(n) Vnew(n)
            tc_fence_after();
            // the 128-row view of P starts 2 KB before the buffer (rows 0..63, discarded)
            const int pa = L::OFF_P + (n & 1) * 8192 - 2048, vb = L::OFF_VN + (n & 1) * VS * 128;
            if (views_ok(pa, pa + 10240, vb, vb + VS * 128))
            for (int kk = 0; kk < 4; ++kk)
                umma<0>(tmem + L::TM_D1 + (n & 1) * VS,
                        desc_kmaj<32, 2>(sbase + L::OFF_P + (n & 1) * 8192 - 2048, CH, kk * 16),
                        desc_mnmaj<128>(sbase + L::OFF_VN + (n & 1) * VS * 128, CH, kk * 16), id_h, 1u);
            commit(B_MB);
            if (n + 2 < nseg) commit(B_PE0 + (n & 1));  // P(n) read
        };

        bool ok = *s_abort == 0 && nseg > 0;
        if (ok) {
            ok = wait1(B_VT, 0u) && wait1(B_T0, 0u);
            if (ok) mma_u(0);
        }
        for (int n = 0; ok && n < nseg; ++n) {
            const bool more = n + 1 < nseg;
            if (!(ok = wait1(B_S0, (uint32_t)(n & 1)))) break;      // S0(n)
            if (!(ok = wait1(B_W0 + (n % WS), (uint32_t)((n / WS) & 1)))) break;  // WQ(n)
            if (n >= 2 && !(ok = wait1(B_OUT0 + (n & 1), (uint32_t)(((n - 2) >> 1) & 1)))) break;  // D1[n&1] free
            mma_1(n);
            if (n >= 1) {
                if (!(ok = wait1(B_P0 + ((n - 1) & 1), (uint32_t)(((n - 1) >> 1) & 1)))) break;  // P(n-1)
                mma_3b(n - 1);
            }
            if (!(ok = wait1(B_VN0 + (n & 1), (uint32_t)((n >> 1) & 1)))) break;  // Vnew(n)
            if (!(ok = wait1(B_K0 + (n & 1), (uint32_t)((n >> 1) & 1)))) break;   // K-hat(n)
            mma_3a(n);
            if (more) {
                if (!(ok = wait1(B_VT, (uint32_t)((n + 1) & 1)))) break;                 // V^T(n+1)
                if (!(ok = wait1(B_T0 + ((n + 1) & 1), (uint32_t)(((n + 1) >> 1) & 1)))) break;  // T'(n+1)
                mma_u(n + 1);  // U is free: Vnew(n) has read it
            }
        }
        if (ok) {  // the last chunk's output block, once output(N-2) has been read
            if (nseg >= 2) ok = wait1(B_OUT0 + (nseg & 1), (uint32_t)(((nseg - 2) >> 1) & 1));
            if (ok) ok = wait1(B_P0 + ((nseg - 1) & 1), (uint32_t)(((nseg - 1) >> 1) & 1));
            if (ok) mma_3b(nseg - 1);
        }
        if (*s_abort) {
            // Leave no product in flight that writes this CTA's TMEM or arrives on
            // its barriers (one phase in flight per barrier, as above).
            for (int i = B_M1; i <= B_PE1; ++i)
                if ((armed >> i) & 1) mbar_wait(bar(i), ((parity >> i) & 1) ^ 1u, ~0ull, prm.st);
        }
    } else if (!loader && !issuer) {
        // =============================== compute warps ===============================
        const int lq = warp & 3;              // TMEM lane quarter of this warp
        const int cg = warp >> 2;             // value-column group of this warp
        const int ch = lq * 32 + lane;        // TMEM lane of this thread
        const uint32_t lane_base = (uint32_t)(lq * 32) << 16;
        const int scol = col0 + cg * CPT;

        float S[CPT];  // S[ch][scol .. scol + CPT - 1]
#pragma unroll
        for (int e = 0; e < CPT; ++e) S[e] = (ident && ch == scol + e) ? 1.f : 0.f;
        // debug build: the state slice this CTA reads and writes
        const bool slice_in = KDA_CHECK(prm.st, seq < prm.gm.nseqs && part < prm.parts && scol + CPT <= s_ld);
        if (ch < DK && s_in != nullptr && slice_in) {
            const float4 *src = reinterpret_cast<const float4 *>(s_in + (size_t)ch * s_ld + scol);
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
            fence_async_smem();
        };
        // values: thread (p, tg) loads columns 2p, 2p + 1 of tokens tg TPT ..
        const int vp = tid % NP, vtg = tid / NP;
        uint32_t vr[TPT];
        auto load_v = [&](int n) {
            const int t0 = (geo.lc0 + n) * CH + vtg * TPT;
            const uint32_t *src = reinterpret_cast<const uint32_t *>(prm.v + ((size_t)(geo.row0 + t0) * H + h) * DV + col0) + vp;
#pragma unroll
            for (int u = 0; u < TPT; ++u)
                vr[u] = (!ident && t0 + u < geo.len && KDA_CHECK(prm.st, geo.row0 + t0 + u < rows))
                            ? __ldg(src + (size_t)u * H * DV / 2) : 0u;
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
            fence_async_smem();
        };
        // output rows of chunk n from D1[n & 1] (lane quarters 2, 3; the TMEM load is
        // warp-collective, only the stores are guarded)
        auto write_output = [&](int n) {
            const int i = ch - 64;
            const int t = (geo.lc0 + n) * CH + i;
            uint16_t *dst = prm.out + ((size_t)(geo.row0 + (t < geo.len ? t : 0)) * H + h) * DV + scol;
#pragma unroll
            for (int c16 = 0; c16 < CPT; c16 += 16) {
                float o[16];
                tmem_ld16(tmem + lane_base + L::TM_D1 + (n & 1) * VS + cg * CPT + c16, o);
                tmem_wait_ld();
                if (t < geo.len && !trans && KDA_CHECK(prm.st, geo.row0 + t < rows && scol + c16 + 16 <= DV)) {
                    float a8[8], b8[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) { a8[e] = prm.scale * o[e]; b8[e] = prm.scale * o[8 + e]; }
                    *reinterpret_cast<uint4 *>(dst + c16) = pack8_bf16(a8);
                    *reinterpret_cast<uint4 *>(dst + c16 + 8) = pack8_bf16(b8);
                }
            }
            tc_fence_before();
        };

        bool ok = *s_abort == 0 && nseg > 0;
        if (ok) {
            store_state_bf16();
            arrive(B_S0);
            load_v(0);
            build_vt();
            arrive(B_VT);
            if (nseg > 1) load_v(1);
        }
        for (int n = 0; ok && n < nseg; ++n) {
            const bool more = n + 1 < nseg;
            if (!(ok = wait_warp(B_M1, (uint32_t)(n & 1)))) break;  // U(n), D1[n&1] rows 0..63
            tc_fence_after();
            if (lq < 2) {  // Vnew(n) = U - W S0 -> Vnew tile n & 1
                uint8_t *vn = sm + L::OFF_VN + (n & 1) * VS * 128;
#pragma unroll
                for (int c16 = 0; c16 < CPT; c16 += 16) {
                    float u[16], w[16];
                    tmem_ld16(tmem + lane_base + L::TM_U + cg * CPT + c16, u);
                    tmem_ld16(tmem + lane_base + L::TM_D1 + (n & 1) * VS + cg * CPT + c16, w);
                    tmem_wait_ld();
                    float a8[8], b8[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) { a8[e] = u[e] - w[e]; b8[e] = u[8 + e] - w[8 + e]; }
                    *reinterpret_cast<uint4 *>(vn + mnmaj<128, 2>(ch, cg * CPT + c16, CH)) = pack8_f16(a8);
                    *reinterpret_cast<uint4 *>(vn + mnmaj<128, 2>(ch, cg * CPT + c16 + 8, CH)) = pack8_f16(b8);
                }
                fence_async_smem();
                tc_fence_before();
                arrive(B_VN0 + (n & 1));
            } else if (n >= 1) {  // output of chunk n-1 once 3b(n-1) is done
                if (!(ok = wait_warp(B_MB, (uint32_t)((n - 1) & 1)))) break;
                tc_fence_after();
                write_output(n - 1);
                arrive(B_OUT0 + ((n - 1) & 1));
            }
            if (more) {  // V^T is free: U(n) completed before product 1(n)
                build_vt();
                arrive(B_VT);
            }
            // state update, S = e^{Gamma_C} S0 + K-hat^T Vnew
            if (!(ok = wait_warp(B_M3, (uint32_t)(n & 1)))) break;
            if (!(ok = wait_warp(B_K0 + (n & 1), (uint32_t)((n >> 1) & 1)))) break;  // e^{Gamma_C}(n) arrived
            tc_fence_after();
            if (ch < DK) {  // warp-uniform
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
            if (n + 2 < nseg) arrive(B_KE0 + (n & 1));  // e^{Gamma_C}(n) read, 3a(n) done
            store_state_bf16();  // S0 is free: product 1(n) completed
            tc_fence_before();
            arrive(B_S0);
            // The values of chunk n + 2, for V^T(n + 2) in the next iteration.  Issued
            // here, not before the state update: global loads in flight there delayed its
            // TMEM load (median 870 -> 270 cycles, chunk period 5.2k -> 4.6k cycles).
            if (n + 2 < nseg) load_v(n + 2);
        }
        if (ok && lq >= 2) {  // the last chunk's output
            if ((ok = wait_warp(B_MB, (uint32_t)((nseg - 1) & 1)))) {
                tc_fence_after();
                write_output(nseg - 1);
            }
        }
        // an empty sequence passes its state through (h0, or zero) once
        const bool write_state = nseg > 0 ? ok : (geo.first && geo.last);
        if (write_state && *s_abort == 0 && s_out != nullptr && ch < DK && slice_in) {
            float4 *dst = reinterpret_cast<float4 *>(s_out + (size_t)ch * s_ld + scol);
#pragma unroll
            for (int e = 0; e < CPT / 4; ++e) dst[e] = make_float4(S[4 * e], S[4 * e + 1], S[4 * e + 2], S[4 * e + 3]);
        }
    }
    __syncwarp();  // the idle lanes of the loader and issuer warps wait for lane 0
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, L::TM_COLS);
    if (tid == 0) stamp_end(prm.stamp);
}

template <int DK, int VS>
static cudaError_t launch_chain_t(const CUtensorMap *maps, const ChainParams &prm, cudaStream_t stream,
                                  cudaEvent_t started) {
    using L = ChainLayout<DK, VS>;
    cudaError_t e = cudaFuncSetAttribute(chain_kernel<DK, VS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         L::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(prm.gm.nseqs * prm.H * prm.nparts * prm.slots);
    cfg.blockDim = dim3(CHAIN_THREADS);
    cfg.dynamicSmemBytes = L::SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    if (started != nullptr) {
        attr[0].id = cudaLaunchAttributeLaunchCompletionEvent;
        attr[0].val.launchCompletionEvent.event = started;
        attr[0].val.launchCompletionEvent.flags = 0;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    return cudaLaunchKernelEx(&cfg, chain_kernel<DK, VS>, maps[0], maps[1], maps[2], maps[3], prm);
}

// maps: the record parts WQ, P, K-hat, T' (see chunk_common.cuh); the value
// slice of a CTA is DV / nslices columns (64 or 128).  `started`, when given,
// is recorded once every CTA of the launch has begun (a launch-completion
// event; the runtime may fire it later, at the kernel's end).
cudaError_t launch_chain(const CUtensorMap *maps, const ChainParams &prm, int dk, cudaStream_t stream,
                         cudaEvent_t started) {
    const int vs = prm.DV / prm.nslices;
    if (dk == 128)
        return vs == 128 ? launch_chain_t<128, 128>(maps, prm, stream, started)
                         : launch_chain_t<128, 64>(maps, prm, stream, started);
    return vs == 128 ? launch_chain_t<64, 128>(maps, prm, stream, started)
                     : launch_chain_t<64, 64>(maps, prm, stream, started);
}

}  // namespace kda
