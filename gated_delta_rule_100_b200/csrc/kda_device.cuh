// kda_device.cuh -- sm_100a device helpers shared by the libkda kernels:
// bounded mbarrier waits, TMA tile loads, tcgen05 (TMEM + UMMA) wrappers,
// shared-memory matrix descriptors and the canonical swizzled layouts.
//
// Layout vocabulary (all offsets in bytes, relative to a 1024-byte aligned
// base, swizzle applied with swz<SWB>):
//   K-major  [R rows][K]  : K split into blocks of SWB/ES elements; block kb
//                           holds rows 0..R-1 at kb*R*SWB + r*SWB.
//   MN-major [K rows][N]  : N split into blocks of SWB/ES elements; block nb
//                           holds K-rows 0..K-1 at nb*K*SWB + k*SWB.
// These are the canonical UMMA layouts (8-row swizzle atoms of 8*SWB bytes).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace kda {

// ---------------------------------------------------------------- status ----
// Bit flags OR-ed into the per-device status word by kernels.
enum : uint32_t { DEV_TIMEOUT = 1u, DEV_BAD_ARG = 2u, DEV_BOUNDS = 4u };

struct DeviceStatus {
    uint32_t *word;        // device-global status word (never NULL at launch)
    uint64_t wait_polls;   // polls a bounded wait makes before giving up
};

__device__ __forceinline__ void report(const DeviceStatus &st, uint32_t bits) {
    atomicOr(st.word, bits);
}

// Index checks of the debug build (KDA_DEBUG, libkda_debug.so): before an
// access whose bounds follow from layout constants and launch geometry rather
// than from the code in front of it, KDA_CHECK(st, cond) tests the bound; a
// failed check records DEV_BOUNDS in the status word and the caller skips the
// access (no trap).  In the release build it is the constant true.
__device__ __forceinline__ bool bounds_ok(const DeviceStatus &st, bool ok) {
    if (!ok) report(st, DEV_BOUNDS);
    return ok;
}
#ifdef KDA_DEBUG
#define KDA_CHECK(st, cond) ::kda::bounds_ok((st), (cond))
#else
#define KDA_CHECK(st, cond) true
#endif

// ------------------------------------------------------------- addressing ----
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

template <int SWB>
__device__ __forceinline__ uint32_t swz(uint32_t L) {
    static_assert(SWB == 32 || SWB == 64 || SWB == 128, "swizzle width");
    constexpr uint32_t B = SWB == 128 ? 3u : (SWB == 64 ? 2u : 1u);
    constexpr uint32_t mask = ((1u << B) - 1u) << 7;
    return L ^ ((L & mask) >> 3);
}

// Byte offset of element (r, k) of a K-major [R][K] operand.
template <int SWB, int ES>
__device__ __forceinline__ uint32_t kmaj(int r, int k, int R) {
    constexpr int KB = SWB / ES;
    return swz<SWB>((uint32_t)((k / KB) * R * SWB + r * SWB + (k % KB) * ES));
}

// Byte offset of element (k, n) of an MN-major [K][N] operand.
template <int SWB, int ES>
__device__ __forceinline__ uint32_t mnmaj(int k, int n, int K) {
    constexpr int NB = SWB / ES;
    return swz<SWB>((uint32_t)((n / NB) * K * SWB + k * SWB + (n % NB) * ES));
}

template <int SWB>
__device__ __forceinline__ constexpr uint64_t layout_code() {
    return SWB == 128 ? 2ull : (SWB == 64 ? 4ull : 6ull);
}

// UMMA shared-memory matrix descriptor (sm_100 format, version 1).
template <int SWB>
__device__ __forceinline__ uint64_t make_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= 1ull << 46;
    d |= layout_code<SWB>() << 61;
    return d;
}

// Byte offset of element (r, k) of a K-major operand whose K-blocks sit
// `kb_stride` bytes apart (kb_stride = R * SWB gives the plain layout; a
// smaller stride lets the unused rows of one K-block overlap the next).
template <int SWB, int ES>
__device__ __forceinline__ uint32_t kmaj_s(int r, int k, int kb_stride) {
    constexpr int KB = SWB / ES;
    return swz<SWB>((uint32_t)((k / KB) * kb_stride + r * SWB + (k % KB) * ES));
}

template <int SWB, int ES>
__device__ __forceinline__ uint64_t desc_kmaj_s(uint32_t base, int kb_stride, int k0) {
    constexpr int KB = SWB / ES;
    uint32_t a = base + (uint32_t)((k0 / KB) * kb_stride + (k0 % KB) * ES);
    return make_desc<SWB>(a, 16u, 8u * SWB);
}

// Descriptor of the K-step starting at element k0 of a K-major [R][K] operand.
template <int SWB, int ES>
__device__ __forceinline__ uint64_t desc_kmaj(uint32_t base, int R, int k0) {
    constexpr int KB = SWB / ES;
    uint32_t a = base + (uint32_t)((k0 / KB) * R * SWB + (k0 % KB) * ES);
    return make_desc<SWB>(a, 16u, 8u * SWB);
}

// Descriptor of the K-step starting at K-row k0 of an MN-major [K][N] operand.
template <int SWB>
__device__ __forceinline__ uint64_t desc_mnmaj(uint32_t base, int K, int k0) {
    uint32_t a = base + (uint32_t)(k0 * SWB);
    return make_desc<SWB>(a, (uint32_t)(K * SWB), 8u * SWB);
}

// UMMA instruction descriptor: fp32 accumulate, dense.
// fmt: 0 = f16, 1 = bf16 (kind::f16); 2 = tf32 (kind::tf32).
__host__ __device__ constexpr uint32_t make_idesc(int fmt, bool a_mn, bool b_mn, int M, int N) {
    return (1u << 4) | ((uint32_t)fmt << 7) | ((uint32_t)fmt << 10) |
           ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// --------------------------------------------------------------- mbarrier ----
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// Launch timing (measurement hook): a launch's slot holds {start, ~end}, both
// initialised to all ones; every CTA folds in its own start and end with
// atomicMin, so the slot ends as {first CTA start, ~(last CTA end)}.
__device__ __forceinline__ void stamp_start(unsigned long long *slot) {
    if (slot != nullptr) atomicMin(slot, (unsigned long long)globaltimer_ns());
}
__device__ __forceinline__ void stamp_end(unsigned long long *slot) {
    if (slot != nullptr) atomicMin(slot + 1, ~(unsigned long long)globaltimer_ns());
}

// Longest a bounded wait polls before giving up, whatever the poll budget.
constexpr uint64_t WAIT_TIMEOUT_NS = 1000000000ull;

// Bounded wait for phase `parity` of the mbarrier.  Gives up after `polls`
// failed try_wait calls or about one second, whichever comes first, records
// DEV_TIMEOUT in the status word and returns false.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint64_t polls,
                                          const DeviceStatus &st) {
    if (mbar_try(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint64_t i = 1; i < polls; ++i) {
        if (mbar_try(bar, parity)) return true;
        if ((i & 255u) == 0 && globaltimer_ns() - t0 > WAIT_TIMEOUT_NS) break;
    }
    report(st, DEV_TIMEOUT);
    return false;
}

// -------------------------------------------------------------------- TMA ----
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap *map, uint32_t bar,
                                            int c0, int c1, int c2, int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *map, uint32_t bar, int c0, int c1,
                                            int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

// 1-D bulk copy global -> shared (both 16-byte aligned, size a multiple of 16).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
        : "memory");
}

// Prefetch `bytes` (a multiple of 16, 16-byte aligned) of global memory into L2.
__device__ __forceinline__ void prefetch_l2(const void *src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<uint64_t>(src)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------- tcgen05 ----
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]; issued by one thread.
template <int KIND>  // 0 = kind::f16, 1 = kind::tf32
__device__ __forceinline__ void umma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                     uint32_t accumulate) {
    if constexpr (KIND == 0) {
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
            "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
            : "memory");
    } else {
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
            "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
            : "memory");
    }
}

// Arrive on `bar` once every tcgen05.mma issued so far by this thread completed.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     bar)
                 : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 32 lanes x 16 consecutive 32-bit columns: thread t of the warp receives
// lane (warp's quarter * 32 + t), columns [col, col + 16).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// 32 lanes x 8 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8]) {
    uint32_t r[8];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                   "=r"(r[7])
                 : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

// ------------------------------------------------------------ gate prologue ----
// Raw projections in: log-decay g = -c softplus(x), with softplus(x) =
// log(1 + e^x) written as max(x, 0) + log(1 + e^-|x|) so that it never
// overflows, and beta = sigmoid(x).  The logarithm's argument lies in (1, 2],
// where the fast __logf is accurate to a few 1e-7 absolute; an e^-|x| below
// 2^-24 (|x| > 16.6) is lost in 1 + e^-|x|, which changes g by less than
// c * 6e-8, negligible for alpha = e^g.  (An accurate log1pf here made the
// prologue's prep ~45% slower.)
__device__ __forceinline__ float gate_logdecay(float x, float c) {
    return -c * (fmaxf(x, 0.f) + __logf(1.f + __expf(-fabsf(x))));
}
__device__ __forceinline__ float gate_sigmoid(float x) { return 1.f / (1.f + __expf(-x)); }

// ------------------------------------------------------------ conversions ----
// fp32 -> tf32 bit pattern, rounded to nearest (ties away), stored in 32 bits.
__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ uint16_t to_bf16_bits(float x) {
    __nv_bfloat16 h = __float2bfloat16_rn(x);
    return *reinterpret_cast<uint16_t *>(&h);
}

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) {
    return __uint_as_float(((uint32_t)b) << 16);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);  // one cvt.rn.bf16x2.f32
    return *reinterpret_cast<const uint32_t *>(&h);
}

}  // namespace kda
