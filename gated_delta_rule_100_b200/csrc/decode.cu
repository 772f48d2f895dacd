// decode.cu -- one recurrent KDA step per (b, h), state updated in place.
//
// For each column j of the fp32 state S (dk x dv):
//   s'  = alpha .* S[:, j]                 (decay first)
//   p_j = k . s'                           (what the memory returns for k)
//   u_j = beta (v_j - p_j)                 (erase along k, then write v)
//   S[:, j] = s' + k u_j
//   o_j = scale (q . s' + (q . k) u_j)     (read after the write)
// which is the combined update of "Kimi Linear's Hybrid Linear Attention
// Architecture: A Technical Breakdown", section 3.3, for one token.
//
// The step is HBM-bound: the state (4 dk dv bytes per head) is read and
// written once.  One CTA owns one (b, h): 256 threads tile the state as
// (row groups) x (dv / 4 float4 column groups), so every warp-wide load or
// store covers one contiguous 512-byte state row.  The two column reductions
// (k.s' and q.s') go through shared memory across row groups.  The gate is
// either one log-decay per key channel (g [B, H, dk]) or one per head shared by
// all channels (g [B, H], the scalar-gate form): g_dk = dk or 1.  With the
// gate prologue the inputs are raw projections (see gate_logdecay): the kernel
// forms g and beta and L2-normalises q and k itself.
#include <cuda_bf16.h>
#include <stdint.h>

#include "kda_device.cuh"

namespace kda {

constexpr int DEC_THREADS = 256;

// PRO: the gate prologue (raw g, beta, q, k), a separate instantiation so that
// the plain kernel carries none of it.
template <int DK, int DV, bool PRO>
__global__ void __launch_bounds__(DEC_THREADS)
decode_step_kernel(const uint16_t *__restrict__ q, const uint16_t *__restrict__ k,
                   const uint16_t *__restrict__ v, const float *__restrict__ g,
                   const float *__restrict__ beta, float scale, float *__restrict__ state,
                   uint16_t *__restrict__ out, int g_dk, float gate_c) {
    constexpr int NCG = DV / 4;              // float4 column groups
    constexpr int NRG = DEC_THREADS / NCG;   // row groups
    constexpr int RPT = DK / NRG;            // state rows per thread
    static_assert(DK % NRG == 0 && NCG <= 32, "tile shape");

    __shared__ float s_k[DK], s_q[DK], s_a[DK];
    __shared__ float s_red[2][NRG][DV];
    __shared__ float s_qk;
    __shared__ float s_nrm[2][DK / 32];  // PRO: per-warp partial sums of q^2, k^2

    const int bh = blockIdx.x;
    const int tid = threadIdx.x;
    const int cg = tid % NCG;   // column group
    const int rg = tid / NCG;   // row group

    const uint16_t *qh = q + (size_t)bh * DK;
    const uint16_t *kh = k + (size_t)bh * DK;
    const float *gh = g + (size_t)bh * g_dk;
    float *S = state + (size_t)bh * DK * DV;

    // Issue the state loads first: they are the long-latency part.
    float4 s[RPT];
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const int r = rg * RPT + i;
        s[i] = __ldcs(reinterpret_cast<const float4 *>(S + (size_t)r * DV) + cg);
    }
    static_assert(DK <= DEC_THREADS, "one thread per key channel");
    float kq = 0.f, qq = 0.f;  // PRO: this thread's raw k and q values
    if (tid < DK) {
        kq = bf16_bits_to_f32(kh[tid]);
        qq = bf16_bits_to_f32(qh[tid]);
        const float gr = gh[g_dk > 1 ? tid : 0];
        s_a[tid] = __expf(PRO ? gate_logdecay(gr, gate_c) : gr);
        if constexpr (PRO) {  // raw q, k: the sums of squares of the L2 norms, per warp
            float sk = kq * kq, sq = qq * qq;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                sk += __shfl_xor_sync(0xffffffffu, sk, o);
                sq += __shfl_xor_sync(0xffffffffu, sq, o);
            }
            if ((tid & 31) == 0) { s_nrm[0][tid >> 5] = sq; s_nrm[1][tid >> 5] = sk; }
        } else {
            s_k[tid] = kq;
            s_q[tid] = qq;
        }
    }
    if constexpr (PRO) {  // normalised q, k rounded to bf16 again, as the prefill's prologue
        __syncthreads();
        if (tid < DK) {
            float sq = 0.f, sk = 0.f;
#pragma unroll
            for (int w = 0; w < DK / 32; ++w) { sq += s_nrm[0][w]; sk += s_nrm[1][w]; }
            s_q[tid] = bf16_bits_to_f32(to_bf16_bits(qq * rsqrtf(fmaxf(sq, 1e-24f))));
            s_k[tid] = bf16_bits_to_f32(to_bf16_bits(kq * rsqrtf(fmaxf(sk, 1e-24f))));
        }
    }
    __syncthreads();
    if (tid < 32) {
        float acc = 0.f;
        for (int r = tid; r < DK; r += 32) acc += s_q[r] * s_k[r];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (tid == 0) s_qk = acc;
    }

    float4 pk = make_float4(0.f, 0.f, 0.f, 0.f), pq = pk;
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const int r = rg * RPT + i;
        const float a = s_a[r], kr = s_k[r], qr = s_q[r];
        s[i].x *= a; s[i].y *= a; s[i].z *= a; s[i].w *= a;
        pk.x += kr * s[i].x; pk.y += kr * s[i].y; pk.z += kr * s[i].z; pk.w += kr * s[i].w;
        pq.x += qr * s[i].x; pq.y += qr * s[i].y; pq.z += qr * s[i].z; pq.w += qr * s[i].w;
    }
    reinterpret_cast<float4 *>(&s_red[0][rg][0])[cg] = pk;
    reinterpret_cast<float4 *>(&s_red[1][rg][0])[cg] = pq;
    __syncthreads();

    // Column totals: every thread needs u for its own 4 columns.
    float4 p = make_float4(0.f, 0.f, 0.f, 0.f), y = p;
#pragma unroll
    for (int j = 0; j < NRG; ++j) {
        const float4 a = reinterpret_cast<const float4 *>(&s_red[0][j][0])[cg];
        const float4 b = reinterpret_cast<const float4 *>(&s_red[1][j][0])[cg];
        p.x += a.x; p.y += a.y; p.z += a.z; p.w += a.w;
        y.x += b.x; y.y += b.y; y.z += b.z; y.w += b.w;
    }
    const float bt = PRO ? gate_sigmoid(beta[bh]) : beta[bh];
    const uint16_t *vh = v + (size_t)bh * DV + cg * 4;
    float4 u;
    u.x = bt * (bf16_bits_to_f32(vh[0]) - p.x);
    u.y = bt * (bf16_bits_to_f32(vh[1]) - p.y);
    u.z = bt * (bf16_bits_to_f32(vh[2]) - p.z);
    u.w = bt * (bf16_bits_to_f32(vh[3]) - p.w);

#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const int r = rg * RPT + i;
        const float kr = s_k[r];
        float4 o = s[i];
        o.x += kr * u.x; o.y += kr * u.y; o.z += kr * u.z; o.w += kr * u.w;
        __stcs(reinterpret_cast<float4 *>(S + (size_t)r * DV) + cg, o);
    }

    if (rg == 0) {
        const float qk = s_qk;
        uint2 pk2;
        pk2.x = pack_bf16x2(scale * (y.x + qk * u.x), scale * (y.y + qk * u.y));
        pk2.y = pack_bf16x2(scale * (y.z + qk * u.z), scale * (y.w + qk * u.w));
        *reinterpret_cast<uint2 *>(out + (size_t)bh * DV + cg * 4) = pk2;
    }
}

template <int DK, int DV>
static cudaError_t launch_decode_t(const void *q, const void *k, const void *v, const float *g,
                                   const float *beta, float scale, float *state, void *out,
                                   int BH, int g_dk, int prologue, float gate_c, cudaStream_t stream) {
    if (prologue)
        decode_step_kernel<DK, DV, true><<<BH, DEC_THREADS, 0, stream>>>(
            (const uint16_t *)q, (const uint16_t *)k, (const uint16_t *)v, g, beta, scale, state,
            (uint16_t *)out, g_dk, gate_c);
    else
        decode_step_kernel<DK, DV, false><<<BH, DEC_THREADS, 0, stream>>>(
            (const uint16_t *)q, (const uint16_t *)k, (const uint16_t *)v, g, beta, scale, state,
            (uint16_t *)out, g_dk, gate_c);
    return cudaGetLastError();
}

// prologue != 0: g, beta, q and k are raw (g = -gate_c softplus(g), beta = sigmoid(beta),
// q and k L2-normalised).
cudaError_t launch_decode(const void *q, const void *k, const void *v, const float *g,
                          const float *beta, float scale, float *state, void *out, int BH, int dk,
                          int dv, int g_dk, int prologue, float gate_c, cudaStream_t stream) {
    if (dk == 128 && dv == 128)
        return launch_decode_t<128, 128>(q, k, v, g, beta, scale, state, out, BH, g_dk, prologue, gate_c, stream);
    if (dk == 128 && dv == 64)
        return launch_decode_t<128, 64>(q, k, v, g, beta, scale, state, out, BH, g_dk, prologue, gate_c, stream);
    if (dk == 64 && dv == 128)
        return launch_decode_t<64, 128>(q, k, v, g, beta, scale, state, out, BH, g_dk, prologue, gate_c, stream);
    return launch_decode_t<64, 64>(q, k, v, g, beta, scale, state, out, BH, g_dk, prologue, gate_c, stream);
}

}  // namespace kda
