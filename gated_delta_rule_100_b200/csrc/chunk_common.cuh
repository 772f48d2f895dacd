// chunk_common.cuh -- constants, the per-chunk record layout and small helpers
// shared by the two prefill kernels (prep_fwd.cu, chain_fwd.cu).
//
// The chunkwise prefill is split in two:
//   prep  (one CTA per (b, h, chunk), no dependence between chunks): builds the
//         decay-scaled operands, the intra-chunk blocks A and P, T = (I + A)^-1
//         and W = T Diag(beta) (K * e^Gamma), and writes one record per chunk;
//   chain (one CTA per (b, h), chunks in order): U = T Diag(beta) V, then the
//         state pass Vnew = U - W S, S <- e^{Gamma_C} S + K-hat^T Vnew and the
//         outputs (Q e^Gamma) S + P Vnew.
// A record holds these arrays (the chain kernel's tensor loads apply the UMMA
// operand swizzle).  The first three are cut into 16-token blocks, each block a
// row-major array of 32-byte rows, so that the prep kernel's warps, which hold
// 16 consecutive tokens of 32 consecutive rows per thread, write them as
// contiguous 1 KB runs:
//   WQ   bf16 [8][dk][16]   [W; Q e^Gamma] over tokens m = 16 blk + e (blocks
//                           0..3 = W, 4..7 = Q e^Gamma), row = key channel
//   P    fp16 [4][64][16]   causal q-k block (incl. diagonal): [J][i][e] = P[i][16 J + e]
//   KH   fp16 [4][128][16]  K-hat^T: [I][c][e] = K-hat[16 I + e][c]
//   T'   fp32 [64][64]      T' = T Diag(beta), unit-lower times beta, row-major
//   DEC  fp32 [128]         e^{Gamma_C} per key channel
// at the offsets below (each 16-byte aligned; 72.5 KB per record).
#pragma once
#include <cuda_fp16.h>
#include <stdint.h>

#include "kda_device.cuh"

namespace kda {

constexpr int CH = 64;          // chunk length
constexpr int SUB = 16;         // sub-block of the decay references
constexpr int NSUB = CH / SUB;  // 4
constexpr int A_LD = 68;        // fp32 row stride of the A / T scratch
constexpr float EXP_CLAMP_HI = 5.5406223843935098e34f;  // e^80
constexpr float EXP_CLAMP_LO = 1.8048513878454153e-35f; // e^-80
constexpr float MILD_DEC_LO = 4.2483542552915889e-18f;   // e^-40: least e^{Gamma_C} of a mild chunk

constexpr int REC_WQ = 0;         // 32 KB (dk = 64 uses the first 16 KB)
constexpr int REC_P = 32768;      // 8 KB
constexpr int REC_KH = 40960;     // 16 KB
constexpr int REC_T = 57344;      // 16 KB
constexpr int REC_DEC = 73728;    // 512 B
constexpr int REC_BYTES = 74240;

__host__ __device__ constexpr int align1k(int x) { return (x + 1023) & ~1023; }
__host__ __device__ constexpr int cmax(int a, int b) { return a > b ? a : b; }

// First TMEM column / Y row of block I's formation product: 16 * I (I + 1) / 2.
__device__ __forceinline__ constexpr int yoff(int I) { return SUB * (I * (I + 1) / 2); }

__device__ __forceinline__ float rcp_clamped(float p) {
    return p < EXP_CLAMP_LO ? EXP_CLAMP_HI : __fdividef(1.0f, p);
}

// fp16 keeps tf32's 10-bit mantissa (rounded to nearest) in half the bytes;
// the values stored as fp16 are bounded by |q| |k| and |k| (P, K-hat) or by
// the values' and the state's magnitudes (Vnew).
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    const __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}

__device__ __forceinline__ uint4 pack8_f16(const float (&v)[8]) {
    return make_uint4(pack_f16x2(v[0], v[1]), pack_f16x2(v[2], v[3]), pack_f16x2(v[4], v[5]),
                      pack_f16x2(v[6], v[7]));
}

__device__ __forceinline__ uint16_t f16_bits(float x) {
    const __half h = __float2half_rn(x);
    return *reinterpret_cast<const uint16_t *>(&h);
}

__device__ __forceinline__ uint4 pack8_bf16(const float (&v)[8]) {
    return make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                      pack_bf16x2(v[6], v[7]));
}

// tf32 operands are stored as fp32 bit patterns: the tensor core reads the
// sign, exponent and top 10 mantissa bits (the conversion instruction runs at
// a sixteenth of the FMA rate, so it is skipped).
__device__ __forceinline__ uint32_t tf32_bits(float x) { return __float_as_uint(x); }

__device__ __forceinline__ uint4 pack4_tf32(float a, float b, float c, float d) {
    return make_uint4(tf32_bits(a), tf32_bits(b), tf32_bits(c), tf32_bits(d));
}

}  // namespace kda
