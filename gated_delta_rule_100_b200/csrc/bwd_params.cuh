// bwd_params.cuh -- launch parameters of the backward pass (bwd.cu), shared
// with the C ABI (kda_api.cu).
#pragma once
#include <stdint.h>

#include "kda_device.cuh"

namespace kda {

struct BwdParams {
    const uint16_t *q, *k, *v;  // bf16 [B, T, H, dk | dk | dv]
    const float *g, *beta;      // [B, T, H, dk], [B, T, H]
    const float *h0;            // [B, H, dk, dv] or NULL
    const uint16_t *dout;       // bf16 [B, T, H, dv] or NULL (zero)
    const float *dhT;           // [B, H, dk, dv] or NULL (zero)
    uint16_t *dq, *dk, *dv;     // bf16 [B, T, H, dk | dk | dv]
    float *dg, *dbeta;          // [B, T, H, dk], [B, T, H]
    float *dh0;                 // [B, H, dk, dv] or NULL
    float *ckpt;                // [B H][ceil(T / 64)][dk][dv] level-1 states, [B H][16][dk][dv] level-2
                                // scratch, then every token's p: [B H][T][dv]
    long long ckpt_elems;       // floats of the ckpt workspace (the debug build's bound)
    float scale;
    int B, T, H;
    DeviceStatus st;            // status word (the debug build's index checks report to it)
    unsigned long long *stamp;  // measurement hook: the launch pair's timing slot, or NULL
};

}  // namespace kda
