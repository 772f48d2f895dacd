// chunk_params.cuh -- launch parameters of the chunkwise prefill kernel,
// shared by the kernel (chunk_fwd.cu) and the C ABI (kda_api.cu).
#pragma once
#include <stdint.h>

#include "kda_device.cuh"

namespace kda {

struct ChunkParams {
    const float *beta;   // [B, T, H]
    const float *h0;     // [B, H, dk, dv] or NULL
    uint16_t *out;       // bf16 [B, T, H, dv]
    float *hT;           // [B, H, dk, dv] or NULL
    float scale;
    int B, T, H, DV, nslices;
    DeviceStatus st;
    uint64_t inject_wait_polls;  // test hook: nonzero = first wait on a barrier nothing signals
};

}  // namespace kda
