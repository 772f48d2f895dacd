// chunk_params.cuh -- launch parameters of the two prefill kernels, shared by
// the kernels (prep_fwd.cu, chain_fwd.cu) and the C ABI (kda_api.cu).
#pragma once
#include <stdint.h>

#include "kda_device.cuh"

namespace kda {

// Items (b, h, chunk) of chunks [n_begin, n_begin + nseg), claimed by persistent CTAs.
struct PrepParams {
    const float *g;      // [B, T, H, g_dk]
    int g_dk;            // gate values per (token, head): dk (per key channel) or 1 (one, broadcast)
    const float *beta;   // [B, T, H]
    uint8_t *ws;         // records [B*H][nseg][REC_BYTES]
    int *ticket;         // item counter, zero at launch: CTAs claim items from it
    int B, T, H, n_begin, nseg;
    DeviceStatus st;
};

// One CTA per (b, h, value slice); walks chunks [n_begin, n_begin + nseg) in order.
struct ChainParams {
    const uint16_t *v;   // bf16 [B, T, H, dv]
    const float *h0;     // [B, H, dk, dv] or NULL (state at chunk n_begin)
    uint16_t *out;       // bf16 [B, T, H, dv]
    float *hT;           // [B, H, dk, dv] or NULL (state after the last chunk of the segment)
    const uint8_t *ws;   // records written by the prep kernel
    float scale;
    int B, T, H, DV, n_begin, nseg, nslices;
    DeviceStatus st;
    uint64_t inject_wait_polls;  // test hook: nonzero = first wait on a barrier nothing signals
};

}  // namespace kda
