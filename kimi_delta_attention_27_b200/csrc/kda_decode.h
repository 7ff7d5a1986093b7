// Internal interface between the C-ABI front end and the decode-step kernel.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace kda {

// One recurrent step for a batch of (request, head) pairs (kda_decode.cu).
struct DecodeParams {
    const uint16_t *q, *k, *v;  // bf16 bits, [units, 128]
    const float *g;             // [units, 128]
    const float *beta;          // [units]
    float scale;
    const void *state_in;       // [units, 128, 128] or nullptr (zero state)
    void *state_out;            // [units, 128, 128] or nullptr (not written); may equal state_in
    int32_t state_fp32;         // 1: fp32 states, 0: bf16
    uint16_t *out;              // bf16 [units, 128]
};
cudaError_t launch_decode(const DecodeParams &p, int64_t units, cudaStream_t stream);

}  // namespace kda
