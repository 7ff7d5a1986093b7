// Internal interface between the C-ABI front end and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace kda {

constexpr int kHeadDim = 128;  // K = V = 128 (the only size the method's library supports)
constexpr int kChunk = 64;     // chunk length C

struct FwdParams {
    const uint16_t *q, *k, *v;  // bf16 bits, [rows, H, 128]
    const float *g;             // [rows, H, 128]
    const float *beta;          // [rows, H]
    float scale;
    const int32_t *cu_seqlens;  // device, or nullptr (fixed-length rows)
    int64_t seq_len;            // tokens per batch row (or packed total)
    int32_t num_seqs;           // sequences (batch rows, or varlen count)
    int32_t num_heads;
    const void *h0;             // [num_seqs, H, 128, 128] or nullptr
    int32_t h0_fp32;            // 1: fp32, 0: bf16
    void *hT;                   // [num_seqs, H, 128, 128] or nullptr
    int32_t hT_fp32;
    uint16_t *out;              // bf16 [rows, H, 128]
};

// First, straightforward CUDA-core path (fp32 arithmetic throughout).
cudaError_t launch_fwd_simt(const FwdParams &p, cudaStream_t stream);

}  // namespace kda
