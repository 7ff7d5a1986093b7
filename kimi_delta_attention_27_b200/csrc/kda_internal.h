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

// Tensor-core path: one 4-CTA cluster per (sequence, head); `rows` is the
// number of token rows of the packed [rows, H, 128] tensors.
cudaError_t launch_fwd_tc(const FwdParams &p, int64_t rows, cudaStream_t stream);

// Allocation-free variant of launch_fwd_tc: the operand-set rings live in a fixed
// module-scope array, one per cluster, so at most kNoAllocMaxUnits (sequence, head)
// pairs are accepted per call (cudaErrorInvalidValue beyond that).
constexpr int kNoAllocMaxUnits = 32;
cudaError_t launch_fwd_tc_noalloc(const FwdParams &p, int64_t rows, cudaStream_t stream);

// Device-side error word of the tensor-core kernel (bit 0: a bounded wait gave up).
cudaError_t read_and_clear_device_error(unsigned int *value);

}  // namespace kda
