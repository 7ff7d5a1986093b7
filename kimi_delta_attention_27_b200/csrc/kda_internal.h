// Internal interface between the C-ABI front end and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace kda {

constexpr int kHeadDim = 128;  // K = V = 128 (the only size the method's library supports)
constexpr int kChunk = 64;     // chunk length C

// how g is given to the forward kernel
constexpr int kGateF32 = 0;     // log alpha per channel, fp32 [rows, H, 128]
constexpr int kGateBF16 = 1;    // log alpha per channel, bf16 [rows, H, 128]
constexpr int kGateScalar = 2;  // one log alpha per token and head, fp32 [rows, H] (all channels)
// FwdParams::flags
constexpr uint32_t kFlagL2NormQK = 1u;        // q and k are L2-normalised per token and head first
constexpr uint32_t kFlagGateLogsigmoid = 2u;  // g is a pre-activation: log alpha = logsigmoid(g)

struct FwdParams {
    const uint16_t *q, *k, *v;  // bf16 bits, [rows, H, 128]
    const void *g;              // see gate_mode
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
    int32_t gate_mode;          // kGateF32, kGateBF16 or kGateScalar
    uint32_t flags;             // kFlag* bits
    // segmented rows (cu_seqlens == nullptr): seg_len > 0 splits each row of seq_len tokens into
    // seg_count pieces of seg_len tokens; unit s = row * seg_count + piece, and h0 is per unit.
    // A plain run then writes only each row's last piece's final state, into hT per row.
    int64_t seg_len;
    int32_t seg_count;
    int32_t mode;               // kModePlain or kModeAffine
    void *hT_aux;               // kModeAffine: fp32 transition matrices, per unit
};

// kModeAffine runs every unit twice and writes no output: from a zero state (its final state
// to hT, fp32) and from the identity with v = 0 (its final state, the unit's transition
// matrix M with S_out = M S_in + B, to hT_aux); the grid holds 2 x num_seqs x H units.
constexpr int32_t kModePlain = 0, kModeAffine = 1;

// Tensor-core path: one 4-CTA cluster per (sequence, head); `rows` is the
// number of token rows of the packed [rows, H, 128] tensors.
cudaError_t launch_fwd_tc(const FwdParams &p, int64_t rows, cudaStream_t stream);

// Allocation-free variant of launch_fwd_tc: the operand-set rings live in a fixed
// module-scope array, one per cluster, so at most kNoAllocMaxUnits (sequence, head)
// pairs are accepted per call (cudaErrorInvalidValue beyond that).
constexpr int kNoAllocMaxUnits = 32;
cudaError_t launch_fwd_tc_noalloc(const FwdParams &p, int64_t rows, cudaStream_t stream);

// Segment scan over pieces (see FwdParams): for each row b and head h, with S the row's
// initial state (fp32 or bf16, or zero when h0 is null) and M, B the pieces' transition
// matrices and zero-state final states (fp32, per unit), writes S_in[b, j] = the state
// entering piece j: S_in[b, 0] = S, S_in[b, j + 1] = M[b, j] S_in[b, j] + B[b, j].
cudaError_t launch_segment_scan(const void *h0, int h0_fp32, const float *M, const float *B, float *S_in,
                                int32_t rows, int32_t seg_count, int32_t num_heads, cudaStream_t stream);

// Backward pass (kda_bwd.cu): gradients of sum(dout . out) + sum(dhT . hT).
struct BwdParams {
    const uint16_t *q, *k, *v;  // bf16 bits, [rows, H, 128]
    const float *g;             // [rows, H, 128], log alpha
    const float *beta;          // [rows, H]
    float scale;
    const int32_t *cu_seqlens;  // device, or nullptr (fixed-length rows)
    int64_t seq_len;
    int32_t num_seqs;
    int32_t num_heads;
    const void *h0;             // [num_seqs, H, 128, 128] or nullptr
    int32_t h0_fp32;
    const uint16_t *dout;       // bf16 [rows, H, 128]
    const float *dhT;           // [num_seqs, H, 128, 128] or nullptr
    float *dq, *dk, *dv, *dg, *dbeta;  // zeroed by the caller's launch sequence (dq, dk, dg, dbeta)
    float *dh0;                 // [num_seqs, H, 128, 128] or nullptr
    float *workspace;           // checkpoint states, bwd_workspace_bytes
};
size_t bwd_workspace_bytes(int64_t rows, int64_t num_seqs, int32_t num_heads);
cudaError_t launch_bwd(const BwdParams &p, cudaStream_t stream);

// Bits of the device-side error word shared by the library's kernels.
constexpr unsigned int kErrTimeout = 1u;    // a bounded wait gave up; the kernel wound down early
constexpr unsigned int kErrRingIndex = 2u;  // a chain CTA ran on an SM id beyond the ring pool
constexpr unsigned int kErrCuSeqlens = 4u;  // cu_seqlens is not 0, ..., seq_len non-decreasing

// Read and clear the device-side error word.
cudaError_t read_and_clear_device_error(unsigned int *value);

}  // namespace kda
