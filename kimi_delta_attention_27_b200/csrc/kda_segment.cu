// kda_segment.cu -- the scan step of the segment-parallel forward.
//
// The recurrence of the Kimi Linear feature page (chapter 4, state-update equation) is
// affine in the state: a run over a piece of a sequence maps its entering state to
// S_out = M S_in + B, where M (128 x 128, key by key) is the final state of the same run
// started from the identity with v = 0, and B the final state of the run started from
// zero. With M and B of every piece (computed by the forward kernel in its affine mode,
// all pieces at once), the states entering the pieces follow from the row's initial
// state by the scan below; a second forward run from those states gives every output.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kda_internal.h"

namespace kda {
namespace {

constexpr int D = kHeadDim;
constexpr int kCols = 16;                 // state columns per CTA
constexpr int kThreads = 256;             // 128 rows x 2 threads, 8 columns each

// grid (rows * H, D / kCols): CTA (b h, cb) scans columns [16 cb, 16 cb + 16) of the state of
// row b, head h, over its pieces: the columns of S_out = M S_in + B depend on the same
// columns of S_in only.
__global__ void __launch_bounds__(kThreads)
    kda_segment_scan_kernel(const void *h0, int h0_fp32, const float *M, const float *B, float *S_in,
                            int seg_count, int H) {
    __shared__ __align__(16) float S[D][kCols];
    const int b = blockIdx.x / H, h = blockIdx.x % H;
    const int c_base = blockIdx.y * kCols;
    const int t = threadIdx.x, i = t >> 1, c0 = (t & 1) * 8;   // row i, columns c0 .. c0 + 7
    {
        const size_t base = (static_cast<size_t>(b) * H + h) * D * D + static_cast<size_t>(i) * D + c_base + c0;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            float x = 0.f;
            if (h0) {
                if (h0_fp32) {
                    x = static_cast<const float *>(h0)[base + c];
                } else {
                    const uint16_t bits = static_cast<const uint16_t *>(h0)[base + c];
                    x = __uint_as_float(static_cast<uint32_t>(bits) << 16);
                }
            }
            S[i][c0 + c] = x;
        }
    }
    __syncthreads();
    for (int j = 0; j < seg_count; ++j) {
        const size_t unit = static_cast<size_t>(b) * seg_count + j;
        const size_t base = (unit * H + h) * D * D;
        const size_t my = base + static_cast<size_t>(i) * D + c_base + c0;
        float acc[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            S_in[my + c] = S[i][c0 + c];
            acc[c] = 0.f;
        }
        if (j + 1 == seg_count) break;   // the state leaving the last piece is not needed here
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[c] = B[my + c];
        const float4 *mrow = reinterpret_cast<const float4 *>(M + base + static_cast<size_t>(i) * D);
#pragma unroll 4
        for (int k4 = 0; k4 < D / 4; ++k4) {
            const float4 m = mrow[k4];
            const float mk[4] = {m.x, m.y, m.z, m.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float4 s0 = *reinterpret_cast<const float4 *>(&S[4 * k4 + e][c0]);
                const float4 s1 = *reinterpret_cast<const float4 *>(&S[4 * k4 + e][c0 + 4]);
                acc[0] = fmaf(mk[e], s0.x, acc[0]);
                acc[1] = fmaf(mk[e], s0.y, acc[1]);
                acc[2] = fmaf(mk[e], s0.z, acc[2]);
                acc[3] = fmaf(mk[e], s0.w, acc[3]);
                acc[4] = fmaf(mk[e], s1.x, acc[4]);
                acc[5] = fmaf(mk[e], s1.y, acc[5]);
                acc[6] = fmaf(mk[e], s1.z, acc[6]);
                acc[7] = fmaf(mk[e], s1.w, acc[7]);
            }
        }
        __syncthreads();
#pragma unroll
        for (int c = 0; c < 8; ++c) S[i][c0 + c] = acc[c];
        __syncthreads();
    }
}

}  // namespace

cudaError_t launch_segment_scan(const void *h0, int h0_fp32, const float *M, const float *B, float *S_in,
                                int32_t rows, int32_t seg_count, int32_t num_heads, cudaStream_t stream) {
    if (rows <= 0 || seg_count <= 0) return cudaSuccess;
    const int64_t bh = static_cast<int64_t>(rows) * num_heads;
    if (bh > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    kda_segment_scan_kernel<<<dim3(static_cast<unsigned>(bh), D / kCols), kThreads, 0, stream>>>(
        h0, h0_fp32, M, B, S_in, seg_count, num_heads);
    return cudaGetLastError();
}

}  // namespace kda
