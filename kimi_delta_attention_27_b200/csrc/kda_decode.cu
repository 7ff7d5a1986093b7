// kda_decode.cu -- one recurrent KDA step (a single new token) for a batch of requests, sm_100a.
//
// Method: the state-update equation of the Kimi Linear feature page (chapter 4, "innovation 2")
// applied to one token, in its delta-rule form (chapter 3, delta-rule equation, on the decayed
// state):
//
//   S' = Diag(alpha) S,          alpha = exp(g) per key channel
//   e  = v - S'^T k              retrieval error
//   S  = S' + beta k e^T
//   o  = scale S^T q = scale (S'^T q + beta (k . q) e)
//
// The step is bound by HBM: every (request, head) reads its 128 x 128 state and writes it back,
// against 1.3 KB of token vectors. One CTA per (request, head), 256 threads for fp32 states: warp
// w owns key rows 16w .. 16w + 15, lane l owns value columns 4l .. 4l + 3, so a warp reads and
// writes whole 512-byte state rows with 16-byte accesses, and each thread issues all 16 of its
// state loads before it uses any of them. bf16 states: 128 threads, 32 rows per warp (below). S'^T k and S'^T q are reduced over the
// eight warps in shared memory in one pass; the state is then updated in registers and written
// back. Each state element is read and written by the same thread, so the output state may be
// the input state (in place).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kda_internal.h"
#include "kda_decode.h"

namespace kda {
namespace dec {

constexpr int D = kHeadDim;
constexpr float kLog2e = 1.4426950408889634f;
// threads per CTA: 256 with fp32 states; 128 with bf16 states, which a thread keeps as the loaded
// bf16 pairs (32 rows x 4 columns in 64 registers) and widens where they are used. A bf16 state
// is half the bytes for the same fixed work per CTA, so more CTAs have to be resident per SM.
template <bool kFp32State>
constexpr int threads() { return kFp32State ? 256 : 128; }

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ uint32_t bf_pack(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
}
// 2^y by the hardware approximation (relative error about 2^-22)
__device__ __forceinline__ float ex2(float y) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(y));
    return r;
}

template <bool kFp32State>
__global__ void __launch_bounds__(threads<kFp32State>(), kFp32State ? 2 : 3) kda_decode_kernel(DecodeParams p) {
    constexpr int NT = threads<kFp32State>(), NW = NT / 32, ROWS = D / NW;   // key rows per warp
    __shared__ float ks[D], qs[D], as[D];       // k, q, alpha of this (request, head)
    __shared__ float4 red[NW][2][D / 4];        // per-warp partial S'^T k and S'^T q
    __shared__ float kq_part[NW];
    __shared__ float4 es[D / 4];                // the retrieval error e, from warp 0
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const size_t bh = blockIdx.x;                               // request * num_heads + head
    const size_t vec = bh * D;                                  // offset of this pair's vectors
    const size_t st = bh * static_cast<size_t>(D) * D;          // offset of its state
    const int r0 = warp * ROWS, c0 = lane * 4;

    // state rows of this thread, loaded before anything else so that they are in flight together
    float s[kFp32State ? ROWS : 1][4];
    uint2 raw[kFp32State ? 1 : ROWS];   // bf16 states: the loaded pairs
    if (p.state_in) {
        if constexpr (kFp32State) {
            const float4 *src = reinterpret_cast<const float4 *>(static_cast<const float *>(p.state_in) + st);
#pragma unroll
            for (int r = 0; r < ROWS; ++r) {
                const float4 x = src[((r0 + r) * D + c0) >> 2];
                s[r][0] = x.x;
                s[r][1] = x.y;
                s[r][2] = x.z;
                s[r][3] = x.w;
            }
        } else {
            const uint2 *src = reinterpret_cast<const uint2 *>(static_cast<const uint16_t *>(p.state_in) + st);
#pragma unroll
            for (int r = 0; r < ROWS; ++r) raw[r] = src[((r0 + r) * D + c0) >> 2];
        }
    } else {
        if constexpr (kFp32State) {
#pragma unroll
            for (int r = 0; r < ROWS; ++r) s[r][0] = s[r][1] = s[r][2] = s[r][3] = 0.f;
        } else {
#pragma unroll
            for (int r = 0; r < ROWS; ++r) raw[r] = make_uint2(0u, 0u);
        }
    }
    // row r of S' = Diag(alpha) S, in fp32
    auto decayed = [&](int r, float a, float (&x)[4]) {
        if constexpr (kFp32State) {
#pragma unroll
            for (int c = 0; c < 4; ++c) x[c] = s[r][c] * a;
        } else {
            x[0] = bf_lo(raw[r].x) * a;
            x[1] = bf_hi(raw[r].x) * a;
            x[2] = bf_lo(raw[r].y) * a;
            x[3] = bf_hi(raw[r].y) * a;
        }
    };
    if (tid < D) {
        ks[tid] = __uint_as_float(static_cast<uint32_t>(p.k[vec + tid]) << 16);
        qs[tid] = __uint_as_float(static_cast<uint32_t>(p.q[vec + tid]) << 16);
        as[tid] = ex2(kLog2e * p.g[vec + tid]);
    }
    const float beta = p.beta[bh];
    uint2 vw = make_uint2(0u, 0u);   // v[c0 .. c0 + 3], needed by warp 0 only
    if (warp == 0) vw = reinterpret_cast<const uint2 *>(p.v + vec)[lane];
    __syncthreads();

    // S' = Diag(alpha) S, and this warp's share of S'^T k, S'^T q and k . q
    float pk[4] = {0.f, 0.f, 0.f, 0.f}, pq[4] = {0.f, 0.f, 0.f, 0.f}, kq = 0.f;
#pragma unroll
    for (int r = 0; r < ROWS; ++r) {
        const float kr = ks[r0 + r], qr = qs[r0 + r];
        float x[4];
        decayed(r, as[r0 + r], x);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            pk[c] = fmaf(x[c], kr, pk[c]);
            pq[c] = fmaf(x[c], qr, pq[c]);
        }
        kq = fmaf(kr, qr, kq);
    }
    red[warp][0][lane] = make_float4(pk[0], pk[1], pk[2], pk[3]);
    red[warp][1][lane] = make_float4(pq[0], pq[1], pq[2], pq[3]);
    if (lane == 0) kq_part[warp] = kq;
    __syncthreads();

    float rk[4] = {0.f, 0.f, 0.f, 0.f}, rq[4] = {0.f, 0.f, 0.f, 0.f};
    kq = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
        const float4 a = red[w][0][lane], b = red[w][1][lane];
        rk[0] += a.x;
        rk[1] += a.y;
        rk[2] += a.z;
        rk[3] += a.w;
        rq[0] += b.x;
        rq[1] += b.y;
        rq[2] += b.z;
        rq[3] += b.w;
        kq += kq_part[w];
    }
    float e[4];
    if (warp == 0) {
        e[0] = bf_lo(vw.x) - rk[0];
        e[1] = bf_hi(vw.x) - rk[1];
        e[2] = bf_lo(vw.y) - rk[2];
        e[3] = bf_hi(vw.y) - rk[3];
        // o = scale (S'^T q + beta (k . q) e)
        const float bkq = beta * kq;
        uint2 ow;
        ow.x = bf_pack(p.scale * fmaf(bkq, e[0], rq[0]), p.scale * fmaf(bkq, e[1], rq[1]));
        ow.y = bf_pack(p.scale * fmaf(bkq, e[2], rq[2]), p.scale * fmaf(bkq, e[3], rq[3]));
        reinterpret_cast<uint2 *>(p.out + vec)[lane] = ow;
        es[lane] = make_float4(e[0], e[1], e[2], e[3]);   // hand e to the other warps
    }
    __syncthreads();
    if (!p.state_out) return;
    {
        const float4 e4 = es[lane];
        e[0] = e4.x;
        e[1] = e4.y;
        e[2] = e4.z;
        e[3] = e4.w;
    }
    // S = S' + beta k e^T, written back row by row
#pragma unroll
    for (int r = 0; r < ROWS; ++r) {
        const float bk = beta * ks[r0 + r];
        float x[4];
        decayed(r, as[r0 + r], x);
#pragma unroll
        for (int c = 0; c < 4; ++c) x[c] = fmaf(bk, e[c], x[c]);
        if constexpr (kFp32State) {
            reinterpret_cast<float4 *>(static_cast<float *>(p.state_out) + st)[((r0 + r) * D + c0) >> 2] =
                make_float4(x[0], x[1], x[2], x[3]);
        } else {
            reinterpret_cast<uint2 *>(static_cast<uint16_t *>(p.state_out) + st)[((r0 + r) * D + c0) >> 2] =
                make_uint2(bf_pack(x[0], x[1]), bf_pack(x[2], x[3]));
        }
    }
}

}  // namespace dec

cudaError_t launch_decode(const DecodeParams &p, int64_t units, cudaStream_t stream) {
    if (units <= 0) return cudaSuccess;
    if (units > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    const dim3 grid(static_cast<unsigned>(units));
    if (p.state_fp32)
        dec::kda_decode_kernel<true><<<grid, dec::threads<true>(), 0, stream>>>(p);
    else
        dec::kda_decode_kernel<false><<<grid, dec::threads<false>(), 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace kda
