// kda_fwd_simt.cu -- first, straightforward CUDA-core path of the chunkwise KDA
// forward pass (fp32 arithmetic throughout, no tensor cores).
//
// It evaluates the recurrence of the Kimi Linear feature page (chapter 4,
// state-update equation) chunk by chunk (C = 64), in the chunk-parallel form
// that the page's DPLR remark allows when both low-rank factors are bound to
// k. Per chunk, with G the in-chunk running sum of g (per key channel) and an
// anchor row a (row 31) to keep the factored exponentials in range:
//
//   Qh = Q e^(G - G_a), Kh = K e^(G - G_a), Kc = K e^(G_a - G), Kt = K e^(G_last - G)
//   A  = strict_lower(diag(beta) Kh Kc^T)             (decayed K.K^T block)
//   Tm = (I + A)^-1                                   (UT / WY transform)
//   W  = Tm diag(beta) Kh,   U = Tm diag(beta) V      (pseudo-values)
//   S' = diag(e^G_a) S                                 (anchored chunk-start state)
//   D  = U - W S'                                      (state-dependent pseudo-value)
//   O  = scale (Qh S' + lower(Qh Kc^T) D)              (intra + inter output)
//   S  <- diag(e^G_last) S + Kt^T D                    (inter-chunk state update)
//
// One CTA owns one (sequence, head, 32-column value slice); the value columns
// of S evolve independently, so slices need no communication.
#include <cuda_bf16.h>

#include "kda_internal.h"

namespace kda {
namespace {

constexpr int D = kHeadDim;
constexpr int C = kChunk;
constexpr int NV = 32;           // value columns per CTA
constexpr int NSLICE = D / NV;   // CTAs per (sequence, head)
constexpr int NT = 256;          // threads per CTA
constexpr int LD = D + 1;        // padded row stride of the C x D tiles
constexpr int LC = C + 1;        // padded row stride of the C x C tiles
constexpr int ANCHOR = 31;       // anchor row of the factored exponentials

struct Smem {
    float G[C * LD];    // running log-decay, then Kt
    float Qh[C * LD];
    float Kh[C * LD];
    float Kc[C * LD];   // then W
    float A[C * LC];    // decayed K.K^T block, then the masked Q.K^T block
    float Tm[C * LC];   // (I + A)^-1
    float S[D * NV];    // fp32 state slice
    float S2[D * NV];   // anchored state slice
    float Vs[C * NV];   // value slice, then the pseudo-value D
    float Us[C * NV];
    float ga[D], gl[D], ega[D], egl[D], bt[C];
};

__device__ __forceinline__ float bf2f(uint16_t x) {
    return __uint_as_float(static_cast<uint32_t>(x) << 16);
}

__device__ __forceinline__ uint16_t f2bf(float x) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

__global__ void __launch_bounds__(NT, 1) kda_fwd_simt_kernel(FwdParams p) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>(smem_raw);
    const int tid = threadIdx.x;
    const int H = p.num_heads;
    int64_t unit = blockIdx.x;
    const int slice = static_cast<int>(unit % NSLICE);
    unit /= NSLICE;
    const int h = static_cast<int>(unit % H);
    const int64_t s = unit / H;
    int64_t bos, eos;
    if (p.cu_seqlens) {
        int64_t a = p.cu_seqlens[s], b = p.cu_seqlens[s + 1];
        a = a < 0 ? 0 : (a > p.seq_len ? p.seq_len : a);
        b = b < 0 ? 0 : (b > p.seq_len ? p.seq_len : b);
        bos = a;
        eos = b < a ? a : b;
    } else {
        bos = s * p.seq_len;
        eos = bos + p.seq_len;
    }
    const int v0 = slice * NV;
    const size_t state_base = (static_cast<size_t>(s) * H + h) * D * D;

    for (int e = tid; e < D * NV; e += NT) {
        const int c = e / NV, j = e % NV;
        float x = 0.f;
        if (p.h0) {
            const size_t off = state_base + static_cast<size_t>(c) * D + v0 + j;
            x = p.h0_fp32 ? static_cast<const float *>(p.h0)[off]
                          : bf2f(static_cast<const uint16_t *>(p.h0)[off]);
        }
        sm.S[e] = x;
    }
    __syncthreads();

    for (int64_t t0 = bos; t0 < eos; t0 += C) {
        const int L = static_cast<int>(eos - t0 < C ? eos - t0 : C);
        // -- load the chunk: gates (zero past the sequence end), beta, value slice
        for (int e = tid; e < C * D; e += NT) {
            const int r = e / D, c = e % D;
            sm.G[r * LD + c] = r < L ? p.g[((t0 + r) * H + h) * D + c] : 0.f;
        }
        for (int e = tid; e < C; e += NT) sm.bt[e] = e < L ? p.beta[(t0 + e) * H + h] : 0.f;
        for (int e = tid; e < C * NV; e += NT) {
            const int r = e / NV, j = e % NV;
            sm.Vs[e] = r < L ? bf2f(p.v[((t0 + r) * H + h) * D + v0 + j]) : 0.f;
        }
        __syncthreads();

        // -- S1: in-chunk running sums of the log-gates, one key channel per thread
        if (tid < D) {
            float acc = 0.f;
            for (int r = 0; r < C; ++r) {
                acc += sm.G[r * LD + tid];
                sm.G[r * LD + tid] = acc;
                if (r == ANCHOR) sm.ga[tid] = acc;
            }
            sm.gl[tid] = acc;
            sm.ega[tid] = expf(sm.ga[tid]);
            sm.egl[tid] = expf(acc);
        }
        __syncthreads();

        // -- decayed q and k factors (each element read and written by one thread)
        for (int e = tid; e < C * D; e += NT) {
            const int r = e / D, c = e % D;
            const float gm = sm.G[r * LD + c];
            const size_t off = ((t0 + r) * H + h) * D + c;
            const float qq = r < L ? bf2f(p.q[off]) : 0.f;
            const float kk = r < L ? bf2f(p.k[off]) : 0.f;
            const float eu = expf(gm - sm.ga[c]);
            const float ed = expf(sm.ga[c] - gm);
            sm.Qh[r * LD + c] = qq * eu;
            sm.Kh[r * LD + c] = kk * eu;
            sm.Kc[r * LD + c] = kk * ed;
            sm.G[r * LD + c] = kk * expf(sm.gl[c] - gm);  // Kt
        }
        __syncthreads();

        // -- S2a: A = strict_lower(diag(beta) Kh Kc^T); 4x4 outputs per thread
        {
            const int tr = tid >> 4, ti = tid & 15;
            float acc[4][4] = {};
            for (int c = 0; c < D; ++c) {
                float a[4], b[4];
#pragma unroll
                for (int m = 0; m < 4; ++m) a[m] = sm.Kh[(tr + 16 * m) * LD + c];
#pragma unroll
                for (int n = 0; n < 4; ++n) b[n] = sm.Kc[(ti + 16 * n) * LD + c];
#pragma unroll
                for (int m = 0; m < 4; ++m)
#pragma unroll
                    for (int n = 0; n < 4; ++n) acc[m][n] = fmaf(a[m], b[n], acc[m][n]);
            }
#pragma unroll
            for (int m = 0; m < 4; ++m)
#pragma unroll
                for (int n = 0; n < 4; ++n) {
                    const int r = tr + 16 * m, i = ti + 16 * n;
                    sm.A[r * LC + i] = i < r ? sm.bt[r] * acc[m][n] : 0.f;
                }
        }
        __syncthreads();

        // -- S3: Tm = (I + A)^-1 by forward substitution, one row at a time:
        //    Tm[r, :] = e_r - sum_{j<r} A[r, j] Tm[j, :]
        for (int r = 0; r < C; ++r) {
            if (tid < C) {
                const int i = tid;
                float x = (i == r) ? 1.f : 0.f;
                for (int j = i; j < r; ++j) x = fmaf(-sm.A[r * LC + j], sm.Tm[j * LC + i], x);
                sm.Tm[r * LC + i] = x;
            }
            __syncthreads();
        }

        // -- S2b: A <- lower(Qh Kc^T) (diagonal included)
        {
            const int tr = tid >> 4, ti = tid & 15;
            float acc[4][4] = {};
            for (int c = 0; c < D; ++c) {
                float a[4], b[4];
#pragma unroll
                for (int m = 0; m < 4; ++m) a[m] = sm.Qh[(tr + 16 * m) * LD + c];
#pragma unroll
                for (int n = 0; n < 4; ++n) b[n] = sm.Kc[(ti + 16 * n) * LD + c];
#pragma unroll
                for (int m = 0; m < 4; ++m)
#pragma unroll
                    for (int n = 0; n < 4; ++n) acc[m][n] = fmaf(a[m], b[n], acc[m][n]);
            }
#pragma unroll
            for (int m = 0; m < 4; ++m)
#pragma unroll
                for (int n = 0; n < 4; ++n) {
                    const int r = tr + 16 * m, i = ti + 16 * n;
                    sm.A[r * LC + i] = i <= r ? acc[m][n] : 0.f;
                }
        }
        __syncthreads();

        // -- S4: W = Tm diag(beta) Kh (into Kc), U = Tm diag(beta) V, S' = diag(e^G_a) S
        {
            const int tr = tid >> 4, tc = tid & 15;
            float acc[4][8] = {};
            for (int i = 0; i < C; ++i) {
                const float b = sm.bt[i];
                float t[4], kv[8];
#pragma unroll
                for (int m = 0; m < 4; ++m) t[m] = sm.Tm[(tr + 16 * m) * LC + i];
#pragma unroll
                for (int n = 0; n < 8; ++n) kv[n] = b * sm.Kh[i * LD + tc + 16 * n];
#pragma unroll
                for (int m = 0; m < 4; ++m)
#pragma unroll
                    for (int n = 0; n < 8; ++n) acc[m][n] = fmaf(t[m], kv[n], acc[m][n]);
            }
#pragma unroll
            for (int m = 0; m < 4; ++m)
#pragma unroll
                for (int n = 0; n < 8; ++n) sm.Kc[(tr + 16 * m) * LD + tc + 16 * n] = acc[m][n];
        }
        {
            const int r = tid >> 2, jb = tid & 3;
            float acc[8] = {};
            for (int i = 0; i < C; ++i) {
                const float t = sm.Tm[r * LC + i] * sm.bt[i];
#pragma unroll
                for (int n = 0; n < 8; ++n) acc[n] = fmaf(t, sm.Vs[i * NV + jb + 4 * n], acc[n]);
            }
#pragma unroll
            for (int n = 0; n < 8; ++n) sm.Us[r * NV + jb + 4 * n] = acc[n];
        }
        for (int e = tid; e < D * NV; e += NT) sm.S2[e] = sm.ega[e / NV] * sm.S[e];
        __syncthreads();

        // -- S5: D = U - W S'  (into Vs)
        {
            const int r = tid >> 2, jb = tid & 3;
            float acc[8];
#pragma unroll
            for (int n = 0; n < 8; ++n) acc[n] = sm.Us[r * NV + jb + 4 * n];
            for (int c = 0; c < D; ++c) {
                const float w = sm.Kc[r * LD + c];
#pragma unroll
                for (int n = 0; n < 8; ++n) acc[n] = fmaf(-w, sm.S2[c * NV + jb + 4 * n], acc[n]);
            }
#pragma unroll
            for (int n = 0; n < 8; ++n) sm.Vs[r * NV + jb + 4 * n] = acc[n];
        }
        __syncthreads();

        // -- S6: O = scale (Qh S' + lower(Qh Kc^T) D), written for the valid rows
        {
            const int r = tid >> 2, jb = tid & 3;
            float acc[8] = {};
            for (int c = 0; c < D; ++c) {
                const float qv = sm.Qh[r * LD + c];
#pragma unroll
                for (int n = 0; n < 8; ++n) acc[n] = fmaf(qv, sm.S2[c * NV + jb + 4 * n], acc[n]);
            }
            for (int i = 0; i <= r; ++i) {
                const float a = sm.A[r * LC + i];
#pragma unroll
                for (int n = 0; n < 8; ++n) acc[n] = fmaf(a, sm.Vs[i * NV + jb + 4 * n], acc[n]);
            }
            if (r < L) {
                uint16_t *o = p.out + ((t0 + r) * H + h) * D + v0;
#pragma unroll
                for (int n = 0; n < 8; ++n) o[jb + 4 * n] = f2bf(p.scale * acc[n]);
            }
        }
        // -- S7: S <- diag(e^G_last) S + Kt^T D
        {
            const int c = tid >> 1, jb = tid & 1;
            float acc[16];
            const float dec = sm.egl[c];
#pragma unroll
            for (int n = 0; n < 16; ++n) acc[n] = dec * sm.S[c * NV + jb + 2 * n];
            for (int i = 0; i < C; ++i) {
                const float kt = sm.G[i * LD + c];
#pragma unroll
                for (int n = 0; n < 16; ++n) acc[n] = fmaf(kt, sm.Vs[i * NV + jb + 2 * n], acc[n]);
            }
#pragma unroll
            for (int n = 0; n < 16; ++n) sm.S[c * NV + jb + 2 * n] = acc[n];
        }
        __syncthreads();
    }

    // -- S8: final state slice
    if (p.hT) {
        for (int e = tid; e < D * NV; e += NT) {
            const int c = e / NV, j = e % NV;
            const size_t off = state_base + static_cast<size_t>(c) * D + v0 + j;
            if (p.hT_fp32) static_cast<float *>(p.hT)[off] = sm.S[e];
            else static_cast<uint16_t *>(p.hT)[off] = f2bf(sm.S[e]);
        }
    }
}

}  // namespace

cudaError_t launch_fwd_simt(const FwdParams &p, cudaStream_t stream) {
    const int64_t grid = static_cast<int64_t>(p.num_seqs) * p.num_heads * NSLICE;
    if (grid == 0) return cudaSuccess;
    if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    const size_t smem = sizeof(Smem);
    cudaError_t err = cudaFuncSetAttribute(kda_fwd_simt_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    kda_fwd_simt_kernel<<<static_cast<unsigned>(grid), NT, smem, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace kda
