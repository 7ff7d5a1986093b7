// kda_bwd.cu -- backward pass of the chunkwise KDA forward (gradients of q, k, v, g, beta and
// the initial state), fp32 on CUDA cores.
//
// The forward is the recurrence of the Kimi Linear feature page (chapter 4, state-update
// equation). Written in chunks of CB tokens (G the chunk's running log-decay per key channel,
// Kd = K e^G, Qd = Q e^G, Kn = K e^-G, Kt = K e^(Gl - G), e^Gl the decay over the chunk):
//
//   Akk = strict_lower(Diag(beta) Kd Kn^T),  Aqk = lower(Qd Kn^T),  T = (I + Akk)^-1
//   X = V - Kd S0,  D = T Diag(beta) X,  O = scale (Qd S0 + Aqk D),  S1 = Diag(e^Gl) S0 + Kt^T D
//
// and its reverse, chunk by chunk from the last (dS the gradient of the state leaving the chunk):
//
//   dQd = scale dO S0^T + dAqk Kn          dAqk = lower(scale dO D^T)
//   dD  = scale Aqk^T dO + Kt dS           dKt  = D dS^T,    dGl = e^Gl (.) rowsum(dS (.) S0)
//   dTp = dD X^T,  dX = (T Diag(beta))^T dD,  dV = dX,   dKd = -dX S0^T + dB Kn
//   dbeta = colsum(dTp (.) T) + rowsum(dAkk (.) B),  dAkk = strict_lower(-T^T (dTp Diag(beta)) T^T)
//   dB = Diag(beta) dAkk (B = Kd Kn^T),    dKn = dB^T Kd + dAqk^T Qd
//   dS0 = scale Qd^T dO + Diag(e^Gl) dS - Kd^T dX
//   dK = dKd e^G + dKn e^-G + dKt e^(Gl - G),   dQ = dQd e^G
//   dG = dKd (.) Kd + dQd (.) Qd - dKn (.) Kn - dKt (.) Kt  (+ dGl + colsum(dKt (.) Kt) on the last row)
//   dg = the reverse running sum of dG over the chunk
//
// Layout of the work:
//  * CB = 16 tokens per chunk, so that one anchor row a = 7 per chunk keeps every decayed factor
//    in range: with per-token log-decays floored at -10 (as in the forward's sub-block path),
//    |G_r - G_a| <= 8 x 10, and the factors K e^(G - G_a), K e^(G_a - G) stay below e^80. Every
//    product with e^-G is formed from them: e^(G_r - G_i) = e^(G_r - G_a) e^(G_a - G_i).
//  * Four CTAs per (sequence, head), each owning 32 of the 128 value columns of the state and
//    of dS: the state and dS recurrences act on value columns independently. The gradients of
//    q, k, g and beta are sums over value columns of terms linear in the CTA's partial sums, so
//    each CTA adds its share to them (fp32 atomics on outputs the host zeroed first); v and the
//    initial-state gradient are per column.
//  * A forward sweep stores the state entering every 64 tokens (a checkpoint) in the workspace;
//    the reverse sweep takes the 64-token groups last first, recomputes the states entering its
//    four chunks from the checkpoint, then runs the chunks backwards.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "kda_internal.h"

namespace kda {
namespace bwd {

constexpr int D = kHeadDim;      // 128
constexpr int CB = 16;           // tokens per chunk
constexpr int GRP = 64;          // tokens per checkpoint
constexpr int NSUB = GRP / CB;   // chunks per checkpoint group
constexpr int NV = 4;            // value-column slices (CTAs) per (sequence, head)
constexpr int VS = D / NV;       // 32 value columns per CTA
constexpr int VP = VS + 1;       // padded row pitch of a state slice: rows c, c + 1 in distinct banks
constexpr int NT = 256;
constexpr int AP = CB + 1;       // pitch of the CB x CB matrices
constexpr int DP = D + 1;        // pitch of the CB x D tiles: 16 lanes reading one column of 16 rows hit distinct banks
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kFloorLog2 = -14.426950408889634f;   // log2 of e^-10

// shared memory (floats)
constexpr int SM_SCK = 0;                          // NSUB states [D][VP] entering the group's chunks
constexpr int SM_DS = SM_SCK + NSUB * D * VP;      // dS [D][VP]
constexpr int SM_K = SM_DS + D * VP;               // [CB][D] each: K, Q, G (log2 units)
constexpr int SM_Q = SM_K + CB * DP;
constexpr int SM_G = SM_Q + CB * DP;
constexpr int SM_KD = SM_G + CB * DP;              // Kd, Qd, Kt
constexpr int SM_QD = SM_KD + CB * DP;
constexpr int SM_KT = SM_QD + CB * DP;
constexpr int SM_KL = SM_KT + CB * DP;             // K e^(G - Ga), Q e^(G - Ga), K e^(Ga - G)
constexpr int SM_QL = SM_KL + CB * DP;
constexpr int SM_KR = SM_QL + CB * DP;
constexpr int SM_P1 = SM_KR + CB * DP;             // partial sums [CB][D]: dQd, dKt, dKd
constexpr int SM_P2 = SM_P1 + CB * DP;
constexpr int SM_P3 = SM_P2 + CB * DP;
constexpr int SM_V = SM_P3 + CB * DP;              // [CB][VP] slices: V, dO, X, D, dD, dX
constexpr int SM_DO = SM_V + CB * VP;
constexpr int SM_X = SM_DO + CB * VP;
constexpr int SM_DD = SM_X + CB * VP;
constexpr int SM_DX = SM_DD + CB * VP;
constexpr int SM_D = SM_DX + CB * VP;
constexpr int SM_B = SM_D + CB * VP;               // [CB][AP]: B = Kd Kn^T, Aqk, T, dAqk, dTp, dAkk
constexpr int SM_AQK = SM_B + CB * AP;
constexpr int SM_T = SM_AQK + CB * AP;
constexpr int SM_DAQK = SM_T + CB * AP;
constexpr int SM_DTP = SM_DAQK + CB * AP;
constexpr int SM_DAKK = SM_DTP + CB * AP;
constexpr int SM_BETA = SM_DAKK + CB * AP;         // [CB]
constexpr int SM_EC = SM_BETA + CB;                // [D] e^Gl
constexpr int SM_DGL = SM_EC + D;                  // [D] dGl partial
constexpr int SM_DBETA = SM_DGL + D;               // [CB]
constexpr int SM_FLOATS = SM_DBETA + CB;
constexpr size_t SMEM_BYTES = static_cast<size_t>(SM_FLOATS) * sizeof(float);
static_assert(SMEM_BYTES <= 227 * 1024, "backward shared memory");

__device__ __forceinline__ float ex2(float y) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(y));
    return r;
}
__device__ __forceinline__ float bf(uint16_t x) { return __uint_as_float(static_cast<uint32_t>(x) << 16); }

struct Unit {
    int64_t bos, eos;   // token range of the sequence
    int64_t slot0;      // first checkpoint slot of the sequence
    int s, h, vs;       // sequence, head, value slice
};

__device__ __forceinline__ Unit unit_of(const BwdParams &p) {
    Unit u;
    const int64_t cta = blockIdx.x;
    u.vs = static_cast<int>(cta % NV);
    const int64_t pair = cta / NV;
    u.h = static_cast<int>(pair % p.num_heads);
    u.s = static_cast<int>(pair / p.num_heads);
    if (p.cu_seqlens) {
        int64_t a = p.cu_seqlens[u.s], b = p.cu_seqlens[u.s + 1];
        a = a < 0 ? 0 : (a > p.seq_len ? p.seq_len : a);
        b = b < 0 ? 0 : (b > p.seq_len ? p.seq_len : b);
        u.bos = a;
        u.eos = b < a ? a : b;
    } else {
        u.bos = static_cast<int64_t>(u.s) * p.seq_len;
        u.eos = u.bos + p.seq_len;
    }
    // collision-free: a sequence of L tokens needs ceil(L / 64) <= floor(L / 64) + 1 slots
    u.slot0 = u.bos / GRP + u.s;
    return u;
}

__device__ __forceinline__ void prefetch_l2(const void *ptr) { asm volatile("prefetch.global.L2 [%0];" ::"l"(ptr)); }

// Ask L2 for the inputs of the chunk at t0 (the next one this CTA loads), one request per 128-byte
// line of its rows: the chunks run in a sequential order, so the loads of each one would otherwise
// wait on HBM latency in full.
__device__ void prefetch_chunk(const BwdParams &p, const Unit &u, int64_t t0, bool with_do) {
    const int t = threadIdx.x;
    if (t0 < u.bos || t0 >= u.eos) return;
    const int L = static_cast<int>(u.eos - t0 < CB ? u.eos - t0 : CB);
    const int H = p.num_heads;
    const int r = t >> 4, part = t & 15;
    if (r >= L) return;
    const size_t row = (static_cast<size_t>(t0) + r) * H + u.h;
    if (part < 2) {                          // k and q rows: 256 bytes each
        prefetch_l2(p.k + row * D + part * 64);
        prefetch_l2(p.q + row * D + part * 64);
    } else if (part < 6) {                   // g rows: 512 bytes
        prefetch_l2(p.g + row * D + (part - 2) * 32);
    } else if (part == 6) {                  // this CTA's value slice of v and dO: 64 bytes
        prefetch_l2(p.v + row * D + u.vs * VS);
        if (with_do) prefetch_l2(p.dout + row * D + u.vs * VS);
    } else if (part == 7) {
        prefetch_l2(p.beta + row);
    }
}

// Load chunk n of the unit (rows past the end are zero, with no decay) and form its factors:
// G (floored, log2 units), Kd, Qd, Kt, the anchored Kl, Ql, Kr, e^Gl, beta, and the V and dO
// slices (dO only when `with_do`).
__device__ void load_chunk(const BwdParams &p, const Unit &u, int64_t t0, int L, bool with_do, float *sm) {
    const int t = threadIdx.x;
    const int H = p.num_heads;
    {   // K, Q and g: thread t takes row t >> 4, channels 8 (t & 15) .. + 8
        const int r = t >> 4, c0 = (t & 15) * 8;
        const size_t off = ((static_cast<size_t>(t0) + r) * H + u.h) * D + c0;
        if (r < L) {
            // 16-byte loads: 8 bf16 of k and of q, 2 x 4 fp32 of g (rows start 256 / 512 B apart)
            const uint4 kw = *reinterpret_cast<const uint4 *>(p.k + off);
            const uint4 qw = *reinterpret_cast<const uint4 *>(p.q + off);
            const float4 g0 = *reinterpret_cast<const float4 *>(p.g + off);
            const float4 g1 = *reinterpret_cast<const float4 *>(p.g + off + 4);
            const uint32_t kk[4] = {kw.x, kw.y, kw.z, kw.w}, qq[4] = {qw.x, qw.y, qw.z, qw.w};
            const float gg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const uint32_t kb2 = kk[e >> 1], qb2 = qq[e >> 1];
                sm[SM_K + r * DP + c0 + e] = __uint_as_float((e & 1) ? (kb2 & 0xFFFF0000u) : (kb2 << 16));
                sm[SM_Q + r * DP + c0 + e] = __uint_as_float((e & 1) ? (qb2 & 0xFFFF0000u) : (qb2 << 16));
                sm[SM_G + r * DP + c0 + e] = fmaxf(gg[e] * kLog2e, kFloorLog2);
            }
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) sm[SM_K + r * DP + c0 + e] = sm[SM_Q + r * DP + c0 + e] = sm[SM_G + r * DP + c0 + e] = 0.f;
        }
    }
    {   // V and dO slices: thread t takes row t >> 4, columns 2 (t & 15) .. + 2 of the slice
        const int r = t >> 4, j0 = (t & 15) * 2;
        const size_t off = ((static_cast<size_t>(t0) + r) * H + u.h) * D + u.vs * VS + j0;
        uint32_t vw = 0u, dw = 0u;   // two bf16 each
        if (r < L) {
            vw = *reinterpret_cast<const uint32_t *>(p.v + off);
            if (with_do) dw = *reinterpret_cast<const uint32_t *>(p.dout + off);
        }
        sm[SM_V + r * VP + j0] = __uint_as_float(vw << 16);
        sm[SM_V + r * VP + j0 + 1] = __uint_as_float(vw & 0xFFFF0000u);
        if (with_do) {
            sm[SM_DO + r * VP + j0] = __uint_as_float(dw << 16);
            sm[SM_DO + r * VP + j0 + 1] = __uint_as_float(dw & 0xFFFF0000u);
        }
    }
    if (t < CB) {
        float b = 0.f;
        if (t < L) b = p.beta[(static_cast<size_t>(t0) + t) * H + u.h];
        sm[SM_BETA + t] = b;
    }
    __syncthreads();
    if (t < D) {   // running sum over the chunk's rows, per channel
        float run = 0.f;
#pragma unroll
        for (int r = 0; r < CB; ++r) {
            run += sm[SM_G + r * DP + t];
            sm[SM_G + r * DP + t] = run;
        }
        sm[SM_EC + t] = ex2(run);
    }
    __syncthreads();
    {
        // row t >> 4, channels (t & 15) + 16 e: consecutive lanes take consecutive channels
        const int r = t >> 4;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int c = (t & 15) + 16 * e;
            const float gr = sm[SM_G + r * DP + c], ga = sm[SM_G + 7 * DP + c], gl = sm[SM_G + (CB - 1) * DP + c];
            const float k = sm[SM_K + r * DP + c], q = sm[SM_Q + r * DP + c];
            const float ed = ex2(gr), el = ex2(gr - ga), er = ex2(ga - gr);
            sm[SM_KD + r * DP + c] = k * ed;
            sm[SM_QD + r * DP + c] = q * ed;
            sm[SM_KT + r * DP + c] = k * ex2(gl - gr);
            sm[SM_KL + r * DP + c] = k * el;
            sm[SM_QL + r * DP + c] = q * el;
            sm[SM_KR + r * DP + c] = k * er;
        }
    }
    __syncthreads();
}

// B = Kd Kn^T (r >= i), Aqk = lower(Qd Kn^T), and T = (I + strict_lower(Diag(beta) B))^-1.
__device__ void chunk_blocks(float *sm) {
    const int t = threadIdx.x;
    {
        const int r = t >> 4, i = t & 15;
        float b = 0.f, a = 0.f;
        if (i <= r) {
#pragma unroll 8
            for (int c = 0; c < D; ++c) {
                const float kr = sm[SM_KR + i * DP + c];
                b = fmaf(sm[SM_KL + r * DP + c], kr, b);
                a = fmaf(sm[SM_QL + r * DP + c], kr, a);
            }
        }
        sm[SM_B + r * AP + i] = b;
        sm[SM_AQK + r * AP + i] = a;
    }
    __syncthreads();
    if (t < CB) {
        // column t of T by forward substitution: T[r][t] = [r == t] - sum_{i<r} A[r][i] T[i][t]
        const int col = t;
        float x[CB];
#pragma unroll
        for (int r = 0; r < CB; ++r) {
            float v = r == col ? 1.f : 0.f;
            const float br = sm[SM_BETA + r];
#pragma unroll
            for (int i = 0; i < r; ++i) v = fmaf(-br * sm[SM_B + r * AP + i], x[i], v);
            x[r] = v;
        }
#pragma unroll
        for (int r = 0; r < CB; ++r) sm[SM_T + r * AP + col] = x[r];
    }
    __syncthreads();
}

// X = V - Kd S0 and D = T Diag(beta) X on this CTA's value slice; S0 is a [D][VP] state slice.
__device__ void chunk_xd(float *sm, const float *S0) {
    const int t = threadIdx.x;
    const int r = t >> 4, j0 = (t & 15) * 2;
    {
        float x0 = sm[SM_V + r * VP + j0], x1 = sm[SM_V + r * VP + j0 + 1];
#pragma unroll 8
        for (int c = 0; c < D; ++c) {
            const float kd = sm[SM_KD + r * DP + c];
            x0 = fmaf(-kd, S0[c * VP + j0], x0);
            x1 = fmaf(-kd, S0[c * VP + j0 + 1], x1);
        }
        sm[SM_X + r * VP + j0] = x0;
        sm[SM_X + r * VP + j0 + 1] = x1;
    }
    __syncthreads();
    {
        float d0 = 0.f, d1 = 0.f;
#pragma unroll
        for (int i = 0; i < CB; ++i) {
            const float w = sm[SM_T + r * AP + i] * sm[SM_BETA + i];
            d0 = fmaf(w, sm[SM_X + i * VP + j0], d0);
            d1 = fmaf(w, sm[SM_X + i * VP + j0 + 1], d1);
        }
        sm[SM_D + r * VP + j0] = d0;
        sm[SM_D + r * VP + j0 + 1] = d1;
    }
    __syncthreads();
}

// S1 = Diag(e^Gl) S0 + Kt^T D on the slice (S1 may not alias S0).
__device__ void chunk_state(float *sm, const float *S0, float *S1) {
    const int t = threadIdx.x;
    const int c = t >> 1, j0 = (t & 1) * 16;
    const float ec = sm[SM_EC + c];
    float acc[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) acc[e] = ec * S0[c * VP + j0 + e];
#pragma unroll
    for (int r = 0; r < CB; ++r) {
        const float kt = sm[SM_KT + r * DP + c];
#pragma unroll
        for (int e = 0; e < 16; ++e) acc[e] = fmaf(kt, sm[SM_D + r * VP + j0 + e], acc[e]);
    }
#pragma unroll
    for (int e = 0; e < 16; ++e) S1[c * VP + j0 + e] = acc[e];
    __syncthreads();
}

// state slice global <-> shared
__device__ void state_to_global(const float *S, float *dst) {
    const int t = threadIdx.x;
    for (int e = t; e < D * VS; e += NT) {
        const int c = e / VS, j = e % VS;
        dst[static_cast<size_t>(c) * D + j] = S[c * VP + j];
    }
}
__device__ void state_from_global(float *S, const float *src) {
    const int t = threadIdx.x;
    for (int e = t; e < D * VS; e += NT) {
        const int c = e / VS, j = e % VS;
        S[c * VP + j] = src[static_cast<size_t>(c) * D + j];
    }
}

__global__ void __launch_bounds__(NT, 1) kda_bwd_kernel(const BwdParams p) {
    extern __shared__ __align__(16) float sm[];
    const int t = threadIdx.x;
    const Unit u = unit_of(p);
    const int H = p.num_heads;
    const int64_t len = u.eos - u.bos;
    const int ngrp = static_cast<int>((len + GRP - 1) / GRP);
    const size_t head_state = static_cast<size_t>(D) * D;
    // this CTA's view of a [.., H, D, D] state array: row 0 of its value slice
    auto state_at = [&](float *base, int64_t index) -> float * {
        return base + (static_cast<size_t>(index) * H + u.h) * head_state + static_cast<size_t>(u.vs) * VS;
    };
    float *S = sm + SM_SCK;           // forward sweep: the running state (slot 0), next (slot 1)
    float *dS = sm + SM_DS;

    // ---------------------------------------------------------------- forward sweep
    for (int e = t; e < D * VS; e += NT) {
        const int c = e / VS, j = e % VS;
        float x = 0.f;
        if (p.h0) {
            const size_t idx = ((static_cast<size_t>(u.s) * H + u.h) * D + c) * D + u.vs * VS + j;
            x = p.h0_fp32 ? static_cast<const float *>(p.h0)[idx] : bf(static_cast<const uint16_t *>(p.h0)[idx]);
        }
        S[c * VP + j] = x;
    }
    __syncthreads();
    for (int gi = 0; gi < ngrp; ++gi) {
        state_to_global(S, state_at(p.workspace, u.slot0 + gi));
        __syncthreads();
        for (int sub = 0; sub < NSUB; ++sub) {
            const int64_t t0 = u.bos + static_cast<int64_t>(gi) * GRP + sub * CB;
            if (t0 >= u.eos) break;
            const int L = static_cast<int>(u.eos - t0 < CB ? u.eos - t0 : CB);
            prefetch_chunk(p, u, t0 + CB, false);
            load_chunk(p, u, t0, L, false, sm);
            chunk_blocks(sm);
            chunk_xd(sm, S);
            chunk_state(sm, S, S + D * VP);
            for (int e = t; e < D * VS; e += NT) {
                const int c = e / VS, j = e % VS;
                S[c * VP + j] = S[D * VP + c * VP + j];
            }
            __syncthreads();
        }
    }

    // ---------------------------------------------------------------- reverse sweep
    for (int e = t; e < D * VS; e += NT) {
        const int c = e / VS, j = e % VS;
        dS[c * VP + j] = p.dhT ? state_at(const_cast<float *>(p.dhT), u.s)[static_cast<size_t>(c) * D + j] : 0.f;
    }
    __syncthreads();
    const float scale = p.scale;
    for (int gi = ngrp - 1; gi >= 0; --gi) {
        const int64_t g0 = u.bos + static_cast<int64_t>(gi) * GRP;
        const int nsub = static_cast<int>((u.eos - g0 < GRP ? u.eos - g0 : GRP) + CB - 1) / CB;
        // the states entering the group's chunks, from its checkpoint
        state_from_global(sm + SM_SCK, state_at(p.workspace, u.slot0 + gi));
        __syncthreads();
        for (int sub = 0; sub + 1 < nsub; ++sub) {
            const int64_t t0 = g0 + sub * CB;
            const int L = static_cast<int>(u.eos - t0 < CB ? u.eos - t0 : CB);
            prefetch_chunk(p, u, t0 + CB, sub + 2 == nsub);   // the last one is next taken backwards
            load_chunk(p, u, t0, L, false, sm);
            chunk_blocks(sm);
            chunk_xd(sm, sm + SM_SCK + sub * D * VP);
            chunk_state(sm, sm + SM_SCK + sub * D * VP, sm + SM_SCK + (sub + 1) * D * VP);
        }
        for (int sub = nsub - 1; sub >= 0; --sub) {
            const int64_t t0 = g0 + sub * CB;
            const int L = static_cast<int>(u.eos - t0 < CB ? u.eos - t0 : CB);
            const float *S0 = sm + SM_SCK + sub * D * VP;
            if (sub > 0) {
                prefetch_chunk(p, u, t0 - CB, true);
            } else if (gi > 0) {
                // the next group: its checkpoint, then its first chunk
                if (t < D) prefetch_l2(state_at(p.workspace, u.slot0 + gi - 1) + static_cast<size_t>(t) * D);
                prefetch_chunk(p, u, g0 - GRP, false);   // a full group: recomputed forwards first
            }
            load_chunk(p, u, t0, L, true, sm);
            chunk_blocks(sm);
            chunk_xd(sm, S0);
            // ---- partial sums over this CTA's value columns
            {
                // dQd0 = scale dO S0^T [r][c] (SM_P1), dKt = D dS^T (SM_P2): row t >> 4, channels
                // (t & 15) + 16 e
                const int r = t >> 4, c0 = t & 15;
                float q8[8], k8[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) q8[e] = k8[e] = 0.f;
#pragma unroll 4
                for (int j = 0; j < VS; ++j) {
                    const float dO = sm[SM_DO + r * VP + j], dd = sm[SM_D + r * VP + j];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        q8[e] = fmaf(dO, S0[(c0 + 16 * e) * VP + j], q8[e]);
                        k8[e] = fmaf(dd, dS[(c0 + 16 * e) * VP + j], k8[e]);
                    }
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    sm[SM_P1 + r * DP + c0 + 16 * e] = scale * q8[e];
                    sm[SM_P2 + r * DP + c0 + 16 * e] = k8[e];
                }
            }
            {
                // dAqk = lower(scale dO D^T) (partial), r = t >> 4, i = t & 15
                const int r = t >> 4, i = t & 15;
                float a = 0.f;
                if (i <= r) {
#pragma unroll 8
                    for (int j = 0; j < VS; ++j) a = fmaf(sm[SM_DO + r * VP + j], sm[SM_D + i * VP + j], a);
                }
                sm[SM_DAQK + r * AP + i] = scale * a;
            }
            if (t < D) {
                // dGl = e^Gl (.) rowsum(dS (.) S0) (partial)
                float a = 0.f;
#pragma unroll 8
                for (int j = 0; j < VS; ++j) a = fmaf(dS[t * VP + j], S0[t * VP + j], a);
                sm[SM_DGL + t] = sm[SM_EC + t] * a;
            }
            __syncthreads();
            {
                // dD = scale Aqk^T dO + Kt dS (slice), row t >> 4, columns 2 (t & 15)
                const int r = t >> 4, j0 = (t & 15) * 2;
                float d0 = 0.f, d1 = 0.f;
#pragma unroll
                for (int i = 0; i < CB; ++i) {
                    const float a = sm[SM_AQK + i * AP + r];
                    d0 = fmaf(a, sm[SM_DO + i * VP + j0], d0);
                    d1 = fmaf(a, sm[SM_DO + i * VP + j0 + 1], d1);
                }
                d0 *= scale;
                d1 *= scale;
#pragma unroll 8
                for (int c = 0; c < D; ++c) {
                    const float kt = sm[SM_KT + r * DP + c];
                    d0 = fmaf(kt, dS[c * VP + j0], d0);
                    d1 = fmaf(kt, dS[c * VP + j0 + 1], d1);
                }
                sm[SM_DD + r * VP + j0] = d0;
                sm[SM_DD + r * VP + j0 + 1] = d1;
            }
            __syncthreads();
            {
                // dTp = dD X^T (partial) [r][i], and dX = (T Diag(beta))^T dD (slice)
                const int r = t >> 4, i = t & 15;
                float a = 0.f;
#pragma unroll 8
                for (int j = 0; j < VS; ++j) a = fmaf(sm[SM_DD + r * VP + j], sm[SM_X + i * VP + j], a);
                sm[SM_DTP + r * AP + i] = a;
                const int j0 = (t & 15) * 2;
                float x0 = 0.f, x1 = 0.f;
#pragma unroll
                for (int rr = 0; rr < CB; ++rr) {
                    const float w = sm[SM_T + rr * AP + r] * sm[SM_BETA + r];
                    x0 = fmaf(w, sm[SM_DD + rr * VP + j0], x0);
                    x1 = fmaf(w, sm[SM_DD + rr * VP + j0 + 1], x1);
                }
                sm[SM_DX + r * VP + j0] = x0;
                sm[SM_DX + r * VP + j0 + 1] = x1;
                if (r < L) {   // dv = dX
                    const size_t off = ((static_cast<size_t>(t0) + r) * H + u.h) * D + u.vs * VS + j0;
                    p.dv[off] = x0;
                    p.dv[off + 1] = x1;
                }
            }
            __syncthreads();
            {
                // dKd0 = -dX S0^T (partial) [r][c] (SM_P3), channels (t & 15) + 16 e
                const int r = t >> 4, c0 = t & 15;
                float a8[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) a8[e] = 0.f;
#pragma unroll 4
                for (int j = 0; j < VS; ++j) {
                    const float dx = sm[SM_DX + r * VP + j];
#pragma unroll
                    for (int e = 0; e < 8; ++e) a8[e] = fmaf(dx, S0[(c0 + 16 * e) * VP + j], a8[e]);
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) sm[SM_P3 + r * DP + c0 + 16 * e] = -a8[e];
            }
            {
                // dS <- scale Qd^T dO + Diag(e^Gl) dS - Kd^T dX (slice); each thread its own entries
                const int c = t >> 1, j0 = (t & 1) * 16;
                const float ec = sm[SM_EC + c];
                float acc[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) acc[e] = ec * dS[c * VP + j0 + e];
#pragma unroll
                for (int r = 0; r < CB; ++r) {
                    const float qd = scale * sm[SM_QD + r * DP + c], kd = sm[SM_KD + r * DP + c];
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        acc[e] = fmaf(qd, sm[SM_DO + r * VP + j0 + e], fmaf(-kd, sm[SM_DX + r * VP + j0 + e], acc[e]));
                }
                __syncthreads();   // every read of dS (the dKt, dGl and dD sums) is done
#pragma unroll
                for (int e = 0; e < 16; ++e) dS[c * VP + j0 + e] = acc[e];
            }
            // ---- dAkk = strict_lower(-T^T dT T^T), dT = dTp Diag(beta); dbeta (partial)
            {
                const int r = t >> 4, i = t & 15;
                // M = dT T^T: M[r][i] = sum_m dTp[r][m] beta_m T[i][m]
                float m = 0.f;
#pragma unroll
                for (int mm = 0; mm < CB; ++mm)
                    m = fmaf(sm[SM_DTP + r * AP + mm] * sm[SM_BETA + mm], sm[SM_T + i * AP + mm], m);
                __syncthreads();
                sm[SM_DAKK + r * AP + i] = m;   // M, in place of dAkk for now
                __syncthreads();
                // dAkk[r][i] = -sum_m T[m][r] M[m][i], strictly lower
                float a = 0.f;
                if (i < r) {
#pragma unroll
                    for (int mm = 0; mm < CB; ++mm) a = fmaf(sm[SM_T + mm * AP + r], sm[SM_DAKK + mm * AP + i], a);
                    a = -a;
                }
                __syncthreads();
                sm[SM_DAKK + r * AP + i] = a;
                __syncthreads();
            }
            if (t < CB) {
                // dbeta[t] = sum_r dTp[r][t] T[r][t] + sum_i dAkk[t][i] B[t][i]
                float a = 0.f;
#pragma unroll
                for (int r = 0; r < CB; ++r) a = fmaf(sm[SM_DTP + r * AP + t], sm[SM_T + r * AP + t], a);
#pragma unroll
                for (int i = 0; i < CB; ++i) a = fmaf(sm[SM_DAKK + t * AP + i], sm[SM_B + t * AP + i], a);
                if (t < L) atomicAdd(&p.dbeta[(static_cast<size_t>(t0) + t) * H + u.h], a);
            }
            // ---- dK, dQ, dG (partials) for row r = t >> 4, channels 8 (t & 15) .. + 8
            {
                const int r = t >> 4;
                const float br = sm[SM_BETA + r];
#pragma unroll 2
                for (int e = 0; e < 8; ++e) {
                    const int c = (t & 15) + 16 * e;
                    const float gr = sm[SM_G + r * DP + c], ga = sm[SM_G + 7 * DP + c], gl = sm[SM_G + (CB - 1) * DP + c];
                    const float lk = ex2(gr - ga), rs = ex2(ga - gr), ed = ex2(gr), et = ex2(gl - gr);
                    // (dB Kn) e^G and (dAqk Kn) e^G: lk * sum_i x[r][i] Kr[i]; dB = Diag(beta) dAkk
                    float bk = 0.f, ak = 0.f;
                    for (int i = 0; i <= r; ++i) {
                        const float kr = sm[SM_KR + i * DP + c];
                        bk = fmaf(sm[SM_DAKK + r * AP + i], kr, bk);
                        ak = fmaf(sm[SM_DAQK + r * AP + i], kr, ak);
                    }
                    bk *= br * lk;
                    ak *= lk;
                    // (dB^T Kd) e^-G and (dAqk^T Qd) e^-G: rs * sum_m x[m][r] Kl[m], Ql[m]
                    float bt = 0.f, at = 0.f;
                    for (int mm = r; mm < CB; ++mm) {
                        bt = fmaf(sm[SM_DAKK + mm * AP + r] * sm[SM_BETA + mm], sm[SM_KL + mm * DP + c], bt);
                        at = fmaf(sm[SM_DAQK + mm * AP + r], sm[SM_QL + mm * DP + c], at);
                    }
                    const float dkn = rs * (bt + at);                 // dKn e^-G
                    const float dkd = sm[SM_P3 + r * DP + c] * ed + bk;  // dKd e^G
                    const float dqd = sm[SM_P1 + r * DP + c] * ed + ak;  // dQd e^G = dQ
                    const float dkt = sm[SM_P2 + r * DP + c] * et;       // dKt e^(Gl - G)
                    const float k = sm[SM_K + r * DP + c], q = sm[SM_Q + r * DP + c];
                    float dgam = k * dkd + q * dqd - k * dkn - k * dkt;
                    sm[SM_P1 + r * DP + c] = dqd;
                    sm[SM_P3 + r * DP + c] = dkd + dkn + dkt;
                    sm[SM_P2 + r * DP + c] = k * dkt;   // dKt (.) Kt, summed over rows below
                    sm[SM_KD + r * DP + c] = dgam;      // Kd is not read again in this chunk
                }
            }
            __syncthreads();
            if (t < D) {
                // the last row's extra terms, then dg = reverse running sum of dG, floored gates 0
                const int c = t;
                float extra = sm[SM_DGL + c];
#pragma unroll
                for (int r = 0; r < CB; ++r) extra += sm[SM_P2 + r * DP + c];
                sm[SM_KD + (CB - 1) * DP + c] += extra;
                float run = 0.f;
                for (int r = CB - 1; r >= 0; --r) {
                    run += sm[SM_KD + r * DP + c];
                    sm[SM_KD + r * DP + c] = run;
                }
            }
            __syncthreads();
            {
                // this CTA's share of dq, dk, dg (dG is with respect to the natural-log decay, as is
                // dg); channels (t & 15) + 16 e, so a warp's atomics cover two 64-byte runs
                const int r = t >> 4;
                if (r < L) {
                    const size_t off = ((static_cast<size_t>(t0) + r) * H + u.h) * D;
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int c = (t & 15) + 16 * e;
                        atomicAdd(&p.dq[off + c], sm[SM_P1 + r * DP + c]);
                        atomicAdd(&p.dk[off + c], sm[SM_P3 + r * DP + c]);
                        // a log-decay raised to the floor has no gradient
                        const float dg = p.g[off + c] * kLog2e >= kFloorLog2 ? sm[SM_KD + r * DP + c] : 0.f;
                        atomicAdd(&p.dg[off + c], dg);
                    }
                }
            }
            __syncthreads();
        }
    }
    // the gradient of the initial state
    if (p.dh0) {
        float *dst = state_at(p.dh0, u.s);
        for (int e = t; e < D * VS; e += NT) {
            const int c = e / VS, j = e % VS;
            dst[static_cast<size_t>(c) * D + j] = dS[c * VP + j];
        }
    }
}

}  // namespace bwd

size_t bwd_workspace_bytes(int64_t rows, int64_t num_seqs, int32_t num_heads) {
    const int64_t slots = rows / bwd::GRP + num_seqs + 1;
    return static_cast<size_t>(slots) * num_heads * kHeadDim * kHeadDim * sizeof(float);
}

cudaError_t launch_bwd(const BwdParams &p, cudaStream_t stream) {
    const int64_t ctas = static_cast<int64_t>(p.num_seqs) * p.num_heads * bwd::NV;
    if (ctas == 0) return cudaSuccess;
    if (ctas > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    cudaError_t err = cudaFuncSetAttribute(bwd::kda_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(bwd::SMEM_BYTES));
    if (err != cudaSuccess) return err;
    bwd::kda_bwd_kernel<<<static_cast<unsigned>(ctas), bwd::NT, bwd::SMEM_BYTES, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace kda
