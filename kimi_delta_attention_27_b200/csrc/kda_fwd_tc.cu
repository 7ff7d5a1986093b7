// kda_fwd_tc.cu -- tensor-core (tcgen05 / TMEM / TMA) chunkwise KDA forward for sm_100a.
//
// Method: the recurrence of the Kimi Linear feature page (chapter 4, state-update
// equation), evaluated in chunks of C = 64 tokens in the chunk-parallel form the
// page's DPLR remark allows when both low-rank factors are bound to k. Per chunk,
// with G the in-chunk running log-decay per key channel and an anchor row a = 31:
//
//   Kh = K e^(G-Ga), Qh = Q e^(G-Ga), Kc = K e^(Ga-G)      (anchored, bf16)
//   Kt = K e^(Gl-G)                                         (decayed keys, fp16)
//   [Akk_raw; Aqk] = [Kh; Qh] Kc^T                          (S2, one M=128 MMA)
//   Akk = strict_lower(diag(beta) Akk_raw), Aqk = lower(Aqk)
//   T' = (I + Akk)^-1 diag(beta)                            (S3, blocked substitution)
//   W' = T' Kh;  W = W' diag(e^Ga)                          (S4)
//   Qt = (Qh - Aqk W') diag(e^Ga)                           (output read-out folded with the
//                                                            intra-chunk attention)
//   AV = [T'; Aqk T']                                       (S4, value side)
//   X  = [-W; Qt] S + AV V        ->  X[0:64] = D (pseudo-values), X[64:128] = O / scale   (S5 + S6)
//   S <- diag(e^Gl) S + Kt^T D                              (S7)
//
// Layout on the GPU: one cluster of 4 CTAs per (sequence, head); CTA r owns value
// columns [32 r, 32 r + 32) of the state, its output slice and the state-dependent
// chain (S5-S7) for them. The state-independent work of a chunk (S1-S4) depends on
// q, k, g, beta only, so chunk n is prepared by CTA n % 4 alone, which then pushes
// the finished operand tiles (64.5 KB) into a slot of every CTA's shared memory by
// bulk copies; each CTA reads q, k, g for a quarter of the chunks and v for its own
// slice, so every input byte crosses HBM once.
//
// Warp roles (384 threads): w0 value-slice TMA, w1 chain MMA issuer, w2 prep MMA
// issuer, w3 prep TMA, w4-7 chain epilogue (TMEM lanes = state rows / chunk rows),
// w8-11 chunk preparation (elementwise gates, UT solve, epilogues).
//
// Precision: anchored factors (Kh, Qh, Kc), W, Qt and the state copy S' are bf16;
// T', AV, the value slice, Kt and D are fp16 (10-bit mantissa) because the state
// update is most sensitive to them; every product accumulates in fp32 (TMEM) and the
// state itself is carried in fp32 registers.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include "kda_internal.h"
#include "sm100_ptx.cuh"

namespace kda {

__device__ unsigned int g_kda_device_error = 0;

#ifdef KDA_TRACE
// Development-only timeline: when built with -DKDA_TRACE, the first cluster
// records %globaltimer at fixed points per chunk into g_kda_trace
// [rank][chunk < 64][point < 16]. The product build compiles none of this.
__device__ unsigned long long g_kda_trace[4 * 64 * 16];
#define KDA_TRACE_POINT(chunk, point)                                                               \
    do {                                                                                            \
        if (blockIdx.x < 4 && (chunk) < 64)                                                         \
            g_kda_trace[(rank * 64 + (chunk)) * 16 + (point)] = ptx::globaltimer();                 \
    } while (0)
#else
#define KDA_TRACE_POINT(chunk, point) \
    do {                              \
    } while (0)
#endif

namespace tc {

using namespace ptx;

constexpr int D = kHeadDim;
constexpr int C = kChunk;
constexpr int NS = 4;          // CTAs per cluster = value slices
constexpr int NV = D / NS;     // 32 value columns per CTA
constexpr int NTHREADS = 384;
constexpr int ANCHOR = 31;

// ---- shared memory map (byte offsets from a 1024-aligned base)
constexpr uint32_t SLOT_BYTES = 65536;
constexpr uint32_t SLOT_KT = 0, SLOT_W = 16384, SLOT_Q = 32768, SLOT_AV = 49152;
constexpr uint32_t OFF_DEC = 2 * SLOT_BYTES;       // e^Gl per slot, 128 fp32
constexpr uint32_t DEC_BYTES = 512;
constexpr uint32_t SLOT_TX = 4 * 16384 + DEC_BYTES;
constexpr uint32_t OFF_STAGE = OFF_DEC + 1024;     // q, k, g staging; then UT workspace
constexpr uint32_t STG_Q = 0, STG_K = 16384, STG_G = 32768, STAGE_TX = 65536;
constexpr uint32_t AKK_LD = 68;                    // fp32 row stride (floats) of A and T
constexpr uint32_t WS_AKK = 0, WS_T = 17408, WS_P = 34816, WS_TB = 0, WS_AQB = 40960, WS_WP = 49152;
constexpr uint32_t OFF_SP = OFF_STAGE + 65536;     // S' [128 x 32] bf16, MN-major SW64
constexpr uint32_t OFF_DL = OFF_SP + 8192;         // D  [64 x 32] fp16, MN-major SW64
constexpr uint32_t OFF_V = OFF_DL + 4096;          // V  2 x [64 x 32], SW64
constexpr uint32_t OFF_MISC = OFF_V + 8192;
constexpr uint32_t OFF_BAR = OFF_MISC;             // 32 mbarriers
constexpr uint32_t OFF_BETA = OFF_BAR + 256;       // 64 fp32
constexpr uint32_t OFF_EGA = OFF_BETA + 256;       // 128 fp32
constexpr uint32_t OFF_TMEMPTR = OFF_EGA + 512;
constexpr uint32_t OFF_ABORT = OFF_TMEMPTR + 16;
constexpr uint32_t SMEM_USED = OFF_ABORT + 16;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;  // + alignment slack

// barrier indices
enum {
    B_SLOT_FULL = 0,   // 2
    B_SLOT_EMPTY = 2,  // 2
    B_VFULL = 4,       // 2
    B_VCONV = 6,       // 2
    B_VFREE = 8,       // 2
    B_C1_FULL = 10, B_C1_FREE, B_S_READY, B_D_READY, B_C3_FULL,
    B_STAGE_FULL, B_STAGE_FREE, B_EW_DONE, B_P1_DONE, B_SOLVE_DONE, B_WAV_DONE, B_WEPI_DONE, B_Q_DONE,
    B_COUNT
};
static_assert(B_COUNT * 8 <= 256, "barrier area");

// ---- TMEM columns
constexpr uint32_t COL_P1 = 0, COL_W = 64, COL_AV = 128, COL_Q = 192, COL_C1 = 256, COL_C3 = 288;
constexpr uint32_t TMEM_COLS = 512;

// ---- instruction descriptors (M = 128)
constexpr uint32_t ID_P1 = idesc_f16(128, 64, 1, 1, 1);     // bf16, A MN-major, B MN-major
constexpr uint32_t ID_W = idesc_f16(128, 64, 1, 0, 0);      // bf16, K-major / K-major
constexpr uint32_t ID_AV = idesc_f16(128, 64, 0, 0, 1);     // fp16, K-major / MN-major
constexpr uint32_t ID_Q = idesc_f16(128, 64, 1, 0, 0);      // bf16
constexpr uint32_t ID_VPART = idesc_f16(128, NV, 0, 0, 1);  // fp16, A K-major, B MN-major
constexpr uint32_t ID_STATE = idesc_f16(128, NV, 1, 1, 1);  // bf16, A MN-major, B MN-major
constexpr uint32_t ID_C3 = idesc_f16(128, NV, 0, 0, 1);     // fp16

constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s: far above any legitimate wait

struct TmaMaps {
    CUtensorMap q, k, g, v;
};

__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile uint32_t *abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    for (;;) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer() - t0 > kWaitLimitNs) {
            *abort_flag = 1;
            atomicOr(&g_kda_device_error, 1u);
            return false;
        }
    }
}

__device__ __forceinline__ float bf2f(uint16_t x) { return __uint_as_float(static_cast<uint32_t>(x) << 16); }

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
}
__device__ __forceinline__ uint32_t pack_f16(float a, float b) {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
}

// byte offset of 16-byte chunk j of row r in a tile of 128-byte rows, 128B swizzle
__device__ __forceinline__ uint32_t sw128(uint32_t r, uint32_t j) { return r * 128u + ((j ^ (r & 7u)) << 4); }
// byte offset of 16-byte chunk j of row r in a tile of 64-byte rows, 64B swizzle
__device__ __forceinline__ uint32_t sw64(uint32_t r, uint32_t j) { return r * 64u + ((j ^ ((r >> 1) & 3u)) << 4); }

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
                 : "memory");
}
__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}

__global__ void __launch_bounds__(NTHREADS, 1)
    kda_fwd_tc_kernel(const FwdParams p, const __grid_constant__ TmaMaps maps) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = raw + ((1024u - (raw & 1023u)) & 1023u);
    unsigned char *sgen = smem_raw + (sbase - raw);
    const uint32_t bar0 = sbase + OFF_BAR;
    auto BAR = [&](int i) -> uint32_t { return bar0 + 8u * static_cast<uint32_t>(i); };
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(sgen + OFF_ABORT);
    float *beta_s = reinterpret_cast<float *>(sgen + OFF_BETA);
    float *ega_s = reinterpret_cast<float *>(sgen + OFF_EGA);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = cluster_ctarank();
    const int H = p.num_heads;
    const int64_t unit = blockIdx.x / NS;
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
    const int nch = static_cast<int>((eos - bos + C - 1) / C);
    const int v0 = static_cast<int>(rank) * NV;
    const size_t state_base = (static_cast<size_t>(s) * H + h) * D * D;

    // ---------------------------------------------------------------- setup
    if (tid == 0) {
        mbar_init(BAR(B_SLOT_FULL + 0), 1);
        mbar_init(BAR(B_SLOT_FULL + 1), 1);
        mbar_init(BAR(B_SLOT_EMPTY + 0), NS);
        mbar_init(BAR(B_SLOT_EMPTY + 1), NS);
        for (int b = 0; b < 2; ++b) {
            mbar_init(BAR(B_VFULL + b), 1);
            mbar_init(BAR(B_VCONV + b), 4);
            mbar_init(BAR(B_VFREE + b), 1);
        }
        mbar_init(BAR(B_C1_FULL), 1);
        mbar_init(BAR(B_C1_FREE), 4);
        mbar_init(BAR(B_S_READY), 4);
        mbar_init(BAR(B_D_READY), 2);
        mbar_init(BAR(B_C3_FULL), 1);
        mbar_init(BAR(B_STAGE_FULL), 1);
        mbar_init(BAR(B_STAGE_FREE), 1);
        mbar_init(BAR(B_EW_DONE), 1);
        mbar_init(BAR(B_P1_DONE), 1);
        mbar_init(BAR(B_SOLVE_DONE), 1);
        mbar_init(BAR(B_WAV_DONE), 1);
        mbar_init(BAR(B_WEPI_DONE), 1);
        mbar_init(BAR(B_Q_DONE), 1);
        *abort_flag = 0;
        fence_mbar_init();
        // the first two chunks' slots start free: arm them for the bytes a peer will push
        for (int n = 0; n < 2 && n < nch; ++n)
            if (n % NS != static_cast<int>(rank)) mbar_expect_tx(BAR(B_SLOT_FULL + (n & 1)), SLOT_TX);
    }
    if (warp == 2) {
        tmem_alloc(sbase + OFF_TMEMPTR, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    cluster_arrive();
    cluster_wait();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sgen + OFF_TMEMPTR);

    if (warp == 0) {
        // ============================================================ value-slice TMA
        for (int n = 0; n < nch; ++n) {
            const int b = n & 1;
            if (n >= 2 && !wait_bar(BAR(B_VFREE + b), ((n - 2) >> 1) & 1, abort_flag)) break;
            if (lane == 0) {
                mbar_arrive_expect_tx(BAR(B_VFULL + b), 4096);
                tma_load_3d(sbase + OFF_V + b * 4096, &maps.v, BAR(B_VFULL + b), v0, h,
                            static_cast<int32_t>(bos + static_cast<int64_t>(n) * C));
            }
            __syncwarp();
        }
    } else if (warp == 3) {
        // ============================================================ prep TMA (q, k, g)
        int kk = 0;
        for (int m = static_cast<int>(rank); m < nch; m += NS, ++kk) {
            if (kk >= 1 && !wait_bar(BAR(B_STAGE_FREE), (kk - 1) & 1, abort_flag)) break;
            if (lane == 0) {
                const int32_t row = static_cast<int32_t>(bos + static_cast<int64_t>(m) * C);
                mbar_arrive_expect_tx(BAR(B_STAGE_FULL), STAGE_TX);
                tma_load_3d(sbase + OFF_STAGE + STG_Q, &maps.q, BAR(B_STAGE_FULL), 0, h, row);
                tma_load_3d(sbase + OFF_STAGE + STG_K, &maps.k, BAR(B_STAGE_FULL), 0, h, row);
                tma_load_3d(sbase + OFF_STAGE + STG_G, &maps.g, BAR(B_STAGE_FULL), 0, h, row);
            }
            __syncwarp();
        }
    } else if (warp == 1) {
        // ============================================================ chain MMA issuer
        for (int n = 0; n < nch; ++n) {
            const int sl = n & 1, b = n & 1;
            const uint32_t slot = sbase + sl * SLOT_BYTES;
            if (!wait_bar(BAR(B_SLOT_FULL + sl), (n >> 1) & 1, abort_flag)) break;
            if (lane == 0) KDA_TRACE_POINT(n, 12);
            if (!wait_bar(BAR(B_VCONV + b), (n >> 1) & 1, abort_flag)) break;
            if (n >= 1 && !wait_bar(BAR(B_C1_FREE), (n - 1) & 1, abort_flag)) break;
            tc_fence_after();
            if (lane == 0) {
                // value part: [T'; Aqk T'] * V   (fp16)
                for (int ks = 0; ks < 4; ++ks)
                    mma_f16(tmem + COL_C1, smem_desc(slot + SLOT_AV + ks * 32, 16, 1024, kSwizzle128),
                            smem_desc(sbase + OFF_V + b * 4096 + ks * 1024, 4096, 512, kSwizzle64), ID_VPART,
                            ks > 0);
                mma_commit(BAR(B_VFREE + b));
            }
            __syncwarp();
            if (!wait_bar(BAR(B_S_READY), n & 1, abort_flag)) break;
            tc_fence_after();
            if (lane == 0) KDA_TRACE_POINT(n, 13);
            if (lane == 0) {
                // state part: [-W; Qt] * S'   (bf16)
                for (int ks = 0; ks < 8; ++ks)
                    mma_f16(tmem + COL_C1, smem_desc(slot + SLOT_W + ks * 2048, 16384, 1024, kSwizzle128),
                            smem_desc(sbase + OFF_SP + ks * 1024, 4096, 512, kSwizzle64), ID_STATE, 1);
                mma_commit(BAR(B_C1_FULL));
            }
            __syncwarp();
            if (!wait_bar(BAR(B_D_READY), n & 1, abort_flag)) break;
            tc_fence_after();
            if (lane == 0) {
                // state increment: Kt^T * D   (fp16)
                for (int ks = 0; ks < 4; ++ks)
                    mma_f16(tmem + COL_C3, smem_desc(slot + SLOT_KT + ks * 32, 16, 1024, kSwizzle128),
                            smem_desc(sbase + OFF_DL + ks * 1024, 4096, 512, kSwizzle64), ID_C3, ks > 0);
                mma_commit(BAR(B_C3_FULL));
            }
            __syncwarp();
        }
    } else if (warp == 2) {
        // ============================================================ prep MMA issuer
        int kk = 0;
        for (int m = static_cast<int>(rank); m < nch; m += NS, ++kk) {
            const uint32_t slot = sbase + (m & 1) * SLOT_BYTES;
            const uint32_t ws = sbase + OFF_STAGE;
            if (!wait_bar(BAR(B_EW_DONE), kk & 1, abort_flag)) break;
            tc_fence_after();
            if (lane == 0) {
                // [Kh; Qh] Kc^T : A = Kh^T | Qh^T (MN-major, 64-row blocks 16 KB apart), B = Kc^T
                for (int ks = 0; ks < 8; ++ks)
                    mma_f16(tmem + COL_P1, smem_desc(slot + SLOT_W + ks * 2048, 16384, 1024, kSwizzle128),
                            smem_desc(slot + SLOT_AV + ks * 2048, 16384, 1024, kSwizzle128), ID_P1, ks > 0);
                mma_commit(BAR(B_P1_DONE));
            }
            __syncwarp();
            if (!wait_bar(BAR(B_SOLVE_DONE), kk & 1, abort_flag)) break;
            tc_fence_after();
            if (lane == 0) {
                // W'^T = Kh^T T'^T (bf16)
                for (int ks = 0; ks < 4; ++ks)
                    mma_f16(tmem + COL_W, smem_desc(slot + SLOT_W + ks * 32, 16, 1024, kSwizzle128),
                            smem_desc(ws + WS_TB + ks * 32, 16, 1024, kSwizzle128), ID_W, ks > 0);
                // [T'; Aqk] T' (fp16); only rows 64..127 (Aqk T') are used
                for (int ks = 0; ks < 4; ++ks)
                    mma_f16(tmem + COL_AV, smem_desc(slot + SLOT_AV + ks * 32, 16, 1024, kSwizzle128),
                            smem_desc(slot + SLOT_AV + ks * 2048, 16384, 1024, kSwizzle128), ID_AV, ks > 0);
                mma_commit(BAR(B_WAV_DONE));
            }
            __syncwarp();
            if (!wait_bar(BAR(B_WEPI_DONE), kk & 1, abort_flag)) break;
            tc_fence_after();
            if (lane == 0) {
                // W'^T Aqk^T (bf16)
                for (int ks = 0; ks < 4; ++ks)
                    mma_f16(tmem + COL_Q, smem_desc(ws + WS_WP + ks * 32, 16, 1024, kSwizzle128),
                            smem_desc(ws + WS_AQB + ks * 32, 16, 1024, kSwizzle128), ID_Q, ks > 0);
                mma_commit(BAR(B_Q_DONE));
            }
            __syncwarp();
        }
    } else if (warp < 8) {
        // ============================================================ chain epilogue (w4..w7)
        const int t = tid - 128;               // TMEM lane = state row k = chunk row for C1
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        float S[NV];
        if (p.h0) {
            const size_t off = state_base + static_cast<size_t>(t) * D + v0;
            if (p.h0_fp32) {
                const float4 *src = reinterpret_cast<const float4 *>(static_cast<const float *>(p.h0) + off);
#pragma unroll
                for (int j = 0; j < NV / 4; ++j) {
                    float4 x = src[j];
                    S[4 * j] = x.x; S[4 * j + 1] = x.y; S[4 * j + 2] = x.z; S[4 * j + 3] = x.w;
                }
            } else {
                const uint4 *src = reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(p.h0) + off);
#pragma unroll
                for (int j = 0; j < NV / 8; ++j) {
                    uint4 x = src[j];
                    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        S[8 * j + 2 * e] = __uint_as_float(w[e] << 16);
                        S[8 * j + 2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
                    }
                }
            }
        } else {
#pragma unroll
            for (int j = 0; j < NV; ++j) S[j] = 0.f;
        }
        auto write_sprime = [&]() {
#pragma unroll
            for (int j = 0; j < 4; ++j)
                st_shared_v4(sbase + OFF_SP + sw64(t, j), pack_bf16(S[8 * j], S[8 * j + 1]),
                             pack_bf16(S[8 * j + 2], S[8 * j + 3]), pack_bf16(S[8 * j + 4], S[8 * j + 5]),
                             pack_bf16(S[8 * j + 6], S[8 * j + 7]));
        };
        auto convert_v = [&](int n) -> bool {
            const int b = n & 1;
            if (!wait_bar(BAR(B_VFULL + b), (n >> 1) & 1, abort_flag)) return false;
#pragma unroll
            for (int c2 = 0; c2 < 2; ++c2) {
                const uint32_t a = sbase + OFF_V + b * 4096 + (t + 128 * c2) * 16;
                uint4 x = ld_shared_v4(a);
                uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    w[e] = pack_f16(__uint_as_float(w[e] << 16), __uint_as_float(w[e] & 0xFFFF0000u));
                st_shared_v4(a, w[0], w[1], w[2], w[3]);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(BAR(B_VCONV + b));
            return true;
        };
        write_sprime();
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(B_S_READY));
        bool ok = nch > 0 ? convert_v(0) : true;
        for (int n = 0; ok && n < nch; ++n) {
            const int sl = n & 1;
            const int64_t t0 = bos + static_cast<int64_t>(n) * C;
            const int L = static_cast<int>(eos - t0 < C ? eos - t0 : C);
            if (!wait_bar(BAR(B_C1_FULL), n & 1, abort_flag)) break;
            tc_fence_after();
            if (t == 0) KDA_TRACE_POINT(n, 9);
            uint32_t r[32];
            tmem_ld32(tmem + lane_base + COL_C1, r);
            tmem_wait_ld();
            if (t < 64) {
                // pseudo-values D (row t of the chunk) -> fp16 B operand of the state increment
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    st_shared_v4(sbase + OFF_DL + sw64(t, j),
                                 pack_f16(__uint_as_float(r[8 * j]), __uint_as_float(r[8 * j + 1])),
                                 pack_f16(__uint_as_float(r[8 * j + 2]), __uint_as_float(r[8 * j + 3])),
                                 pack_f16(__uint_as_float(r[8 * j + 4]), __uint_as_float(r[8 * j + 5])),
                                 pack_f16(__uint_as_float(r[8 * j + 6]), __uint_as_float(r[8 * j + 7])));
                fence_proxy_async_smem();
            } else {
                const int rr = t - 64;
                if (rr < L) {
                    uint4 *dst = reinterpret_cast<uint4 *>(p.out + ((t0 + rr) * H + h) * D + v0);
                    const float sc = p.scale;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        uint4 o;
                        o.x = pack_bf16(sc * __uint_as_float(r[8 * j]), sc * __uint_as_float(r[8 * j + 1]));
                        o.y = pack_bf16(sc * __uint_as_float(r[8 * j + 2]), sc * __uint_as_float(r[8 * j + 3]));
                        o.z = pack_bf16(sc * __uint_as_float(r[8 * j + 4]), sc * __uint_as_float(r[8 * j + 5]));
                        o.w = pack_bf16(sc * __uint_as_float(r[8 * j + 6]), sc * __uint_as_float(r[8 * j + 7]));
                        dst[j] = o;
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(BAR(B_C1_FREE));
                if (t < 64) mbar_arrive(BAR(B_D_READY));
            }
            if (n + 1 < nch && !convert_v(n + 1)) break;
            if (!wait_bar(BAR(B_C3_FULL), n & 1, abort_flag)) break;
            tc_fence_after();
            if (t == 0) KDA_TRACE_POINT(n, 10);
            tmem_ld32(tmem + lane_base + COL_C3, r);
            tmem_wait_ld();
            const float dec = reinterpret_cast<const float *>(sgen + OFF_DEC + sl * DEC_BYTES)[t];
#pragma unroll
            for (int j = 0; j < NV; ++j) S[j] = fmaf(dec, S[j], __uint_as_float(r[j]));
            if (n + 1 < nch) {
                write_sprime();
                fence_proxy_async_smem();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0 && n + 1 < nch) mbar_arrive(BAR(B_S_READY));
            // hand slot `sl` on to the producer of chunk n + 2 once all four warps are done with it
            named_bar_sync(1, 128);
            if (t == 0) KDA_TRACE_POINT(n, 11);
            if (t == 0 && n + 2 < nch) {
                const uint32_t prod = static_cast<uint32_t>((n + 2) % NS);
                if (prod != rank) mbar_expect_tx(BAR(B_SLOT_FULL + sl), SLOT_TX);
                mbar_arrive_remote(mapa(BAR(B_SLOT_EMPTY + sl), prod));
            }
        }
        // final state slice
        if (p.hT && !*abort_flag) {
            const size_t off = state_base + static_cast<size_t>(t) * D + v0;
            if (p.hT_fp32) {
                float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(p.hT) + off);
#pragma unroll
                for (int j = 0; j < NV / 4; ++j) dst[j] = make_float4(S[4 * j], S[4 * j + 1], S[4 * j + 2], S[4 * j + 3]);
            } else {
                uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(p.hT) + off);
#pragma unroll
                for (int j = 0; j < NV / 8; ++j)
                    dst[j] = make_uint4(pack_bf16(S[8 * j], S[8 * j + 1]), pack_bf16(S[8 * j + 2], S[8 * j + 3]),
                                        pack_bf16(S[8 * j + 4], S[8 * j + 5]), pack_bf16(S[8 * j + 6], S[8 * j + 7]));
            }
        }
    } else {
        // ============================================================ chunk preparation (w8..w11)
        const int t = tid - 256;               // key channel in the gate pass; TMEM lane in epilogues
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t ws = sbase + OFF_STAGE;
        float *wsf = reinterpret_cast<float *>(sgen + OFF_STAGE);
        int kk = 0;
        for (int m = static_cast<int>(rank); m < nch; m += NS, ++kk) {
            const int sl = m & 1;
            const uint32_t slot = sbase + sl * SLOT_BYTES;
            const int64_t t0 = bos + static_cast<int64_t>(m) * C;
            const int L = static_cast<int>(eos - t0 < C ? eos - t0 : C);
            // my slot must have been released by every CTA (chunk m - 2)
            if (m >= 2) {
                const int j = static_cast<int>(rank) >= 2 ? kk : kk - 1;
                if (!wait_bar(BAR(B_SLOT_EMPTY + sl), j & 1, abort_flag)) break;
            }
            if (t == 0) KDA_TRACE_POINT(m, 0);
            if (t < C) beta_s[t] = t < L ? p.beta[(t0 + t) * H + h] : 0.f;
            if (!wait_bar(BAR(B_STAGE_FULL), kk & 1, abort_flag)) break;
            named_bar_sync(2, 128);
            if (t == 0) KDA_TRACE_POINT(m, 1);

            // -------- S1: running log-decay of channel t, decayed factors (T-format tiles)
            {
                const int c = t;
                const float *gcol = reinterpret_cast<const float *>(sgen + OFF_STAGE + STG_G) + c;
                const uint16_t *qcol = reinterpret_cast<const uint16_t *>(sgen + OFF_STAGE + STG_Q) + c;
                const uint16_t *kcol = reinterpret_cast<const uint16_t *>(sgen + OFF_STAGE + STG_K) + c;
                float ga = 0.f, gl = 0.f;
                for (int r = 0; r < L; ++r) {
                    gl += gcol[r * D];
                    if (r == ANCHOR) ga = gl;
                }
                if (L <= ANCHOR) ga = gl;
                const float eca = __expf(gl - ga);
                float G = 0.f;
#pragma unroll 1
                for (int rb = 0; rb < 8; ++rb) {
                    uint32_t ph[4], pq[4], pc[4], pt[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        float kh[2], qh[2], kc[2], kt[2];
#pragma unroll
                        for (int u = 0; u < 2; ++u) {
                            const int r = rb * 8 + 2 * e + u;
                            const bool valid = r < L;
                            G += valid ? gcol[r * D] : 0.f;
                            const float x = G - ga;
                            const float ep = __expf(x), em = __expf(-x);
                            const float kv = valid ? bf2f(kcol[r * D]) : 0.f;
                            const float qv = valid ? bf2f(qcol[r * D]) : 0.f;
                            kh[u] = kv * ep;
                            qh[u] = qv * ep;
                            kc[u] = kv * em;
                            kt[u] = kc[u] * eca;
                        }
                        ph[e] = pack_bf16(kh[0], kh[1]);
                        pq[e] = pack_bf16(qh[0], qh[1]);
                        pc[e] = pack_bf16(kc[0], kc[1]);
                        pt[e] = pack_f16(kt[0], kt[1]);
                    }
                    const uint32_t o = sw128(c, rb);
                    st_shared_v4(slot + SLOT_W + o, ph[0], ph[1], ph[2], ph[3]);   // Kh^T (scratch)
                    st_shared_v4(slot + SLOT_Q + o, pq[0], pq[1], pq[2], pq[3]);   // Qh^T (scratch)
                    st_shared_v4(slot + SLOT_AV + o, pc[0], pc[1], pc[2], pc[3]);  // Kc^T (scratch)
                    st_shared_v4(slot + SLOT_KT + o, pt[0], pt[1], pt[2], pt[3]);  // Kt^T
                }
                reinterpret_cast<float *>(sgen + OFF_DEC + sl * DEC_BYTES)[c] = __expf(gl);
                ega_s[c] = __expf(ga);
            }
            fence_proxy_async_smem();
            named_bar_sync(2, 128);
            if (t == 0) { mbar_arrive(BAR(B_EW_DONE)); KDA_TRACE_POINT(m, 2); }

            // -------- S2 epilogue: A (fp32, masked, beta-scaled) and Aqk (fp16 + bf16)
            if (!wait_bar(BAR(B_P1_DONE), kk & 1, abort_flag)) break;
            tc_fence_after();
            if (t == 0) KDA_TRACE_POINT(m, 3);
            {
                uint32_t a0[32], a1[32];
                tmem_ld32(tmem + lane_base + COL_P1, a0);
                tmem_ld32(tmem + lane_base + COL_P1 + 32, a1);
                tmem_wait_ld();
                if (t < 64) {
                    const int r = t;
                    const float br = beta_s[r];
                    float *row = wsf + WS_AKK / 4 + r * AKK_LD;
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        float v4[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int i = 4 * j + e;
                            const float a = __uint_as_float(i < 32 ? a0[i] : a1[i - 32]);
                            v4[e] = i < r ? br * a : 0.f;
                        }
                        *reinterpret_cast<float4 *>(row + 4 * j) = make_float4(v4[0], v4[1], v4[2], v4[3]);
                    }
                } else {
                    const int r = t - 64;
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        float v8[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int i = 8 * j + e;
                            const float a = __uint_as_float(i < 32 ? a0[i] : a1[i - 32]);
                            v8[e] = i <= r ? a : 0.f;
                        }
                        st_shared_v4(slot + SLOT_AV + sw128(64 + r, j), pack_f16(v8[0], v8[1]),
                                     pack_f16(v8[2], v8[3]), pack_f16(v8[4], v8[5]), pack_f16(v8[6], v8[7]));
                        st_shared_v4(ws + WS_AQB + sw128(r, j), pack_bf16(v8[0], v8[1]), pack_bf16(v8[2], v8[3]),
                                     pack_bf16(v8[4], v8[5]), pack_bf16(v8[6], v8[7]));
                    }
                }
            }
            tc_fence_before();
            named_bar_sync(2, 128);

            // -------- S3: T = (I + A)^-1, blocked forward substitution on 16 x 16 blocks
            {
                const float *A = wsf + WS_AKK / 4;
                float *T = wsf + WS_T / 4;
                float *P = wsf + WS_P / 4;
                // diagonal blocks: warp w inverts block w, lane i < 16 owns column i
                const int wb = t >> 5, li = t & 31;
                if (li < 16) {
                    float x[16];
#pragma unroll
                    for (int r = 0; r < 16; ++r) {
                        float acc = (r == li) ? 1.f : 0.f;
                        const float *arow = A + (16 * wb + r) * AKK_LD + 16 * wb;
#pragma unroll
                        for (int j = 0; j < r; ++j) acc = fmaf(-arow[j], x[j], acc);
                        x[r] = acc;
                    }
#pragma unroll
                    for (int r = 0; r < 16; ++r) T[(16 * wb + r) * AKK_LD + 16 * wb + li] = x[r];
                }
                named_bar_sync(2, 128);
                // off-diagonal blocks by distance d = I - J: T_IJ = -T_II * sum_{K=J}^{I-1} A_IK T_KJ
#pragma unroll 1
                for (int d = 1; d < 4; ++d) {
                    const int nb = 4 - d;
                    for (int e = t; e < nb * 256; e += 128) {
                        const int J = e >> 8, I = J + d, r = (e >> 4) & 15, c = e & 15;
                        float acc = 0.f;
                        for (int K = J; K < I; ++K) {
                            const float *arow = A + (16 * I + r) * AKK_LD + 16 * K;
                            const float *tcol = T + (16 * K) * AKK_LD + 16 * J + c;
#pragma unroll
                            for (int j = 0; j < 16; ++j) acc = fmaf(arow[j], tcol[j * AKK_LD], acc);
                        }
                        P[J * 256 + r * 16 + c] = acc;
                    }
                    named_bar_sync(2, 128);
                    for (int e = t; e < nb * 256; e += 128) {
                        const int J = e >> 8, I = J + d, r = (e >> 4) & 15, c = e & 15;
                        const float *trow = T + (16 * I + r) * AKK_LD + 16 * I;
                        float acc = 0.f;
#pragma unroll
                        for (int j = 0; j < 16; ++j) acc = fmaf(trow[j], P[J * 256 + j * 16 + c], acc);
                        T[(16 * I + r) * AKK_LD + 16 * J + c] = -acc;
                    }
                    named_bar_sync(2, 128);
                }
                // T' = T diag(beta): fp16 into the slot's AV rows 0..63, bf16 into the workspace
                {
                    const int r = t >> 1, half = t & 1;
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        const int j = half * 4 + jj;
                        float v8[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int i = 8 * j + e;
                            v8[e] = i <= r ? T[r * AKK_LD + i] * beta_s[i] : 0.f;
                        }
                        st_shared_v4(slot + SLOT_AV + sw128(r, j), pack_f16(v8[0], v8[1]), pack_f16(v8[2], v8[3]),
                                     pack_f16(v8[4], v8[5]), pack_f16(v8[6], v8[7]));
                        // WS_TB overlays the fp32 A block; A is no longer read after the barrier above
                        st_shared_v4(ws + WS_TB + sw128(r, j), pack_bf16(v8[0], v8[1]), pack_bf16(v8[2], v8[3]),
                                     pack_bf16(v8[4], v8[5]), pack_bf16(v8[6], v8[7]));
                    }
                }
            }
            fence_proxy_async_smem();
            named_bar_sync(2, 128);
            if (t == 0) { mbar_arrive(BAR(B_SOLVE_DONE)); KDA_TRACE_POINT(m, 4); }

            // -------- S4 epilogues: W (anchored copy + final negated/unanchored), Aqk T'
            if (!wait_bar(BAR(B_WAV_DONE), kk & 1, abort_flag)) break;
            tc_fence_after();
            if (t == 0) KDA_TRACE_POINT(m, 5);
            {
                uint32_t a0[32], a1[32];
                tmem_ld32(tmem + lane_base + COL_W, a0);
                tmem_ld32(tmem + lane_base + COL_W + 32, a1);
                tmem_wait_ld();
                const float sc = -ega_s[t];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    float v8[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) v8[e] = __uint_as_float(j < 4 ? a0[8 * j + e] : a1[8 * (j - 4) + e]);
                    st_shared_v4(ws + WS_WP + sw128(t, j), pack_bf16(v8[0], v8[1]), pack_bf16(v8[2], v8[3]),
                                 pack_bf16(v8[4], v8[5]), pack_bf16(v8[6], v8[7]));
                    st_shared_v4(slot + SLOT_W + sw128(t, j), pack_bf16(sc * v8[0], sc * v8[1]),
                                 pack_bf16(sc * v8[2], sc * v8[3]), pack_bf16(sc * v8[4], sc * v8[5]),
                                 pack_bf16(sc * v8[6], sc * v8[7]));
                }
                if (t >= 64) {
                    tmem_ld32(tmem + lane_base + COL_AV, a0);
                    tmem_ld32(tmem + lane_base + COL_AV + 32, a1);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        float v8[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            v8[e] = __uint_as_float(j < 4 ? a0[8 * j + e] : a1[8 * (j - 4) + e]);
                        st_shared_v4(slot + SLOT_AV + sw128(t, j), pack_f16(v8[0], v8[1]), pack_f16(v8[2], v8[3]),
                                     pack_f16(v8[4], v8[5]), pack_f16(v8[6], v8[7]));
                    }
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar_sync(2, 128);
            if (t == 0) { mbar_arrive(BAR(B_WEPI_DONE)); KDA_TRACE_POINT(m, 6); }

            // -------- Qt = (Qh - Aqk W') e^Ga, row t of Qt^T, in place over Qh^T
            if (!wait_bar(BAR(B_Q_DONE), kk & 1, abort_flag)) break;
            tc_fence_after();
            if (t == 0) KDA_TRACE_POINT(m, 7);
            {
                uint32_t a0[32], a1[32];
                tmem_ld32(tmem + lane_base + COL_Q, a0);
                tmem_ld32(tmem + lane_base + COL_Q + 32, a1);
                tmem_wait_ld();
                const float sc = ega_s[t];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const uint4 qv = ld_shared_v4(slot + SLOT_Q + sw128(t, j));
                    const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w};
                    uint32_t o[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float c0 = __uint_as_float(j < 4 ? a0[8 * j + 2 * e] : a1[8 * (j - 4) + 2 * e]);
                        const float c1 = __uint_as_float(j < 4 ? a0[8 * j + 2 * e + 1] : a1[8 * (j - 4) + 2 * e + 1]);
                        const float q0 = __uint_as_float(qw[e] << 16), q1 = __uint_as_float(qw[e] & 0xFFFF0000u);
                        o[e] = pack_bf16(sc * (q0 - c0), sc * (q1 - c1));
                    }
                    st_shared_v4(slot + SLOT_Q + sw128(t, j), o[0], o[1], o[2], o[3]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar_sync(2, 128);
            if (t == 0) {
                mbar_arrive(BAR(B_STAGE_FREE));
                // publish the slot: bulk copies to the three peers, then one arrival each
                const uint32_t full = BAR(B_SLOT_FULL + sl);
                for (uint32_t pr = 0; pr < NS; ++pr) {
                    if (pr == rank) continue;
                    const uint32_t rfull = mapa(full, pr);
                    for (uint32_t part = 0; part < 4; ++part)
                        bulk_copy_to_peer(mapa(slot + part * 16384, pr), slot + part * 16384, 16384, rfull);
                    bulk_copy_to_peer(mapa(sbase + OFF_DEC + sl * DEC_BYTES, pr), sbase + OFF_DEC + sl * DEC_BYTES,
                                      DEC_BYTES, rfull);
                    mbar_arrive_remote(rfull);
                }
                mbar_arrive(full);
                KDA_TRACE_POINT(m, 8);
            }
        }
    }

    // ---------------------------------------------------------------- teardown
    if (*abort_flag) {
        // let any copy still in flight land before the CTA's memory is released
        const uint64_t t0 = globaltimer();
        while (globaltimer() - t0 < 20000000ull) {
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 2) tmem_dealloc(tmem, TMEM_COLS);
    cluster_arrive();
    cluster_wait();
}

}  // namespace tc

// ---------------------------------------------------------------- host side
namespace {

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

bool encode3d(CUtensorMap *map, const void *base, CUtensorMapDataType dt, uint32_t esize, int H, int64_t rows,
              uint32_t box0, CUtensorMapSwizzle swz) {
    auto enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(kHeadDim), static_cast<cuuint64_t>(H),
                          static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(kHeadDim) * esize,
                             static_cast<cuuint64_t>(kHeadDim) * esize * static_cast<cuuint64_t>(H)};
    cuuint32_t box[3] = {box0, 1, static_cast<cuuint32_t>(kChunk)};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, dt, 3, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_fwd_tc(const FwdParams &p, int64_t rows, cudaStream_t stream) {
    const int64_t units = static_cast<int64_t>(p.num_seqs) * p.num_heads;
    if (units == 0) return cudaSuccess;
    const int64_t grid = units * tc::NS;
    if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    tc::TmaMaps maps;
    memset(&maps, 0, sizeof(maps));
    if (rows > 0) {
        if (rows > 0x7fffffffLL) return cudaErrorInvalidValue;
        if (!encode3d(&maps.q, p.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.num_heads, rows, 128,
                      CU_TENSOR_MAP_SWIZZLE_NONE) ||
            !encode3d(&maps.k, p.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.num_heads, rows, 128,
                      CU_TENSOR_MAP_SWIZZLE_NONE) ||
            !encode3d(&maps.g, p.g, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, p.num_heads, rows, 128,
                      CU_TENSOR_MAP_SWIZZLE_NONE) ||
            !encode3d(&maps.v, p.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.num_heads, rows, tc::NV,
                      CU_TENSOR_MAP_SWIZZLE_64B))
            return cudaErrorInvalidValue;
    }
    cudaError_t err = cudaFuncSetAttribute(tc::kda_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(tc::SMEM_BYTES));
    if (err != cudaSuccess) return err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
    cfg.blockDim = dim3(tc::NTHREADS, 1, 1);
    cfg.dynamicSmemBytes = tc::SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = tc::NS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    err = cudaLaunchKernelEx(&cfg, tc::kda_fwd_tc_kernel, p, maps);
    if (err != cudaSuccess) return err;
    return cudaGetLastError();
}

#ifdef KDA_TRACE
extern "C" int kda_trace_read(unsigned long long *host) {
    return static_cast<int>(cudaMemcpyFromSymbol(host, g_kda_trace, sizeof(g_kda_trace)));
}
#endif

cudaError_t read_and_clear_device_error(unsigned int *value) {
    cudaError_t err = cudaMemcpyFromSymbol(value, g_kda_device_error, sizeof(unsigned int));
    if (err != cudaSuccess) return err;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_kda_device_error, &zero, sizeof(unsigned int));
}

}  // namespace kda
