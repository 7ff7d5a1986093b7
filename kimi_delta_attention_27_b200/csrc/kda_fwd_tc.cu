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
//   W' = T' Kh;  W = W' diag(e^Ga);  U = T' V               (S4)
//   Qd = Qh diag(e^Ga) = Q e^G                              (decayed queries)
//   D  = U - W S                                            (S5, pseudo-values)
//   O  = scale (Qd S + Aqk D)                               (S6, inter + intra chunk)
//   S <- diag(e^Gl) S + Kt^T D                              (S7)
//
// When some channel decays too fast for one anchor per chunk (more than 2^-50 over 16 rows),
// the chunk's decayed blocks are formed instead with one anchor per 16 rows (the sub-block
// path); the rest of the chunk is the same.
//
// Work split: one 4-CTA cluster per (sequence, head).
//  * rank 0 ("chain") owns the whole fp32 state (128 x 128) and runs the sequential
//    part, S5-S7 (and U = T' V), with 128-column MMAs: the dependent-step latency of a
//    tcgen05 MMA barely depends on N up to 128, so the state is not split.
//  * ranks 1-3 ("prep") take chunks from a counter in the chain CTA's shared
//    memory and prepare them (S0-S4: gates, decayed blocks, UT solve, W, Qd, Kt),
//    writing each finished 80.5 KB operand set into a per-cluster ring of 6 slots
//    in global memory (it stays in L2); the chain CTA pulls each set with TMA bulk
//    loads. Shared memory of another CTA (DSMEM) carries only barrier signals and
//    counters: its bulk bandwidth is a fraction of an L2 TMA load's.
//  Every input byte is read from HBM once (q, k, v, g, beta by a prep CTA) and
//  every output byte written once (by the chain CTA).
//
// Precision: anchored factors (Kh, Qh, Kc), W, Qd and the state copy S' are bf16;
// T', Aqk, V, Kt and D are fp16 (10-bit mantissa) because the state update is most
// sensitive to them; every product accumulates in fp32 (TMEM) and the state itself is
// carried in fp32 registers.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include <cstdlib>
#include <cstring>
#include <mutex>

#include "kda_internal.h"
#include "sm100_ptx.cuh"

namespace kda {

__device__ unsigned int g_kda_device_error = 0;

#ifdef KDA_TEST_HOOKS
// Test-only build (never the product library): the publisher of chunk
// g_kda_test_skip_chunk leaves that chunk's ring slot unsignalled, so that the
// chain CTA's bounded wait for it runs out and the kernel winds down early.
__device__ int g_kda_test_skip_chunk = -1;
#endif

#ifdef KDA_TRACE
// Development-only timeline: when built with -DKDA_TRACE, the first cluster
// records %globaltimer at fixed points per chunk into g_kda_trace
// [rank][chunk < 64][point < 48]. The product build compiles none of this.
__device__ unsigned long long g_kda_trace[4 * 64 * 48];
// per cluster: chain CTA start, end, SM id, then the SM ids of ranks 1-3 and the ring address
__device__ unsigned long long g_kda_cluster_trace[1024 * 8];
#define KDA_TRACE_CLUSTER(slot, value)                                                              \
    do {                                                                                            \
        if (blockIdx.x / 4 < 1024) g_kda_cluster_trace[(blockIdx.x / 4) * 8 + (slot)] = (value);    \
    } while (0)
#ifndef KDA_TRACE_CLUSTER_ID
#define KDA_TRACE_CLUSTER_ID 0   // the cluster whose chunks are timed
#endif
#define KDA_TRACE_POINT(chunk, point)                                                               \
    do {                                                                                            \
        if (blockIdx.x / 4 == KDA_TRACE_CLUSTER_ID && (chunk) < 64)                                 \
            g_kda_trace[(rank * 64 + (chunk)) * 48 + (point)] = ptx::globaltimer();                 \
    } while (0)
#else
#define KDA_TRACE_CLUSTER(slot, value) \
    do {                               \
    } while (0)
#define KDA_TRACE_POINT(chunk, point) \
    do {                              \
    } while (0)
#endif

namespace tc {

using namespace ptx;

constexpr int D = kHeadDim;
constexpr int C = kChunk;
constexpr int NS = 4;          // CTAs per cluster: 1 chain + 3 prep
constexpr int NPREP = NS - 1;
constexpr int NTHREADS = 384;
#ifndef KDA_NRING
#define KDA_NRING 6
#endif
constexpr int NRING = KDA_NRING;  // ring slots per cluster (a multiple of NPREP)
static_assert(NRING % NPREP == 0 && NRING >= 6 && NRING <= 15, "ring depth");

// ---- operand set of one chunk (same byte layout in the global ring and in smem), 128B-swizzled tiles:
//   Kt^T fp16 [128 key][64 token]              B operand of C3^T (K-major)
//   -W^T, Qd^T bf16 [128 key][64 token] each   together the B operand of the state product (MN-major)
//   V fp16 [64 token][128 value], two boxes    A operand of the value-side product (MN-major)
//   T' fp16 [64][64 token]                     B operand of the value-side product (K-major)
//   Aqk fp16 [64 token][64 token]              B operand of the intra-chunk output product (K-major)
//   e^Gl fp32 [128]
constexpr uint32_t SET_KT = 0, SET_W = 16384, SET_Q = 32768, SET_V = 49152, SET_T = 65536, SET_AQK = 73728,
                   SET_DEC = 81920;
constexpr uint32_t SET_TX = 4 * 16384 + 2 * 8192 + 512;   // bytes per set
constexpr uint32_t SET_STRIDE = 83968;             // 82 KB, 1024-aligned
static_assert(SET_DEC + 512 <= SET_STRIDE, "operand set");
constexpr uint64_t RING_BYTES = static_cast<uint64_t>(NRING) * SET_STRIDE;
constexpr int kMaxRings = 256;                     // indexed by the chain CTA's SM id

// ---- chain CTA shared memory: two operand-set slots and two output staging tiles
constexpr uint32_t CH_SLOT = 0;                    // 2 x SET_STRIDE
constexpr uint32_t CH_OST = 2 * SET_STRIDE;        // 2 x [64 token][128 value] bf16 (two 64-channel boxes)
constexpr uint32_t CH_MISC = CH_OST + 2 * 16384;
// ---- prep CTA shared memory
constexpr uint32_t PR_STG = 0;                     // q 16 KB, k 16 KB, g 32 KB, v 16 KB
constexpr uint32_t STG_Q = 0, STG_K = 16384, STG_G = 32768, STG_V = 65536, STAGE_TX = 65536, VSTAGE_TX = 16384;
constexpr uint32_t PR_KH = 81920, PR_QH = PR_KH + 16384, PR_KC = PR_QH + 16384;
constexpr uint32_t AKK_LD = 68;                    // fp32 row stride of A and T
constexpr uint32_t PR_AKK = PR_KC + 16384;         // 17408 B
constexpr uint32_t PR_T = PR_AKK + 17408;          // 17408 B
constexpr uint32_t PR_P = PR_T + 17408;            // 4096 B
constexpr uint32_t PR_AVT = 169984;                // [T'; Aqk] fp16, 128 rows K-major SW128
constexpr uint32_t PR_TB = PR_AVT + 16384;         // T' bf16
constexpr uint32_t PR_MISC = PR_TB + 8192;
static_assert(PR_P + 4096 <= PR_AVT, "prep map");
static_assert(PR_AVT % 1024 == 0 && PR_AKK % 1024 == 0 && PR_KH % 1024 == 0 &&
                  SET_STRIDE % 1024 == 0 && SET_V % 1024 == 0, "alignment");

// misc area (offsets from the misc base of either role)
constexpr uint32_t M_BAR = 0;                      // up to 32 barriers
constexpr uint32_t M_BETA = 256, M_EGA = 512;                  // 64, 128 floats
// prep: beta of the two staged chunks (2 x 64 floats), the chunk index of the last four local
// chunks, the number of chunks the chain CTA has pulled (written by the chain CTA);
// chain: the next chunk to hand out (incremented by the prep CTAs)
constexpr uint32_t M_BETAQ = 1024, M_CHUNKQ = 1536, M_CONSUMED = 1552, M_NEXT = 1568;   // the last two: chain
constexpr uint32_t M_DEC = 2048;                               // 2 x 128 floats (e^Gl, part of the set)
constexpr uint32_t M_TMEM = 3072, M_ABORT = 3088, M_SMID = 3104;
constexpr uint32_t M_HTINFO = 3136;   // chain: where the final state goes (pointer, offset, flags)
constexpr uint32_t M_GSCALQ = 3584;                            // prep: 2 x 64 floats, a per-token gate
constexpr uint32_t M_INVN = 4096;     // prep: 1 / ||q||, 1 / ||k|| of the chunk's 64 rows (128 floats)
constexpr uint32_t MISC_BYTES = 4608;
constexpr uint32_t SMEM_USED = (CH_MISC > PR_MISC ? CH_MISC : PR_MISC) + MISC_BYTES;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;

// chain barriers
enum {
    CB_FULL = 0,     // 2: operand set landed in smem slot (1 arrival + tx)
    CB_SFREE = 2,    // 2: smem slot consumed (8 epilogue warps, the release warp, the output-product warp)
    CB_C1_FULL = 4,  // value-side + state products done
    CB_O_FULL = 5,   // intra-chunk output product done
    CB_OST_FREE = 6, // 2: output staging tile read out by the store warp
    CB_C3_FULL = 8,
    CB_O_READY = 9,  // output tile staged (4 warps)
    CB_READY = 10,   // NRING: ring slot written by a prep CTA (remote arrival)
    CB_COUNT = CB_READY + NRING
};
// prep barriers
enum {
    PB_STAGE_FULL = 0, PB_STAGE_FREE, PB_VSTAGE_FULL, PB_VSTAGE_FREE,
    PB_STAGE_RAW,       // tx: the tiles of a partial chunk, before the loader zeroes its tail rows
    PB_P1_DONE, PB_SPARE6,
    PB_WAV_DONE, PB_SPARE8, PB_SPARE9,
    PB_OUTA_READY,      // Kt^T final (over Kc^T)
    PB_OUTB_READY,      // -W^T (over the fp32 T workspace) and Qd^T (over A) final
    PB_OUTC_READY,      // T' and Aqk, e^Gl final (after the solve)
    PB_OUTA_FREE,       // publisher has read part A out
    PB_OUTC_FREE,       // publisher has read parts C and B out
    PB_COUNT
};
static_assert(CB_COUNT * 8 <= M_BETA && PB_COUNT * 8 <= M_BETA, "barrier area");

// ---- TMEM columns
// chain: C1^T (two buffers), C3^T, S'^T (bf16 pairs), D^T (fp16 pairs)
constexpr uint32_t COL_C1 = 0, COL_C3 = 256, COL_SP = 384, COL_DT = 448;
constexpr uint32_t COL_P1 = 0, COL_W = 64;                                           // prep
constexpr uint32_t COL_RB = 256;   // prep, sub-block path: one 64-column product per 16-row block
constexpr uint32_t TMEM_COLS = 512;

// ---- gate range. A chunk takes the single-anchor path when, on every channel, each 16-row
// quarter of the chunk decays by less than 2^-50 (so each half by less than 2^-100, which keeps
// every anchored factor within 2^+-100); otherwise the sub-block path, on which per-token
// log-decays are floored at -10 (alpha >= e^-10 = 4.5e-5): a channel that keeps less than that of
// its state per token has forgotten it to far below the precision of the bf16 operands either way.
constexpr float kFloorLog2 = -14.426950408889634f;   // log2(e^-10)
constexpr float kQuarterRangeLog2 = 50.f;

// ---- instruction descriptors (M = 128)
constexpr uint32_t ID_P1 = idesc_f16(128, 64, 1, 1, 1);      // bf16, A MN-major, B MN-major
constexpr uint32_t ID_W = idesc_f16(128, 64, 1, 0, 0);       // bf16, K-major / K-major
constexpr uint32_t ID_UVT = idesc_f16(128, 64, 0, 1, 0);       // fp16, A (V) MN-major, B (T') K-major
constexpr uint32_t ID_STATE_T = idesc_f16(128, 128, 1, 0, 1);  // bf16, A (S'^T) in TMEM, B MN-major
constexpr uint32_t ID_STATE_H = idesc_f16(128, 64, 1, 0, 1);   // the same, one 64-column half
constexpr uint32_t ID_C3T = idesc_f16(128, 128, 0, 0, 0);      // fp16, A (D^T) in TMEM, B K-major
constexpr uint32_t ID_OQK = idesc_f16(128, 64, 0, 0, 0);       // fp16, A (D^T) in TMEM, B (Aqk) K-major

#ifdef KDA_TEST_HOOKS
constexpr uint64_t kWaitLimitNs = 100000000ull;   // 100 ms in the test-only build
#else
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s: far above any legitimate wait
#endif

struct TmaMaps {
    CUtensorMap q, k, g, v, o;
};

__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile uint32_t *abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    for (;;) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer() - t0 > kWaitLimitNs) {
            *abort_flag = 1;
            atomicOr(&g_kda_device_error, kErrTimeout);
            return false;
        }
    }
}

__device__ __forceinline__ float bf2f(uint16_t x) { return __uint_as_float(static_cast<uint32_t>(x) << 16); }
__device__ __forceinline__ float lo_bf(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float hi_bf(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
// fp32 -> tf32 (round to nearest, ties away from zero), the operand format of the tf32 MMA
__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}
// d (16 x 8, fp32) += a (16 x 8, tf32, row-major) * b (8 x 8, tf32), one warp. Fragments, with
// g = lane / 4 and i = lane % 4: a = {(g, i), (g + 8, i), (g, i + 4), (g + 8, i + 4)},
// b = {(i, g), (i + 4, g)}, d = {(g, 2i), (g, 2i + 1), (g + 8, 2i), (g + 8, 2i + 1)}.
__device__ __forceinline__ void mma_tf32_16x8x8(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
}
__device__ __forceinline__ uint32_t pack_f16(float a, float b) {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
}

constexpr float kLog2e = 1.4426950408889634f;   // log2(e)

// 2^y by the hardware approximation (relative error about 2^-22; subnormal results flush to 0)
__device__ __forceinline__ float ex2_approx(float y) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(y));
    return r;
}

__device__ __forceinline__ float lg2_approx(float x) {
    float r;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

constexpr float kLn2 = 0.6931471805599453f;

// log2(sigmoid(x)) = min(x, 0) log2(e) - log2(1 + 2^(-|x| log2(e))), i.e. logsigmoid(x) in
// log2 units, from the hardware 2^y and log2 approximations (absolute error about 1e-7)
__device__ __forceinline__ float log2_sigmoid(float x) {
    return fminf(x, 0.f) * kLog2e - lg2_approx(1.f + ex2_approx(-fabsf(x) * kLog2e));
}

// byte offset of 16-byte chunk j of row r in a tile of 128-byte rows, 128B swizzle
__device__ __forceinline__ uint32_t sw128(uint32_t r, uint32_t j) { return r * 128u + ((j ^ (r & 7u)) << 4); }

// packed fp32 pairs (sm_100 f32x2 instructions): one instruction for both lanes of a float2
__device__ __forceinline__ float2 f2_mul(float2 a, float2 b) {
    float2 r;
    asm("{\n\t.reg .b64 ra, rb, rc;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rc, ra, rb;\n\tmov.b64 {%0, %1}, rc;\n\t}"
        : "=f"(r.x), "=f"(r.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return r;
}
__device__ __forceinline__ float2 f2_add(float2 a, float2 b) {
    float2 r;
    asm("{\n\t.reg .b64 ra, rb, rc;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rc, ra, rb;\n\tmov.b64 {%0, %1}, rc;\n\t}"
        : "=f"(r.x), "=f"(r.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return r;
}

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
__device__ __forceinline__ void st_shared_u32(uint32_t addr, uint32_t x) {
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(addr), "r"(x) : "memory");
}
__device__ __forceinline__ void st_shared_v2(uint32_t addr, uint32_t a, uint32_t b) {
    asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(addr), "r"(a), "r"(b) : "memory");
}
__device__ __forceinline__ void st_shared_u16(uint32_t addr, uint16_t x) {
    asm volatile("st.shared.u16 [%0], %1;" ::"r"(addr), "h"(x) : "memory");
}
__device__ __forceinline__ uint16_t bf16_bits(float x) {
    __nv_bfloat16 h = __float2bfloat16_rn(x);
    return *reinterpret_cast<uint16_t *>(&h);
}
__device__ __forceinline__ void st_global_v4(void *p, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.global.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(a), "r"(b), "r"(c), "r"(d)
                 : "memory");
}
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}
// bulk copy global -> this CTA's shared memory, completing tx bytes on a local barrier
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}
// bulk copy this CTA's shared memory -> global, tracked by the executing thread's bulk groups
__device__ __forceinline__ void bulk_s2g(void *dst, uint32_t src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void tma_store_3d(const CUtensorMap *map, uint32_t src, int32_t c0, int32_t c1, int32_t c2) {
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(src), "r"(c0), "r"(c1), "r"(c2)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ uint32_t ld_shared_cluster_u32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}
// named barrier that also ORs a predicate over the participating threads: every thread gets the
// same answer, so a loop left on it is left by all of them (no thread is stranded at a barrier)
__device__ __forceinline__ bool named_bar_any(uint32_t id, uint32_t nthreads, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 q, %1, 0;\n\t"
        "bar.red.or.pred p, %2, %3, q;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0;
}

// atomic add on a u32 in shared memory of a cluster CTA (shared::cluster address); returns the old value
__device__ __forceinline__ uint32_t atom_add_cluster(uint32_t addr, uint32_t v) {
    uint32_t old;
    asm volatile("atom.shared::cluster.add.u32 %0, [%1], %2;" : "=r"(old) : "r"(addr), "r"(v) : "memory");
    return old;
}
__device__ __forceinline__ void st_release_cluster(uint32_t addr, uint32_t v) {
    asm volatile("st.release.cluster.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t ld_acquire_remote(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.acquire.cluster.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}
// bounded wait until the u32 at `addr` (another CTA's shared memory) reaches `target`
__device__ __forceinline__ bool wait_count_remote(uint32_t addr, uint32_t target, volatile uint32_t *abort_flag) {
    if (ld_acquire_remote(addr) >= target) return true;
    const uint64_t t0 = globaltimer();
    for (;;) {
        if (ld_acquire_remote(addr) >= target) return true;
        if (*abort_flag) return false;
        if (globaltimer() - t0 > kWaitLimitNs) {
            *abort_flag = 1;
            atomicOr(&g_kda_device_error, kErrTimeout);
            return false;
        }
    }
}
__device__ __forceinline__ uint32_t smid() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(r));
    return r;
}

// kRingPerCluster == false: `rings` holds kMaxRings rings and a cluster uses the one of
// its chain CTA's SM (a chain CTA fills an SM's shared memory, so no two resident
// clusters, of this launch or of any other, share a ring).
// kRingPerCluster == true: `rings` holds one ring per cluster of this launch and
// cluster c uses ring c (the allocation-free entry point, whose fixed scratch bounds
// the cluster count).
// kGate: how g is given (kGateF32 / kGateBF16: log alpha per channel, fp32 or bf16 [rows, H, 128];
// kGateScalar: one fp32 log alpha per token and head [rows, H], the same for every channel)
// kNorm: q and k are L2-normalised per token and head first (the norms are applied in fp32 where
// the operands are formed, so the normalised values are rounded only once)
// kSeg: the launch may be segmented or affine (FwdParams::seg_len, mode); other launches compile
// none of that bookkeeping
template <bool kRingPerCluster, int kGate, bool kNorm, bool kSeg>
__global__ void __launch_bounds__(NTHREADS, 1)
    kda_fwd_tc_kernel(const FwdParams p, const __grid_constant__ TmaMaps maps, unsigned char *rings) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = raw + ((1024u - (raw & 1023u)) & 1023u);
    unsigned char *sgen = smem_raw + (sbase - raw);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = cluster_ctarank();
    const bool is_chain = rank == 0;
    const uint32_t misc = sbase + (is_chain ? CH_MISC : PR_MISC);
    unsigned char *miscg = sgen + (is_chain ? CH_MISC : PR_MISC);
    auto BAR = [&](int i) -> uint32_t { return misc + M_BAR + 8u * static_cast<uint32_t>(i); };
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(miscg + M_ABORT);

    const int H = p.num_heads;
    int64_t unit = blockIdx.x / NS;
    // affine mode: units [0, N H) run each piece from a zero state, units [N H, 2 N H) from the
    // identity with v = 0 (the piece's transition matrix); neither writes an output
    const bool affine = kSeg && p.mode == kModeAffine;
    bool transition = false;
    if (affine && unit >= static_cast<int64_t>(p.num_seqs) * p.num_heads) {
        transition = true;
        unit -= static_cast<int64_t>(p.num_seqs) * p.num_heads;
    }
    const int h = static_cast<int>(unit % H);
    const int64_t s = unit / H;
    int64_t bos, eos;
    bool cu_bad = false;
    // segmented rows: unit s is segment j of row b, tokens [b T + j L, min(b T + (j + 1) L, (b + 1) T))
    const bool segmented = kSeg && p.seg_len > 0;
    const int64_t seg_row = segmented ? s / p.seg_count : s;
    const int64_t seg_idx = segmented ? s % p.seg_count : 0;
    if (segmented) {
        bos = seg_row * p.seq_len + seg_idx * p.seg_len;
        const int64_t row_end = (seg_row + 1) * p.seq_len;
        eos = bos + p.seg_len < row_end ? bos + p.seg_len : row_end;
    } else if (p.cu_seqlens) {
        int64_t a = p.cu_seqlens[s], b = p.cu_seqlens[s + 1];
        cu_bad = a < 0 || b < a || b > p.seq_len || (s == 0 && a != 0) || (s + 1 == p.num_seqs && b != p.seq_len);
        a = a < 0 ? 0 : (a > p.seq_len ? p.seq_len : a);
        b = b < 0 ? 0 : (b > p.seq_len ? p.seq_len : b);
        bos = a;
        eos = b < a ? a : b;
    } else {
        bos = s * p.seq_len;
        eos = bos + p.seq_len;
    }
    const int nch = static_cast<int>((eos - bos + C - 1) / C);
    const size_t state_base = (static_cast<size_t>(s) * H + h) * D * D;

    // ---------------------------------------------------------------- setup
    if (tid == 0) {
        if (is_chain) {
            for (int i = 0; i < 2; ++i) {
                mbar_init(BAR(CB_FULL + i), 1);
                mbar_init(BAR(CB_SFREE + i), 10);
                mbar_init(BAR(CB_OST_FREE + i), 1);
            }
            mbar_init(BAR(CB_C1_FULL), 1);
            mbar_init(BAR(CB_O_FULL), 1);
            mbar_init(BAR(CB_C3_FULL), 1);
            mbar_init(BAR(CB_O_READY), 4);
            for (int i = 0; i < NRING; ++i) mbar_init(BAR(CB_READY + i), 1);
            const uint32_t sm = smid();
            *reinterpret_cast<volatile uint32_t *>(miscg + M_SMID) = sm;
            *reinterpret_cast<volatile uint32_t *>(miscg + M_NEXT) = 0u;
            *reinterpret_cast<volatile uint32_t *>(miscg + M_CONSUMED) = 0u;   // sets pulled so far
            // the shared pool holds a ring per SM id; a launch with one ring per cluster does not
            // index it by SM
            const bool no_ring = !kRingPerCluster && sm >= static_cast<uint32_t>(kMaxRings);
            *abort_flag = no_ring ? 1u : 0u;
            if (no_ring) atomicOr(&g_kda_device_error, kErrRingIndex);
            // a malformed cu_seqlens entry is reported (the sequence bounds were clamped above)
            if (cu_bad) atomicOr(&g_kda_device_error, kErrCuSeqlens);
            // where the final state goes: per unit, except that a segmented plain run writes only
            // the last piece's, as its row's final state
            void *const hT_ptr = transition ? p.hT_aux : p.hT;
            const bool hT_write = hT_ptr != nullptr && (affine || !segmented || seg_idx == p.seg_count - 1);
            *reinterpret_cast<void *volatile *>(miscg + M_HTINFO) = hT_ptr;
            *reinterpret_cast<volatile size_t *>(miscg + M_HTINFO + 8) =
                (!affine && segmented) ? (static_cast<size_t>(seg_row) * H + h) * D * D : state_base;
            *reinterpret_cast<volatile uint32_t *>(miscg + M_HTINFO + 16) =
                (hT_write ? 1u : 0u) | ((transition || p.hT_fp32 != 0) ? 2u : 0u);
        } else {
            for (int i = 0; i < PB_COUNT; ++i) mbar_init(BAR(i), i == PB_STAGE_FULL ? 2 : 1);
            *abort_flag = 0;
        }
        fence_mbar_init();
    }
    if (warp == 2) {
        tmem_alloc(misc + M_TMEM, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    cluster_arrive();
    cluster_wait();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(miscg + M_TMEM);
    uint32_t ring_id;
    if constexpr (kRingPerCluster) {
        ring_id = blockIdx.x / NS;
    } else {
        // this cluster's ring: indexed by the chain CTA's SM (unique among resident clusters)
        ring_id = is_chain ? *reinterpret_cast<volatile uint32_t *>(miscg + M_SMID)
                           : ld_shared_cluster_u32(mapa(sbase + CH_MISC + M_SMID, 0));
        if (!is_chain && ring_id >= static_cast<uint32_t>(kMaxRings) && tid == 0) *abort_flag = 1;
    }
    unsigned char *ring = rings + static_cast<uint64_t>(ring_id < kMaxRings ? ring_id : 0) * RING_BYTES;

    if (tid == 0) {
        if (is_chain) {
            KDA_TRACE_CLUSTER(0, globaltimer());
            KDA_TRACE_CLUSTER(7, static_cast<unsigned long long>(clock64()));
        }
        KDA_TRACE_CLUSTER(2 + rank, smid());
    }
    if (is_chain) {
        // ======================================================================= chain CTA
        if (warp == 0) {
            // ---- output tiles: two staging tiles (each two 64-channel boxes, 128B swizzle);
            // TMA-stored for full chunks, copied row by row otherwise
            for (int n = 0; n < nch; ++n) {
                const int sl = n & 1;
                const int64_t t0 = bos + static_cast<int64_t>(n) * C;
                const int L = static_cast<int>(eos - t0 < C ? eos - t0 : C);
                const uint32_t stage = sbase + CH_OST + sl * 16384;
                if (!wait_bar(BAR(CB_O_READY), n & 1, abort_flag)) break;
                if (affine) {
                    // no output in affine mode
                } else if (L == C) {
                    if (lane == 0) {
                        tma_store_3d(&maps.o, stage, 0, h, static_cast<int32_t>(t0));
                        tma_store_3d(&maps.o, stage + 8192, 64, h, static_cast<int32_t>(t0));
                        bulk_commit();
                        bulk_wait_read0();
                    }
                } else {
                    // partial chunk: rows < L only, 16 bytes per lane, a row is 2 x 8 chunks
                    for (int e = lane; e < L * 16; e += 32) {
                        const int rr = e >> 4, hb = (e >> 3) & 1, j = e & 7;
                        const uint4 v = ld_shared_v4(stage + hb * 8192 + sw128(rr, j));
                        st_global_v4(p.out + ((t0 + rr) * H + h) * D + hb * 64 + j * 8, v.x, v.y, v.z, v.w);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(BAR(CB_OST_FREE + sl));
            }
            if (lane == 0) bulk_wait0();
            __syncwarp();
        } else if (warp == 2) {
            // ---- operand sets: ring slot (global, L2) -> smem slot
            for (int n = 0; n < nch; ++n) {
                const int sl = n & 1, r = n % NRING;
                if (!wait_bar(BAR(CB_READY + r), (n / NRING) & 1, abort_flag)) break;
                if (lane == 0) KDA_TRACE_POINT(n, 37);
                if (n >= 2 && !wait_bar(BAR(CB_SFREE + sl), ((n - 2) >> 1) & 1, abort_flag)) break;
                if (lane == 0) KDA_TRACE_POINT(n, 38);
                if (lane == 0) {
                    const unsigned char *src = ring + static_cast<uint64_t>(r) * SET_STRIDE;
                    const uint32_t dst = sbase + CH_SLOT + sl * SET_STRIDE;
                    mbar_arrive_expect_tx(BAR(CB_FULL + sl), SET_TX);
                    for (uint32_t part = 0; part < 4; ++part)
                        bulk_g2s(dst + part * 16384, src + part * 16384, 16384, BAR(CB_FULL + sl));
                    bulk_g2s(dst + SET_T, src + SET_T, 16384, BAR(CB_FULL + sl));   // T' and Aqk
                    bulk_g2s(dst + SET_DEC, src + SET_DEC, 512, BAR(CB_FULL + sl));
                }
                __syncwarp();
            }
        } else if (warp == 3) {
            // ---- ring slot release: once chunk n's set has landed in shared memory, its ring
            // slot goes back to the producer of chunk n + NRING. A cluster-scope remote arrival
            // can hold the issuing thread for a while, so it is kept off the MMA warp.
            for (int n = 0; n < nch; ++n) {
                const int sl = n & 1;
                if (!wait_bar(BAR(CB_FULL + sl), (n >> 1) & 1, abort_flag)) break;
                if (lane == 0) KDA_TRACE_POINT(n, 39);
                if (lane == 0) {
                    mbar_arrive(BAR(CB_SFREE + sl));
                    // chunks 0..n have been pulled: any prep CTA may reuse the slot of chunk n. One
                    // store into this CTA's own shared memory, which the prep CTAs poll: a release
                    // store into each of them measured about 0.6 us apiece and held the ring full.
                    if (n + NRING < nch) st_release_cluster(sbase + CH_MISC + M_CONSUMED, static_cast<uint32_t>(n + 1));
                }
                __syncwarp();
            }
        } else if (warp == 1) {
            // ---- intra-chunk output product, C1^T[:, 64..127] += D^T Aqk^T, issued once C3^T
            // (the other reader of D^T, on the critical path) has completed
            for (int n = 0; n < nch; ++n) {
                if (!__all_sync(0xffffffffu, wait_bar(BAR(CB_C3_FULL), n & 1, abort_flag))) break;
                tc_fence_after();
                if (elect_one()) {
                    const uint32_t slot = sbase + CH_SLOT + (n & 1) * SET_STRIDE;
                    for (int ks = 0; ks < 4; ++ks)
                        mma_f16_ts(tmem + COL_C1 + (n & 1) * 128 + 64, tmem + COL_DT + ks * 8,
                                   smem_desc(slot + SET_AQK + ks * 32, 16, 1024, kSwizzle128), ID_OQK, 1);
                    mma_commit(BAR(CB_O_FULL));
                }
                __syncwarp();
                // that product was the last reader of the slot's Aqk
                if (!wait_bar(BAR(CB_O_FULL), n & 1, abort_flag)) break;
                if (lane == 0) mbar_arrive(BAR(CB_SFREE + (n & 1)));
                __syncwarp();
            }
        } else if (warp >= 4) {
            // ---- epilogues: 8 warps. The state is kept transposed: a thread owns S^T[v][j] for
            // one value channel v = TMEM lane 32*(warp%4) + lane and 64 key channels
            // j in [64*half, 64*half + 64). Per chunk (all products accumulate in fp32 TMEM):
            //   C1^T = [U^T | 0] + S'^T [-W; Qd]^T       columns 0..63: D^T = (U - W S')^T,
            //                                            columns 64..127: (Qd S')^T
            //   C3^T = D^T Kt                            S^T <- e^Gl (.) S^T + C3^T
            //   C1^T[:, 64..127] += D^T Aqk^T            O = scale (Qd S' + Aqk D)
            // The bf16 state copy S'^T and the fp16 pseudo-values D^T are written straight into
            // TMEM, where they are the A operands of the next products. Warps of half 0 turn
            // columns 0..63 into D^T; warps of half 1 write the output of chunk n after the chunk's
            // closing barrier, while the state product of chunk n + 1 runs.
            const int q4 = warp & 3, half = (warp - 4) >> 2;
            const int v = q4 * 32 + lane;              // value channel = TMEM lane
            const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
            const int j0 = half * 64;                  // first key channel of this thread
            float S[64];
            if (transition) {
#pragma unroll
                for (int i = 0; i < 64; ++i) S[i] = (j0 + i == v) ? 1.f : 0.f;
            } else if (p.h0 && !affine) {
                if (p.h0_fp32) {
                    const float *src = static_cast<const float *>(p.h0) + state_base + v;
#pragma unroll
                    for (int i = 0; i < 64; ++i) S[i] = src[static_cast<size_t>(j0 + i) * D];
                } else {
                    const uint16_t *src = static_cast<const uint16_t *>(p.h0) + state_base + v;
#pragma unroll
                    for (int i = 0; i < 64; ++i) S[i] = bf2f(src[static_cast<size_t>(j0 + i) * D]);
                }
            } else {
#pragma unroll
                for (int i = 0; i < 64; ++i) S[i] = 0.f;
            }
            // S'^T (bf16, two key channels per TMEM column) -> columns COL_SP + 32*half
            auto write_sprime = [&]() {
                uint32_t w[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) w[i] = pack_bf16(S[2 * i], S[2 * i + 1]);
                tmem_st32(tmem + lane_base + COL_SP + 32 * half, w);
                tmem_wait_st();
            };
            // The products are issued by warp 4 (a D^T warp) as soon as their operands are in place
            // (a named barrier among the writers), with no hop through another warp: the warp enters
            // converged and one elected lane issues, so that the operands stay warp-uniform.
            // value-side product of chunk n into its C1^T buffer (no state involved); C1^T has two
            // buffers, so chunk n's buffer was last read in chunk n - 2
            auto issue_uv = [&](int n) -> bool {
                const int s1 = n & 1;
                const uint32_t slot = sbase + CH_SLOT + s1 * SET_STRIDE;
                // the lanes agree on the outcome before the election
                if (!__all_sync(0xffffffffu, wait_bar(BAR(CB_FULL + s1), (n >> 1) & 1, abort_flag))) return false;
                tc_fence_after();
                if (elect_one()) {
                    for (int ks = 0; ks < 4; ++ks)
                        mma_f16(tmem + COL_C1 + s1 * 128, smem_desc(slot + SET_V + ks * 2048, 8192, 1024, kSwizzle128),
                                smem_desc(slot + SET_T + ks * 32, 16, 1024, kSwizzle128), ID_UVT, ks > 0);
                }
                __syncwarp();
                return true;
            };
            auto issue_state = [&](int n) {
                const int s1 = n & 1;
                const uint32_t slot = sbase + CH_SLOT + s1 * SET_STRIDE;
                tc_fence_after();
                if (elect_one()) {
                    KDA_TRACE_POINT(n, 13);
                    // first K step in two halves: columns 0..63 accumulate onto U^T, columns 64..127
                    // (the output half, not touched by the value-side product) start from zero
                    mma_f16_ts(tmem + COL_C1 + s1 * 128, tmem + COL_SP,
                               smem_desc(slot + SET_W, 16384, 1024, kSwizzle128), ID_STATE_H, 1);
                    mma_f16_ts(tmem + COL_C1 + s1 * 128 + 64, tmem + COL_SP,
                               smem_desc(slot + SET_Q, 16384, 1024, kSwizzle128), ID_STATE_H, 0);
                    for (int ks = 1; ks < 8; ++ks)
                        mma_f16_ts(tmem + COL_C1 + s1 * 128, tmem + COL_SP + ks * 8,
                                   smem_desc(slot + SET_W + ks * 2048, 16384, 1024, kSwizzle128), ID_STATE_T, 1);
                    mma_commit(BAR(CB_C1_FULL));
                    KDA_TRACE_POINT(n, 3);
                }
                __syncwarp();
            };
            auto issue_c3 = [&](int n) {
                const uint32_t slot = sbase + CH_SLOT + (n & 1) * SET_STRIDE;
                tc_fence_after();
                if (elect_one()) {
                    KDA_TRACE_POINT(n, 4);
                    for (int ks = 0; ks < 4; ++ks)
                        mma_f16_ts(tmem + COL_C3, tmem + COL_DT + ks * 8,
                                   smem_desc(slot + SET_KT + ks * 32, 16, 1024, kSwizzle128), ID_C3T, ks > 0);
                    mma_commit(BAR(CB_C3_FULL));
                    KDA_TRACE_POINT(n, 5);
                }
                __syncwarp();
            };
            write_sprime();
            tc_fence_before();
            named_bar_sync(4, 256);
            if (warp == 4 && nch > 0) {
                if (issue_uv(0)) issue_state(0);
            }
            __syncwarp();
            for (int n = 0; n < nch; ++n) {
                const int sl = n & 1;
                // A wait that gives up (abort) does not leave the loop on its own: the warps leave
                // together at the chunk's closing barrier.
                wait_bar(BAR(CB_C1_FULL), n & 1, abort_flag);
                tc_fence_after();
                if (tid == 128) KDA_TRACE_POINT(n, 9);
                bool ok = true;
                if (half == 0) {
                    // pseudo-values D^T[v][t] -> fp16, two tokens per TMEM column (A operand of
                    // C3^T and of the intra-chunk output product); the previous chunk's output
                    // product must have read the old D^T
                    if (n >= 1) wait_bar(BAR(CB_O_FULL), (n - 1) & 1, abort_flag);
                    const uint32_t acc = tmem + lane_base + COL_C1 + sl * 128;
                    uint32_t r0[32], r1[32];
                    tmem_ld32(acc, r0);
                    tmem_ld32(acc + 32, r1);
                    tmem_wait_ld();
                    if (tid == 128) KDA_TRACE_POINT(n, 0);
                    uint32_t w[32];
#pragma unroll
                    for (int i = 0; i < 16; ++i) w[i] = pack_f16(__uint_as_float(r0[2 * i]), __uint_as_float(r0[2 * i + 1]));
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        w[16 + i] = pack_f16(__uint_as_float(r1[2 * i]), __uint_as_float(r1[2 * i + 1]));
                    tmem_st32(tmem + lane_base + COL_DT, w);
                    tmem_wait_st();
                    if (tid == 128) KDA_TRACE_POINT(n, 1);
                    tc_fence_before();
                    named_bar_sync(3, 128);
                    if (warp == 4) {
                        issue_c3(n);
                        // the next chunk's value-side product follows on the tensor pipe; this
                        // warp waits for its slot here, so that the product runs during the C3^T
                        // epilogue rather than ahead of the next state product
                        if (n + 1 < nch) ok = issue_uv(n + 1);
                    }
                    __syncwarp();
                }
                if (tid == 128) KDA_TRACE_POINT(n, 6);
                (void)ok;
                wait_bar(BAR(CB_C3_FULL), n & 1, abort_flag);
                tc_fence_after();
                if (tid == 128) KDA_TRACE_POINT(n, 10);
                {
                    uint32_t r0[32], r1[32];
                    tmem_ld32(tmem + lane_base + COL_C3 + j0, r0);
                    tmem_ld32(tmem + lane_base + COL_C3 + j0 + 32, r1);
                    const float *decp = reinterpret_cast<const float *>(sgen + CH_SLOT + sl * SET_STRIDE + SET_DEC) + j0;
                    tmem_wait_ld();
#pragma unroll
                    for (int i4 = 0; i4 < 8; ++i4) {
                        const float4 d4 = reinterpret_cast<const float4 *>(decp)[i4];
                        const float dv[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) S[4 * i4 + e] = fmaf(dv[e], S[4 * i4 + e], __uint_as_float(r0[4 * i4 + e]));
                    }
#pragma unroll
                    for (int i4 = 0; i4 < 8; ++i4) {
                        const float4 d4 = reinterpret_cast<const float4 *>(decp)[8 + i4];
                        const float dv[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            S[32 + 4 * i4 + e] = fmaf(dv[e], S[32 + 4 * i4 + e], __uint_as_float(r1[4 * i4 + e]));
                    }
                }
                if (tid == 128) KDA_TRACE_POINT(n, 8);
                if (n + 1 < nch) write_sprime();
                if (tid == 128) KDA_TRACE_POINT(n, 7);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(BAR(CB_SFREE + sl));   // decay reads done
                if (n + 1 < nch) {
                    if (named_bar_any(4, 256, *abort_flag != 0)) break;
                    if (warp == 4) issue_state(n + 1);
                    __syncwarp();
                }
                if (tid == 128) KDA_TRACE_POINT(n, 11);
                if (half == 1) {
                    // output tile O[t][v] = scale * C1^T[v][64 + t] (bf16) -> staging tile `sl`
                    // (two 64-channel boxes, 128B swizzle) for the store warp
                    wait_bar(BAR(CB_O_FULL), n & 1, abort_flag);
                    if (n >= 2) wait_bar(BAR(CB_OST_FREE + sl), ((n - 2) >> 1) & 1, abort_flag);
                    tc_fence_after();
                    const uint32_t acc = tmem + lane_base + COL_C1 + sl * 128 + 64;
                    const uint32_t stage = sbase + CH_OST + sl * 16384 + (v >> 6) * 8192;
                    const uint32_t vc = static_cast<uint32_t>(v & 63);
                    const float sc = p.scale;
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        uint32_t r[32];
                        tmem_ld32(acc + 32 * hh, r);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            const uint32_t t = static_cast<uint32_t>(32 * hh + i);
                            const uint32_t a = stage + t * 128u + ((((vc >> 3) ^ (t & 7u))) << 4) + (vc & 7u) * 2u;
                            st_shared_u16(a, bf16_bits(sc * __uint_as_float(r[i])));
                        }
                    }
                    fence_proxy_async_smem();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(BAR(CB_O_READY));
                }
            }
            // final state: hT[j][v], coalesced across the warp for each key channel j (its place was
            // noted in shared memory at setup, so that nothing of it stays live through the loop)
            void *const hT_ptr = *reinterpret_cast<void *const volatile *>(miscg + M_HTINFO);
            const size_t hT_base = *reinterpret_cast<const volatile size_t *>(miscg + M_HTINFO + 8);
            const uint32_t hT_flags = *reinterpret_cast<const volatile uint32_t *>(miscg + M_HTINFO + 16);
            const bool hT_fp32 = (hT_flags & 2u) != 0;
            if ((hT_flags & 1u) && !*abort_flag) {
                if (hT_fp32) {
                    float *dst = static_cast<float *>(hT_ptr) + hT_base + v;
#pragma unroll
                    for (int i = 0; i < 64; ++i) dst[static_cast<size_t>(j0 + i) * D] = S[i];
                } else {
                    uint16_t *dst = static_cast<uint16_t *>(hT_ptr) + hT_base + v;
#pragma unroll
                    for (int i = 0; i < 64; ++i) dst[static_cast<size_t>(j0 + i) * D] = bf16_bits(S[i]);
                }
            }
        }
    } else {
        // ======================================================================= prep CTA
        if (warp == 0) {
            // ---- chunk hand-out and staging loads. The prep CTAs take chunks from a counter in
            // the chain CTA's shared memory, so a slower CTA simply prepares fewer of them. For
            // each local chunk kk: the chunk index (queue of 4), its beta (queue of 2), q, k, g by
            // TMA, then v.
            volatile uint32_t *chunkq = reinterpret_cast<volatile uint32_t *>(miscg + M_CHUNKQ);
            uint32_t nraw = 0;   // partial chunks staged so far (phases of PB_STAGE_RAW)
            for (int kk = 0;; ++kk) {
                if (kk >= 1 && !wait_bar(BAR(PB_STAGE_FREE), (kk - 1) & 1, abort_flag)) break;
                uint32_t mm = 0;
                if (lane == 0) mm = atom_add_cluster(mapa(sbase + CH_MISC + M_NEXT, 0), 1u);
                mm = __shfl_sync(0xffffffffu, mm, 0);
                const int m = static_cast<int>(mm);
                if (lane == 0) chunkq[kk & 3] = mm;
                if (m >= nch) {
                    // no chunk left: release the other roles of this CTA
                    __syncwarp();
                    if (lane == 0) {
                        mbar_arrive(BAR(PB_STAGE_FULL));
                        mbar_arrive(BAR(PB_STAGE_FULL));
                    }
                    break;
                }
                const int64_t t0 = bos + static_cast<int64_t>(m) * C;
                const int32_t row = static_cast<int32_t>(t0);
                // a partial chunk lands on its own barrier first: this warp zeroes the staged rows
                // past the sequence's end (the next sequence's tokens, or TMA fill) before handing
                // the tiles over, so that S1 needs no row masks
                const int Lz = static_cast<int>(eos - t0 < C ? eos - t0 : C);
                const uint32_t land = Lz < C ? BAR(PB_STAGE_RAW) : BAR(PB_STAGE_FULL);
                if (lane == 0) {
                    mbar_arrive_expect_tx(land, kGate == kGateF32    ? STAGE_TX
                                                : kGate == kGateBF16 ? STAGE_TX - 16384u
                                                                     : STAGE_TX - 32768u);
                    tma_load_3d(sbase + PR_STG + STG_Q, &maps.q, land, 0, h, row);
                    tma_load_3d(sbase + PR_STG + STG_K, &maps.k, land, 0, h, row);
                    // a bf16 gate tile goes to the upper half of the fp32 one's place
                    if constexpr (kGate == kGateF32)
                        tma_load_3d(sbase + PR_STG + STG_G, &maps.g, land, 0, h, row);
                    else if constexpr (kGate == kGateBF16)
                        tma_load_3d(sbase + PR_STG + STG_G + 16384, &maps.g, land, 0, h, row);
                }
                float *betaq = reinterpret_cast<float *>(miscg + M_BETAQ) + (kk & 1) * C;
                for (int i = lane; i < C; i += 32) {
                    const int64_t tok = t0 + i;
                    betaq[i] = tok < eos ? p.beta[tok * H + h] : 0.f;
                }
                if constexpr (kGate == kGateScalar) {
                    // one log alpha per token (activated here when asked); 0 past the end
                    float *gq = reinterpret_cast<float *>(miscg + M_GSCALQ) + (kk & 1) * C;
                    const float *gs = static_cast<const float *>(p.g);
                    for (int i = lane; i < C; i += 32) {
                        const int64_t tok = t0 + i;
                        float x = tok < eos ? gs[tok * H + h] : 0.f;
                        if ((p.flags & kFlagGateLogsigmoid) && tok < eos) x = log2_sigmoid(x) * kLn2;
                        gq[i] = x;
                    }
                }
                if (Lz < C) {
                    if (!wait_bar(BAR(PB_STAGE_RAW), nraw & 1u, abort_flag)) break;
                    ++nraw;
                    for (int e = lane; e < (C - Lz) * 16; e += 32) {
                        const uint32_t off = static_cast<uint32_t>((Lz + (e >> 4)) * 256 + (e & 15) * 16);
                        st_shared_v4(sbase + PR_STG + STG_Q + off, 0u, 0u, 0u, 0u);
                        st_shared_v4(sbase + PR_STG + STG_K + off, 0u, 0u, 0u, 0u);
                    }
                    if constexpr (kGate == kGateF32) {
                        for (int e = lane; e < (C - Lz) * 32; e += 32)
                            st_shared_v4(sbase + PR_STG + STG_G + static_cast<uint32_t>((Lz + (e >> 5)) * 512 + (e & 31) * 16),
                                         0u, 0u, 0u, 0u);
                    } else if constexpr (kGate == kGateBF16) {
                        for (int e = lane; e < (C - Lz) * 16; e += 32)
                            st_shared_v4(sbase + PR_STG + STG_G + 16384 +
                                             static_cast<uint32_t>((Lz + (e >> 4)) * 256 + (e & 15) * 16),
                                         0u, 0u, 0u, 0u);
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(BAR(PB_STAGE_FULL));   // first arrival: the zeroed tiles
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(BAR(PB_STAGE_FULL));   // second arrival: index and beta stored
                if (kk >= 1 && !wait_bar(BAR(PB_VSTAGE_FREE), (kk - 1) & 1, abort_flag)) break;
                if (lane == 0) {
                    if (transition) {
                        mbar_arrive(BAR(PB_VSTAGE_FULL));   // v = 0: the tile was cleared once
                    } else {
                        mbar_arrive_expect_tx(BAR(PB_VSTAGE_FULL), VSTAGE_TX);
                        tma_load_3d(sbase + PR_STG + STG_V, &maps.v, BAR(PB_VSTAGE_FULL), 0, h, row);
                        tma_load_3d(sbase + PR_STG + STG_V + 8192, &maps.v, BAR(PB_VSTAGE_FULL), 64, h, row);
                    }
                }
                __syncwarp();
            }
        } else if (warp == 3) {
            // ---- publisher: finished parts of the operand set (smem) -> ring slot (global),
            // each by bulk stores as soon as the part is final
            volatile uint32_t *chunkq = reinterpret_cast<volatile uint32_t *>(miscg + M_CHUNKQ);
            for (int kk = 0;; ++kk) {
                // part A of the local chunk kk is final (or, past the last chunk, the end signal)
                if (!wait_bar(BAR(PB_OUTA_READY), kk & 1, abort_flag)) break;
                const int m = static_cast<int>(chunkq[kk & 3]);
                if (m >= nch) break;
                const int r = m % NRING;
                unsigned char *set = ring + static_cast<uint64_t>(r) * SET_STRIDE;
#ifdef KDA_TEST_HOOKS
                if (m == g_kda_test_skip_chunk) {
                    // hand the tiles back as if published, but never signal the ring slot
                    if (lane == 0) {
                        mbar_arrive(BAR(PB_OUTA_FREE));
                        mbar_arrive(BAR(PB_VSTAGE_FREE));
                    }
                    __syncwarp();
                    if (!wait_bar(BAR(PB_OUTB_READY), kk & 1, abort_flag)) break;
                    if (!wait_bar(BAR(PB_OUTC_READY), kk & 1, abort_flag)) break;
                    if (lane == 0) mbar_arrive(BAR(PB_OUTC_FREE));
                    __syncwarp();
                    continue;
                }
#endif
                // the ring slot must have been pulled by the chain CTA (chunk m - NRING)
                if (m >= NRING && !wait_count_remote(mapa(sbase + CH_MISC + M_CONSUMED, 0),
                                                     static_cast<uint32_t>(m - NRING + 1), abort_flag))
                    break;
                if (lane == 0) KDA_TRACE_POINT(m, 18);
                if (lane == 0) {
                    KDA_TRACE_POINT(m, 19);
                    bulk_s2g(set + SET_KT, sbase + PR_KC, 16384);
                    bulk_s2g(set + SET_V, sbase + PR_STG + STG_V, 16384);
                    bulk_commit();
                    bulk_wait_read0();
                    mbar_arrive(BAR(PB_OUTA_FREE));     // Kt^T may be overwritten
                    mbar_arrive(BAR(PB_VSTAGE_FREE));   // the next value tile may be loaded
                }
                __syncwarp();
                // part C, final once the solve is done: it is on its way while W' runs, so that
                // only part B is left to write when the chunk ends
                if (!wait_bar(BAR(PB_OUTC_READY), kk & 1, abort_flag)) break;
                if (lane == 0) {
                    KDA_TRACE_POINT(m, 20);
                    bulk_s2g(set + SET_T, sbase + PR_AVT, 8192);
                    bulk_s2g(set + SET_AQK, sbase + PR_AVT + 8192, 8192);
                    bulk_s2g(set + SET_DEC, misc + M_DEC + (kk & 1) * 512, 512);
                    bulk_commit();
                    KDA_TRACE_POINT(m, 21);
                }
                __syncwarp();
                if (!wait_bar(BAR(PB_OUTB_READY), kk & 1, abort_flag)) break;
                if (lane == 0) {
                    KDA_TRACE_POINT(m, 22);
                    bulk_s2g(set + SET_W, sbase + PR_T, 16384);
                    bulk_s2g(set + SET_Q, sbase + PR_AKK, 16384);
                    bulk_commit();
                    bulk_wait_read0();   // parts C and B read out
                    KDA_TRACE_POINT(m, 23);
                    mbar_arrive(BAR(PB_OUTC_FREE));
                    bulk_wait0();
                    KDA_TRACE_POINT(m, 24);
                    fence_proxy_async_global();
                    mbar_arrive_remote(mapa(sbase + CH_MISC + M_BAR + 8u * (CB_READY + r), 0));
                    KDA_TRACE_POINT(m, 8);
                }
                __syncwarp();
            }
        } else if (warp >= 4) {
            // ---- chunk preparation: 8 warps, 256 threads. Outgoing tiles are assembled in
            // dead workspace: Kt^T over Kc^T, -W^T over the fp32 T, Qd^T over the fp32 A.
            const int t = tid - 128;
            const int q4 = warp & 3, half = (warp - 4) >> 2;
            const int lrow = q4 * 32 + lane;                 // TMEM lane in the epilogues
            const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
            float *wsf = reinterpret_cast<float *>(sgen);
            float *ega_s = reinterpret_cast<float *>(miscg + M_EGA);
            float *dec_all = reinterpret_cast<float *>(miscg + M_DEC);
            volatile uint32_t *chunkq = reinterpret_cast<volatile uint32_t *>(miscg + M_CHUNKQ);
            // the blocks of T' above the diagonal are never written per chunk: clear both T' tiles
            for (int e = t; e < 512; e += 256) {
                st_shared_v4(sbase + PR_AVT + e * 16, 0u, 0u, 0u, 0u);   // rows 0..63 (T')
                st_shared_v4(sbase + PR_TB + e * 16, 0u, 0u, 0u, 0u);
            }
            if (transition) {
                // v = 0 for a transition run: the value tile is never loaded; each thread clears the
                // 16-byte pieces it converts every chunk
#pragma unroll
                for (int c2 = 0; c2 < 4; ++c2) st_shared_v4(sbase + PR_STG + STG_V + (t + 256 * c2) * 16, 0u, 0u, 0u, 0u);
            }
            // A wait that gives up (abort) does not leave the loop on its own: the 8 warps leave
            // together at the next named barrier, which ORs the abort flag over them.
            for (int kk = 0;; ++kk) {
#ifdef KDA_TRACE
                const unsigned long long trace_start = globaltimer();
#endif
                // part A of the previous set (over Kc^T) must have been read out by the publisher;
                // part B (over T) is covered by the wait for part C before T is next written
                if (kk >= 1) wait_bar(BAR(PB_OUTA_FREE), (kk - 1) & 1, abort_flag);
#ifdef KDA_TRACE
                const unsigned long long trace_afree = globaltimer();
#endif
                wait_bar(BAR(PB_STAGE_FULL), kk & 1, abort_flag);
#ifdef KDA_TRACE
                const unsigned long long trace_sfull = globaltimer();
#endif
                const int m = static_cast<int>(chunkq[kk & 3]);   // this CTA's kk-th chunk
                // past the last chunk the phase below still runs up to its first barrier (on stale
                // tiles, which is harmless), and every warp leaves there together
                const bool no_chunk = m >= nch;
                // rows of this chunk that hold tokens (the others are zero in the staging tiles)
                const int Lrows = static_cast<int>(eos - (bos + static_cast<int64_t>(m) * C) < C
                                                       ? eos - (bos + static_cast<int64_t>(m) * C)
                                                       : C);
                // 1 / ||x|| of each staged row of q (0..63) and k (64..127); a zero row gets a finite
                // factor and stays zero
                float *invn = reinterpret_cast<float *>(miscg + M_INVN);
                if constexpr (kNorm) {
#pragma unroll 1
                    for (int rr = warp - 4; rr < 2 * C; rr += 8) {
                        const uint32_t a = sbase + PR_STG + (rr < C ? STG_Q : STG_K) +
                                           static_cast<uint32_t>((rr & (C - 1)) * 256 + lane * 8);
                        uint32_t w0, w1;
                        asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(w0), "=r"(w1) : "r"(a) : "memory");
                        const float x0 = lo_bf(w0), x1 = hi_bf(w0), x2 = lo_bf(w1), x3 = hi_bf(w1);
                        float ss = x0 * x0 + x1 * x1 + x2 * x2 + x3 * x3;
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
                        if (lane == 0) invn[rr] = rsqrtf(fmaxf(ss, 1e-24f));
                    }
                    if (named_bar_any(2, 256, *abort_flag != 0)) break;
                }
                // a staged q / k element, normalised when asked
                auto qn = [&](int r, float x) -> float {
                    if constexpr (kNorm) return x * invn[r];
                    return x;
                };
                auto kn = [&](int r, float x) -> float {
                    if constexpr (kNorm) return x * invn[C + r];
                    return x;
                };
                const float *beta_s = reinterpret_cast<const float *>(miscg + M_BETAQ) + (kk & 1) * C;
#ifdef KDA_TRACE
                if (t == 0 && blockIdx.x / 4 == KDA_TRACE_CLUSTER_ID && m < 64) {
                    g_kda_trace[(rank * 64 + m) * 48 + 0] = trace_start;
                    g_kda_trace[(rank * 64 + m) * 48 + 25] = trace_afree;
                    g_kda_trace[(rank * 64 + m) * 48 + 26] = trace_sfull;
                }
#endif
                if (t == 0) KDA_TRACE_POINT(m, 1);

                // -------- S1: running log-decay and the anchored factors. A thread owns a pair of
                // adjacent channels (c0, c0 + 1) over one quarter of the rows (16 tokens), so q and k
                // are read as bf16 pairs and g as float pairs. It takes its rows in two passes of 8;
                // lanes 4-7 of every 8 take the two halves in the other order, so that each store
                // instruction covers all eight swizzle phases. Rows past the end of a partial chunk
                // were zeroed above.
                uint32_t ktr[16];   // Kt^T of this thread: 4 fp16 pairs x 2 passes x 2 channels
                const bool flip = (lane >> 2) & 1;
                bool robust = false;   // this chunk takes the sub-block path (CTA-uniform)
                {
                    // the two half-warps take channel groups of different parity, so that their
                    // bf16-pair loads of q and k (rows 16 apart) fall on disjoint banks
                    const int grp = ((warp - 4) & 3) ^ (lane >> 4);
                    const int cp = grp * 16 + (lane & 15);
                    const int tq = 2 * ((warp - 4) >> 2) + (lane >> 4);
                    const int c0 = 2 * cp, r0 = 16 * tq;
                    const int rp0 = r0 + (flip ? 8 : 0), rp1 = r0 + (flip ? 0 : 8);   // first row of each pass
                    const float *gst = reinterpret_cast<const float *>(sgen + PR_STG + STG_G);
                    const uint32_t *gbf = reinterpret_cast<const uint32_t *>(sgen + PR_STG + STG_G + 16384);
                    const float *gsc = reinterpret_cast<const float *>(miscg + M_GSCALQ) + (kk & 1) * C;
                    const bool act = (p.flags & kFlagGateLogsigmoid) && kGate != kGateScalar;
                    const uint32_t *qst = reinterpret_cast<const uint32_t *>(sgen + PR_STG + STG_Q);
                    const uint32_t *kst = reinterpret_cast<const uint32_t *>(sgen + PR_STG + STG_K);
                    // g of the channel pair in log2 units (x, y = channels c0, c0 + 1), in pass order
                    const float2 l2e = make_float2(kLog2e, kLog2e);
                    float2 gv[16];
                    float2 sp[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int rr = (i < 8 ? rp0 : rp1) + (i & 7);
                        if constexpr (kGate == kGateF32) {
                            gv[i] = *reinterpret_cast<const float2 *>(gst + rr * D + c0);
                        } else if constexpr (kGate == kGateBF16) {
                            const uint32_t w = gbf[rr * (D / 2) + cp];
                            gv[i] = make_float2(lo_bf(w), hi_bf(w));
                        } else {
                            gv[i] = make_float2(gsc[rr], gsc[rr]);
                        }
                    }
                    if (act) {
                        // g holds the gate's pre-activation: log alpha = logsigmoid(g); rows past the
                        // end of the sequence keep log alpha = 0
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const int rr = (i < 8 ? rp0 : rp1) + (i & 7);
                            gv[i] = rr < Lrows ? make_float2(log2_sigmoid(gv[i].x), log2_sigmoid(gv[i].y))
                                               : make_float2(0.f, 0.f);
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 16; ++i) gv[i] = f2_mul(gv[i], l2e);
                    }
#pragma unroll
                    for (int i = 0; i < 16; ++i) sp[i >> 3] = f2_add(sp[i >> 3], gv[i]);
                    // row-quarter sums of g per channel, [4][128] floats in the solve's scratch
                    float *gq = reinterpret_cast<float *>(sgen + PR_P);
                    const float2 qsum = f2_add(sp[0], sp[1]);
                    *reinterpret_cast<float2 *>(gq + tq * 128 + c0) = qsum;
                    // one barrier serves both the exchange and the choice of path: it ORs "this
                    // quarter decays beyond the single anchor's range" with the abort flag; only when
                    // that is set does a second barrier tell the two apart
                    const bool unsafe = !(qsum.x >= -kQuarterRangeLog2) || !(qsum.y >= -kQuarterRangeLog2);
                    if (__builtin_expect(named_bar_any(2, 256, unsafe || no_chunk || *abort_flag != 0), 0)) {
                        if (named_bar_any(2, 256, no_chunk || *abort_flag != 0)) {
                            if (t == 0) mbar_arrive(BAR(PB_OUTA_READY));   // the publisher's end signal
                            break;
                        }
                        robust = true;
                        // the sub-block path floors the gates: again with the floored sums
                        sp[0] = sp[1] = make_float2(0.f, 0.f);
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            gv[i] = make_float2(fmaxf(gv[i].x, kFloorLog2), fmaxf(gv[i].y, kFloorLog2));
                            sp[i >> 3] = f2_add(sp[i >> 3], gv[i]);
                        }
                        *reinterpret_cast<float2 *>(gq + tq * 128 + c0) = f2_add(sp[0], sp[1]);
                        if (named_bar_any(2, 256, *abort_flag != 0)) break;
                    }
                    if (t == 0) KDA_TRACE_POINT(m, 30);
                    float2 qs[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) qs[q] = *reinterpret_cast<const float2 *>(gq + q * 128 + c0);
                    const float2 ga = f2_add(qs[0], qs[1]);                  // G at the anchor row 31
                    const float2 gl = f2_add(ga, f2_add(qs[2], qs[3]));      // G at row 63
                    if (__builtin_expect(robust, 0)) {
                        // ---- sub-block path, part 1 (this thread's rows and channels): the running
                        // log-decay G over the chunk, written over g in the staging tile for the factor
                        // phase, Kt = K 2^(Gl - G) (<= 1), e^Gl; the anchored factors are not used.
                        float2 run = make_float2(0.f, 0.f);
#pragma unroll
                        for (int q = 0; q < 3; ++q)
                            if (q < tq) run = f2_add(run, qs[q]);
                        float *gstw = reinterpret_cast<float *>(sgen + PR_STG + STG_G);
#pragma unroll
                        for (int ps = 0; ps < 2; ++ps) {
                            // pass 0 starts after the lower 8 rows when it is the upper half
                            float2 Y = (ps == 0) == flip ? f2_add(run, sp[ps ^ 1]) : run;
                            const int rb = ps == 0 ? rp0 : rp1;
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                float2 kt[2];
#pragma unroll
                                for (int u = 0; u < 2; ++u) {
                                    const int i = ps * 8 + 2 * e + u, rr = rb + 2 * e + u;
                                    Y = f2_add(Y, gv[i]);
                                    *reinterpret_cast<float2 *>(gstw + rr * D + c0) = Y;
                                    const uint32_t kw = kst[rr * (D / 2) + cp];
                                    kt[u] = f2_mul(make_float2(kn(rr, lo_bf(kw)), kn(rr, hi_bf(kw))),
                                                   make_float2(ex2_approx(gl.x - Y.x), ex2_approx(gl.y - Y.y)));
                                }
                                ktr[ps * 4 + e] = pack_f16(kt[0].x, kt[1].x);
                                ktr[8 + ps * 4 + e] = pack_f16(kt[0].y, kt[1].y);
                            }
                        }
                        if (tq == 0) {
                            *reinterpret_cast<float2 *>(dec_all + (kk & 1) * 128 + c0) =
                                make_float2(ex2_approx(gl.x), ex2_approx(gl.y));
                            // W and Qd are built from the chunk-start-relative factors directly
                            *reinterpret_cast<float2 *>(ega_s + c0) = make_float2(1.f, 1.f);
                        }
                    } else {
                    // Y = G - Ga, running over a pass's rows; Y0 is its value before row r0
                    float2 Y0 = make_float2(-ga.x, -ga.y);
#pragma unroll
                    for (int q = 0; q < 3; ++q)
                        if (q < tq) Y0 = f2_add(Y0, qs[q]);
                    const float2 ec = make_float2(ex2_approx(gl.x - ga.x), ex2_approx(gl.y - ga.y));
                    // pass 0 starts after the rows of the lower half when it is the upper half
                    const float2 y1 = f2_add(Y0, sp[1]);
                    float2 Y = flip ? y1 : Y0;
#pragma unroll
                    for (int ps = 0; ps < 2; ++ps) {
                        if (ps == 1) Y = flip ? Y0 : Y;
                        const int rb = ps == 0 ? rp0 : rp1;
                        uint32_t hx[4], hy[4], qx4[4], qy4[4], cx[4], cy[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            float2 kh[2], qh[2], kc[2], kt[2];
#pragma unroll
                            for (int u = 0; u < 2; ++u) {
                                const int i = ps * 8 + 2 * e + u, rr = rb + 2 * e + u;
                                Y = f2_add(Y, gv[i]);
                                const float2 ep = make_float2(ex2_approx(Y.x), ex2_approx(Y.y));
                                const float2 em = make_float2(ex2_approx(-Y.x), ex2_approx(-Y.y));
                                const uint32_t kw = kst[rr * (D / 2) + cp];
                                const uint32_t qw = qst[rr * (D / 2) + cp];
                                const float2 k2 = make_float2(kn(rr, lo_bf(kw)), kn(rr, hi_bf(kw)));
                                const float2 q2 = make_float2(qn(rr, lo_bf(qw)), qn(rr, hi_bf(qw)));
                                kh[u] = f2_mul(k2, ep);
                                qh[u] = f2_mul(q2, ep);
                                kc[u] = f2_mul(k2, em);
                                kt[u] = f2_mul(kc[u], ec);
                            }
                            hx[e] = pack_bf16(kh[0].x, kh[1].x);
                            hy[e] = pack_bf16(kh[0].y, kh[1].y);
                            qx4[e] = pack_bf16(qh[0].x, qh[1].x);
                            qy4[e] = pack_bf16(qh[0].y, qh[1].y);
                            cx[e] = pack_bf16(kc[0].x, kc[1].x);
                            cy[e] = pack_bf16(kc[0].y, kc[1].y);
                            ktr[ps * 4 + e] = pack_f16(kt[0].x, kt[1].x);
                            ktr[8 + ps * 4 + e] = pack_f16(kt[0].y, kt[1].y);
                        }
                        const int j = (rb >> 3);   // 16-byte chunk (8 tokens) of a channel row
#pragma unroll
                        for (int tile = 0; tile < 3; ++tile) {
                            const uint32_t base = sbase + (tile == 0 ? PR_KH : (tile == 1 ? PR_QH : PR_KC));
                            const uint32_t *X = tile == 0 ? hx : (tile == 1 ? qx4 : cx);
                            const uint32_t *Yw = tile == 0 ? hy : (tile == 1 ? qy4 : cy);
                            st_shared_v4(base + sw128(c0, j), X[0], X[1], X[2], X[3]);
                            st_shared_v4(base + sw128(c0 + 1, j), Yw[0], Yw[1], Yw[2], Yw[3]);
                        }
                    }
                    if (tq == 0) {
                        *reinterpret_cast<float2 *>(dec_all + (kk & 1) * 128 + c0) =
                            make_float2(ex2_approx(gl.x), ex2_approx(gl.y));
                        *reinterpret_cast<float2 *>(ega_s + c0) = make_float2(ex2_approx(ga.x), ex2_approx(ga.y));
                    }
                    }   // single-anchor path
                    if (t == 0) KDA_TRACE_POINT(m, 31);
                }
                if (__builtin_expect(robust, 0)) {
                    // ---- sub-block path, part 2: the decayed blocks by 16-row block R, each with its own
                    // anchor row a_R = 16R + 7:
                    //   left  (A operand rows, all R):  [K; Q] 2^(G - G_aR)     rows of block R
                    //   right (B operand of product R): K 2^(G_aR - G)          rows 0 .. 16R + 15, zero after
                    // so that product R holds exactly the rows of block R of [Akk_raw; Aqk]. With the
                    // floor, |G - G_aR| stays below 8 x 14.43 inside a block, and the right factor of an
                    // earlier block is <= 1. The four right factors go to tiles that are dead until the
                    // products have completed (Kt^T, A, T and the [T'; Aqk] tile), so the previous set's
                    // part C must have been read out.
                    if (named_bar_any(2, 256, *abort_flag != 0)) break;
                    if (kk >= 1) wait_bar(BAR(PB_OUTC_FREE), (kk - 1) & 1, abort_flag);
                    const int c = t & 127, hh = t >> 7;        // key channel, token half
                    const float *G = reinterpret_cast<const float *>(sgen + PR_STG + STG_G);
                    const uint16_t *kb = reinterpret_cast<const uint16_t *>(sgen + PR_STG + STG_K);
                    const uint16_t *qb = reinterpret_cast<const uint16_t *>(sgen + PR_STG + STG_Q);
                    float ganc[4];
#pragma unroll
                    for (int R = 0; R < 4; ++R) ganc[R] = G[(16 * R + 7) * D + c];
                    const uint32_t right[4] = {sbase + PR_KC, sbase + PR_AKK, sbase + PR_T, sbase + PR_AVT};
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        const int j = 4 * hh + jj, R = j >> 1;   // 8-token group, its 16-row block
                        float gg[8], kf[8], qf[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int r = 8 * j + e;
                            gg[e] = G[r * D + c];
                            kf[e] = kn(r, bf2f(kb[r * D + c]));
                            qf[e] = qn(r, bf2f(qb[r * D + c]));
                        }
                        // anchor of this group's block, selected without a run-time index into ganc
                        const float ga_own = (jj >> 1) ? (hh ? ganc[3] : ganc[1]) : (hh ? ganc[2] : ganc[0]);
                        uint32_t kw[4], qw[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float f0 = ex2_approx(gg[2 * e] - ga_own), f1 = ex2_approx(gg[2 * e + 1] - ga_own);
                            kw[e] = pack_bf16(kf[2 * e] * f0, kf[2 * e + 1] * f1);
                            qw[e] = pack_bf16(qf[2 * e] * f0, qf[2 * e + 1] * f1);
                        }
                        st_shared_v4(sbase + PR_KH + sw128(c, j), kw[0], kw[1], kw[2], kw[3]);
                        st_shared_v4(sbase + PR_QH + sw128(c, j), qw[0], qw[1], qw[2], qw[3]);
#pragma unroll
                        for (int Rp = 0; Rp < 4; ++Rp) {
                            uint32_t w[4] = {0u, 0u, 0u, 0u};
                            if (Rp >= R) {
#pragma unroll
                                for (int e = 0; e < 4; ++e)
                                    w[e] = pack_bf16(kf[2 * e] * ex2_approx(ganc[Rp] - gg[2 * e]),
                                                     kf[2 * e + 1] * ex2_approx(ganc[Rp] - gg[2 * e + 1]));
                            }
                            st_shared_v4(right[Rp] + sw128(c, j), w[0], w[1], w[2], w[3]);
                        }
                    }
                }
                fence_proxy_async_smem();
                if (named_bar_any(2, 256, *abort_flag != 0)) break;
                // The prep MMAs are issued by warp 4 right after the barrier that ends the phase
                // writing their operands (no hop through another warp); one elected lane issues.
                if (warp == 4) {
                    tc_fence_after();
                    if (elect_one()) {
                        if (__builtin_expect(!robust, 1)) {
                            mbar_arrive(BAR(PB_STAGE_FREE));
                            // [Kh; Qh] Kc^T : A = Kh^T | Qh^T (MN-major, 64-row blocks 16 KB apart), B = Kc^T
                            for (int ks = 0; ks < 8; ++ks)
                                mma_f16(tmem + COL_P1, smem_desc(sbase + PR_KH + ks * 2048, 16384, 1024, kSwizzle128),
                                        smem_desc(sbase + PR_KC + ks * 2048, 16384, 1024, kSwizzle128), ID_P1, ks > 0);
                        } else {
                            // the staging tile is still read after these products (G, q, k)
#pragma unroll
                            for (int R = 0; R < 4; ++R) {
                                const uint32_t rt = sbase + (R == 0 ? PR_KC : R == 1 ? PR_AKK : R == 2 ? PR_T : PR_AVT);
                                for (int ks = 0; ks < 8; ++ks)
                                    mma_f16(tmem + COL_RB + 64 * R,
                                            smem_desc(sbase + PR_KH + ks * 2048, 16384, 1024, kSwizzle128),
                                            smem_desc(rt + ks * 2048, 16384, 1024, kSwizzle128), ID_P1, ks > 0);
                            }
                        }
                        mma_commit(BAR(PB_P1_DONE));
                        KDA_TRACE_POINT(m, 2);
                    }
                    __syncwarp();
                }
                // value tile bf16 -> fp16 in place (B operand of the value-side MMA)
                wait_bar(BAR(PB_VSTAGE_FULL), kk & 1, abort_flag);
#pragma unroll
                for (int c2 = 0; c2 < 4; ++c2) {
                    const uint32_t a = sbase + PR_STG + STG_V + (t + 256 * c2) * 16;
                    const uint4 x = ld_shared_v4(a);
                    st_shared_v4(a, pack_f16(lo_bf(x.x), hi_bf(x.x)), pack_f16(lo_bf(x.y), hi_bf(x.y)),
                                 pack_f16(lo_bf(x.z), hi_bf(x.z)), pack_f16(lo_bf(x.w), hi_bf(x.w)));
                }
                // -------- S2 epilogue: A (fp32, masked, beta-scaled) and Aqk (fp16 + bf16); Kt^T out
                // (part C of the previous set, over A / T and the AV operand, must be read out)
                if (kk >= 1) wait_bar(BAR(PB_OUTC_FREE), (kk - 1) & 1, abort_flag);
                wait_bar(BAR(PB_P1_DONE), kk & 1, abort_flag);
                tc_fence_after();
                if (t == 0) KDA_TRACE_POINT(m, 3);
                {
                    {
                        const int cp = (((warp - 4) & 3) ^ (lane >> 4)) * 16 + (lane & 15);   // as in S1
                        const int tq = 2 * ((warp - 4) >> 2) + (lane >> 4);
#pragma unroll
                        for (int ch = 0; ch < 2; ++ch)
#pragma unroll
                            for (int h8 = 0; h8 < 2; ++h8) {
                                const uint32_t *w4 = ktr + ch * 8 + h8 * 4;
                                st_shared_v4(sbase + PR_KC + sw128(2 * cp + ch, 2 * tq + (h8 ^ (flip ? 1 : 0))), w4[0],
                                             w4[1], w4[2], w4[3]);
                            }
                    }
                    // the products' rows: on the common path one 32-column load per thread; on the
                    // sub-block path row lrow lives in the product of its block (lrow & 63) >> 4, so
                    // lanes 0-15 and 16-31 of a warp take it from two products, one pass each
                    const int npass = robust ? 2 : 1;
                    for (int pass = 0; pass < npass; ++pass) {
                        uint32_t a[32];
                        const uint32_t col = robust ? COL_RB + 64u * static_cast<uint32_t>(2 * (q4 & 1) + pass) + half * 32
                                                    : COL_P1 + half * 32;
                        tmem_ld32(tmem + lane_base + col, a);
                        tmem_wait_ld();
                        if (t == 0) KDA_TRACE_POINT(m, 27);
                        if (robust && (lane >> 4) != pass) continue;
                        if (lrow < 64) {
                            const int rr = lrow;
                            const float br = beta_s[rr];
                            float *rowp = wsf + PR_AKK / 4 + rr * AKK_LD + half * 32;
#pragma unroll
                            for (int j = 0; j < 8; ++j) {
                                float v4[4];
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    const int i = half * 32 + 4 * j + e;
                                    v4[e] = i < rr ? br * __uint_as_float(a[4 * j + e]) : 0.f;
                                }
                                *reinterpret_cast<float4 *>(rowp + 4 * j) = make_float4(v4[0], v4[1], v4[2], v4[3]);
                            }
                        } else {
                            const int rr = lrow - 64;
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                float v8[8];
#pragma unroll
                                for (int e = 0; e < 8; ++e) {
                                    const int i = half * 32 + 8 * j + e;
                                    v8[e] = i <= rr ? __uint_as_float(a[8 * j + e]) : 0.f;
                                }
                                const int jj = half * 4 + j;
                                st_shared_v4(sbase + PR_AVT + sw128(64 + rr, jj), pack_f16(v8[0], v8[1]),
                                             pack_f16(v8[2], v8[3]), pack_f16(v8[4], v8[5]), pack_f16(v8[6], v8[7]));
                            }
                        }
                    }
                    if (t == 0) KDA_TRACE_POINT(m, 32);
                    // blocks of T read as zeros by the fixed-length products below
                    float *T = wsf + PR_T / 4;
                    T[(t >> 4) * AKK_LD + 16 + (t & 15)] = 0.f;               // rows 0-15, cols 16-31
                    T[(32 + (t >> 4)) * AKK_LD + 48 + (t & 15)] = 0.f;        // rows 32-47, cols 48-63
                    // S3 (a): the four 16 x 16 diagonal blocks of T = (I + A)^-1. Warp 4 has just
                    // written blocks 0 and 1 of A, warp 9 blocks 2 and 3; each lane solves one column
                    // of its block by forward substitution, right-looking: once x[j] is final it is
                    // folded into every later row, so a row costs one FMA on the dependent path.
                    if (warp == 4 || warp == 9) {
                        __syncwarp();
                        const int wb = (warp == 4 ? 0 : 2) + (lane >> 4), li = lane & 15;
                        const float *Ab = wsf + PR_AKK / 4 + 16 * wb * AKK_LD + 16 * wb;
                        float x[16];
#pragma unroll
                        for (int r = 0; r < 16; ++r) x[r] = r == li ? 1.f : 0.f;
                        // A is read four columns at a time (one 16-byte broadcast load per row and
                        // column group) just before the group's four steps
#pragma unroll
                        for (int g = 0; g < 4; ++g) {
                            float4 a4[16];
#pragma unroll
                            for (int r = 4 * g + 1; r < 16; ++r)
                                a4[r] = *reinterpret_cast<const float4 *>(Ab + r * AKK_LD + 4 * g);
#pragma unroll
                            for (int jj = 0; jj < 4; ++jj) {
                                const int j = 4 * g + jj;
#pragma unroll
                                for (int r = j + 1; r < 16; ++r) {
                                    const float a = jj == 0 ? a4[r].x : jj == 1 ? a4[r].y : jj == 2 ? a4[r].z : a4[r].w;
                                    x[r] = fmaf(-a, x[j], x[r]);
                                }
                            }
                        }
#pragma unroll
                        for (int r = 0; r < 16; ++r) T[(16 * wb + r) * AKK_LD + 16 * wb + li] = x[r];
                    }
                }
                if (__builtin_expect(robust, 0)) {
                    // ---- sub-block path, part 3 (its products have completed): the W and Qd operands
                    // from the chunk-start-relative factors, K 2^G and Q 2^G (<= 1), over the left factors
                    // (the scale e^Ga applied to them later is 1 on this path); the T' rows of the
                    // [T'; Aqk] tile held a right factor and must read as zero above the diagonal again
                    const int c = t & 127, hh = t >> 7;
                    const float *G = reinterpret_cast<const float *>(sgen + PR_STG + STG_G);
                    const uint16_t *kb = reinterpret_cast<const uint16_t *>(sgen + PR_STG + STG_K);
                    const uint16_t *qb = reinterpret_cast<const uint16_t *>(sgen + PR_STG + STG_Q);
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        const int j = 4 * hh + jj;
                        uint32_t kw[4], qw[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int r = 8 * j + 2 * e;
                            const float f0 = ex2_approx(G[r * D + c]), f1 = ex2_approx(G[(r + 1) * D + c]);
                            kw[e] = pack_bf16(kn(r, bf2f(kb[r * D + c])) * f0, kn(r + 1, bf2f(kb[(r + 1) * D + c])) * f1);
                            qw[e] = pack_bf16(qn(r, bf2f(qb[r * D + c])) * f0, qn(r + 1, bf2f(qb[(r + 1) * D + c])) * f1);
                        }
                        st_shared_v4(sbase + PR_KH + sw128(c, j), kw[0], kw[1], kw[2], kw[3]);
                        st_shared_v4(sbase + PR_QH + sw128(c, j), qw[0], qw[1], qw[2], qw[3]);
                    }
                    for (int e = t; e < 512; e += 256) st_shared_v4(sbase + PR_AVT + e * 16, 0u, 0u, 0u, 0u);
                }
                if (t == 0) KDA_TRACE_POINT(m, 28);
                fence_proxy_async_smem();
                tc_fence_before();
                if (named_bar_any(2, 256, *abort_flag != 0)) break;
                if (t == 0) {
                    mbar_arrive(BAR(PB_OUTA_READY));
                    if (__builtin_expect(robust, 0)) mbar_arrive(BAR(PB_STAGE_FREE));   // q, k and G have been read
                    KDA_TRACE_POINT(m, 9);
                }

                // -------- S3: T = (I + A)^-1 by recursive blocking:
                //   (a) the four 16 x 16 diagonal blocks by forward substitution (done above, in the
                //       S2 epilogue, by the warps that wrote those blocks of A),
                //   (b) the two 16 x 16 blocks below them inside each 32 x 32 diagonal block,
                //   (c) the 32 x 32 block below the diagonal,
                // each off-diagonal block as  T_IJ = -T_II (A_IJ T_JJ). The products of (b) and (c)
                // are warp-level tf32 MMAs (m16n8k8) on operands read straight from the fp32 tiles:
                // a warp owns a 16 x 8 tile of the result, so each operand element is read by a
                // few lanes instead of once per output column.
                {
                    const float *A = wsf + PR_AKK / 4;
                    float *T = wsf + PR_T / 4;
                    float *P = wsf + PR_P / 4;   // 8 tiles of 16 x 8 floats (row stride 8)
                    if (t == 0) KDA_TRACE_POINT(m, 10);
                    // T' = T diag(beta) is written straight into its two operand tiles as each block of
                    // T becomes final: fp16 (rows 0..63 of the [T'; Aqk] tile) and bf16 (TB); the blocks
                    // above the diagonal are zero and were cleared once.
                    // address of T'[r][c..] (c a multiple of 2) in a K-major 128B-swizzled fp16/bf16 tile
                    auto tp_addr = [&](uint32_t base, int r, int c) -> uint32_t {
                        return base + sw128(static_cast<uint32_t>(r), static_cast<uint32_t>(c >> 3)) +
                               static_cast<uint32_t>(c & 7) * 2u;
                    };
                    const int w8 = warp - 4, g8 = lane >> 2, tg = lane & 3;   // MMA fragment coordinates
                    // a 16 x 8 A fragment (rows r0 + g8, r0 + g8 + 8; columns c0 + tg, c0 + tg + 4) of a
                    // row-major fp32 tile with row stride AKK_LD
                    auto frag_a = [&](const float *M, int r0, int c0, uint32_t (&a)[4]) {
                        const float *p0 = M + (r0 + g8) * AKK_LD + c0 + tg;
                        a[0] = to_tf32(p0[0]);
                        a[1] = to_tf32(p0[8 * AKK_LD]);
                        a[2] = to_tf32(p0[4]);
                        a[3] = to_tf32(p0[8 * AKK_LD + 4]);
                    };
                    // an 8 x 8 B fragment (rows k0 + tg, k0 + tg + 4; column n0 + g8) of a row-major tile
                    auto frag_b = [&](const float *M, int ld, int k0, int n0, uint32_t (&b)[2]) {
                        b[0] = to_tf32(M[(k0 + tg) * ld + n0 + g8]);
                        b[1] = to_tf32(M[(k0 + tg + 4) * ld + n0 + g8]);
                    };
                    // T' (= -acc diag(beta)) of the 16 x 8 result tile at rows r0, columns n0
                    auto store_tprime = [&](const float (&acc)[4], int r0, int n0) {
                        const int c = n0 + 2 * tg;
                        const float b0 = -beta_s[c], b1 = -beta_s[c + 1];
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            const float x0 = acc[2 * hh] * b0, x1 = acc[2 * hh + 1] * b1;
                            st_shared_u32(tp_addr(sbase + PR_AVT, r0 + g8 + 8 * hh, c), pack_f16(x0, x1));
                            st_shared_u32(tp_addr(sbase + PR_TB, r0 + g8 + 8 * hh, c), pack_bf16(x0, x1));
                        }
                    };
                    if (w8 < 4) {
                        // (b) warp (blk, nt): T_IJ[:, 8 nt .. 8 nt + 7] for I = 2 blk + 1, J = 2 blk
                        const int blk = w8 >> 1, nt = w8 & 1, I = 2 * blk + 1, J = 2 * blk;
                        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                        for (int ks = 0; ks < 2; ++ks) {   // P = A_IJ T_JJ[:, n-tile]
                            if (ks < nt) continue;         // T_JJ is lower triangular
                            uint32_t a[4], b[2];
                            frag_a(A, 16 * I, 16 * J + 8 * ks, a);
                            frag_b(T, AKK_LD, 16 * J + 8 * ks, 16 * J + 8 * nt, b);
                            mma_tf32_16x8x8(acc, a, b);
                        }
                        // the product tile becomes the B operand of the next step through this warp's
                        // own scratch tile
                        float *Pw = P + w8 * 128;
                        *reinterpret_cast<float2 *>(Pw + g8 * 8 + 2 * tg) = make_float2(acc[0], acc[1]);
                        *reinterpret_cast<float2 *>(Pw + (g8 + 8) * 8 + 2 * tg) = make_float2(acc[2], acc[3]);
                        __syncwarp();
                        float res[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                        for (int ks = 0; ks < 2; ++ks) {   // T_II P
                            uint32_t a[4], b[2];
                            frag_a(T, 16 * I, 16 * I + 8 * ks, a);
                            frag_b(Pw, 8, 8 * ks, 0, b);
                            mma_tf32_16x8x8(res, a, b);
                        }
                        // T_IJ = -T_II P: fp32 for (c), T' for the products
                        const int r = 16 * I + g8, c = 16 * J + 8 * nt + 2 * tg;
                        *reinterpret_cast<float2 *>(T + r * AKK_LD + c) = make_float2(-res[0], -res[1]);
                        *reinterpret_cast<float2 *>(T + (r + 8) * AKK_LD + c) = make_float2(-res[2], -res[3]);
                        store_tprime(res, 16 * I, 16 * J + 8 * nt);
                    } else {
                        // T' of the four diagonal blocks (final since (a)): 128 threads, one row and 8
                        // columns each
                        const int tt = t - 128, r = tt >> 1, c = (r & ~15) + 8 * (tt & 1);
                        const float4 t0 = *reinterpret_cast<const float4 *>(T + r * AKK_LD + c);
                        const float4 t1 = *reinterpret_cast<const float4 *>(T + r * AKK_LD + c + 4);
                        const float4 b0 = *reinterpret_cast<const float4 *>(beta_s + c);
                        const float4 b1 = *reinterpret_cast<const float4 *>(beta_s + c + 4);
                        const float x[8] = {t0.x * b0.x, t0.y * b0.y, t0.z * b0.z, t0.w * b0.w,
                                            t1.x * b1.x, t1.y * b1.y, t1.z * b1.z, t1.w * b1.w};
                        st_shared_v4(tp_addr(sbase + PR_AVT, r, c), pack_f16(x[0], x[1]), pack_f16(x[2], x[3]),
                                     pack_f16(x[4], x[5]), pack_f16(x[6], x[7]));
                        st_shared_v4(tp_addr(sbase + PR_TB, r, c), pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]),
                                     pack_bf16(x[4], x[5]), pack_bf16(x[6], x[7]));
                    }
                    if (t == 0) KDA_TRACE_POINT(m, 13);
                    if (named_bar_any(2, 256, *abort_flag != 0)) break;
                    if (t == 0) KDA_TRACE_POINT(m, 11);
                    // (c) warp (mt, nt): rows 32 + 16 mt .. + 15, columns 8 nt .. 8 nt + 7 of
                    //   P2 = A[32:, :32] T[:32, :32],  T[32:, :32] = -T[32:, 32:] P2.
                    // T[:32, :32] is lower triangular, so the n-tile nt needs k-steps nt .. 3 only;
                    // T[32:48, 48:64] is zero, so rows 32..47 need P2 rows 0..15 (their own tile) and
                    // rows 48..63 wait for that tile from the warp of the same nt (barrier 5 + nt).
                    {
                        const int mt = w8 >> 2, nt = w8 & 3;
                        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks) {
                            if (ks < nt) continue;
                            uint32_t a[4], b[2];
                            frag_a(A, 32 + 16 * mt, 8 * ks, a);
                            frag_b(T, AKK_LD, 8 * ks, 8 * nt, b);
                            mma_tf32_16x8x8(acc, a, b);
                        }
                        float *Pw = P + w8 * 128;   // P2 rows 16 mt .. 16 mt + 15, columns of n-tile nt
                        *reinterpret_cast<float2 *>(Pw + g8 * 8 + 2 * tg) = make_float2(acc[0], acc[1]);
                        *reinterpret_cast<float2 *>(Pw + (g8 + 8) * 8 + 2 * tg) = make_float2(acc[2], acc[3]);
                        if (mt == 0) {
                            named_bar_arrive(5 + nt, 64);   // the tile is written: rows 48..63 may read it
                        } else {
                            named_bar_sync(5 + nt, 64);
                        }
                        __syncwarp();
                        float res[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks) {
                            if (mt == 0 && ks >= 2) continue;
                            uint32_t a[4], b[2];
                            frag_a(T, 32 + 16 * mt, 32 + 8 * ks, a);
                            frag_b(P + ((ks >> 1) * 4 + nt) * 128, 8, 8 * (ks & 1), 0, b);
                            mma_tf32_16x8x8(res, a, b);
                        }
                        // final block of T; T itself is not read again, only T' is written
                        store_tprime(res, 32 + 16 * mt, 8 * nt);
                    }
                    if (t == 0) KDA_TRACE_POINT(m, 12);
                }
                if (t == 0) KDA_TRACE_POINT(m, 16);
                fence_proxy_async_smem();
                if (t == 0) KDA_TRACE_POINT(m, 17);
                if (named_bar_any(2, 256, *abort_flag != 0)) break;
                if (t == 0) mbar_arrive(BAR(PB_OUTC_READY));   // T', Aqk and e^Gl are final
                if (warp == 4) {
                    tc_fence_after();
                    if (elect_one()) {
                        // W'^T = Kh^T T'^T (bf16)
                        for (int ks = 0; ks < 4; ++ks)
                            mma_f16(tmem + COL_W, smem_desc(sbase + PR_KH + ks * 32, 16, 1024, kSwizzle128),
                                    smem_desc(sbase + PR_TB + ks * 32, 16, 1024, kSwizzle128), ID_W, ks > 0);
                        mma_commit(BAR(PB_WAV_DONE));
                        KDA_TRACE_POINT(m, 4);
                    }
                    __syncwarp();
                }
                // -------- Qd = Q e^G = Qh diag(e^Ga) (bf16, over the dead A workspace) while W' runs
                {
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int e = t + 256 * i, rr = e >> 3, jj = e & 7;
                        const uint4 qv = ld_shared_v4(sbase + PR_QH + sw128(rr, jj));
                        const float sc = ega_s[rr];
                        st_shared_v4(sbase + PR_AKK + sw128(rr, jj), pack_bf16(sc * lo_bf(qv.x), sc * hi_bf(qv.x)),
                                     pack_bf16(sc * lo_bf(qv.y), sc * hi_bf(qv.y)),
                                     pack_bf16(sc * lo_bf(qv.z), sc * hi_bf(qv.z)),
                                     pack_bf16(sc * lo_bf(qv.w), sc * hi_bf(qv.w)));
                    }
                }

                // -------- S4 epilogue: W = W' diag(e^Ga), published as -W^T over the dead fp32 T
                // (so that the next chunk may overwrite Kh at once)
                wait_bar(BAR(PB_WAV_DONE), kk & 1, abort_flag);
                tc_fence_after();
                if (t == 0) KDA_TRACE_POINT(m, 5);
                {
                    uint32_t a[32];
                    tmem_ld32(tmem + lane_base + COL_W + half * 32, a);
                    tmem_wait_ld();
                    const float sc = -ega_s[lrow];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int jj = half * 4 + j;
                        st_shared_v4(sbase + PR_T + sw128(lrow, jj),
                                     pack_bf16(sc * __uint_as_float(a[8 * j]), sc * __uint_as_float(a[8 * j + 1])),
                                     pack_bf16(sc * __uint_as_float(a[8 * j + 2]), sc * __uint_as_float(a[8 * j + 3])),
                                     pack_bf16(sc * __uint_as_float(a[8 * j + 4]), sc * __uint_as_float(a[8 * j + 5])),
                                     pack_bf16(sc * __uint_as_float(a[8 * j + 6]), sc * __uint_as_float(a[8 * j + 7])));
                    }
                }
                // hand the finished set to the publisher
                fence_proxy_async_smem();
                tc_fence_before();
                if (named_bar_any(2, 256, *abort_flag != 0)) break;
                if (t == 0) {
                    mbar_arrive(BAR(PB_OUTB_READY));
                    KDA_TRACE_POINT(m, 6);
                }
            }
        }
    }

    if (is_chain && tid == 128) {
        KDA_TRACE_CLUSTER(1, globaltimer());
        KDA_TRACE_CLUSTER(6, static_cast<unsigned long long>(clock64()));
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

// Per-device ring pool of the operand-set exchange, allocated on first use and held
// until the library is unloaded (or the process exits).
std::mutex g_pool_mu;
unsigned char *g_pool[64] = {};
bool g_exiting = false;
void note_exit() { g_exiting = true; }

unsigned char *ring_pool(int dev) {
    if (dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lk(g_pool_mu);
    if (g_pool[dev]) {
        // a device reset since the allocation frees the pool: allocate it again
        cudaPointerAttributes at;
        if (cudaPointerGetAttributes(&at, g_pool[dev]) != cudaSuccess || at.type != cudaMemoryTypeDevice) {
            (void)cudaGetLastError();
            g_pool[dev] = nullptr;
        }
    }
    if (!g_pool[dev]) {
        void *ptr = nullptr;
        if (cudaMalloc(&ptr, static_cast<size_t>(tc::kMaxRings) * tc::RING_BYTES) != cudaSuccess) return nullptr;
        g_pool[dev] = static_cast<unsigned char *>(ptr);
        static std::once_flag once;
        std::call_once(once, [] { std::atexit(note_exit); });
    }
    return g_pool[dev];
}

// Release the pools when the library is unloaded before the process exits. At exit
// nothing is called: the CUDA runtime may already be torn down, and the driver reclaims
// the memory with the process.
__attribute__((destructor)) void release_ring_pools() {
    if (g_exiting) return;
    int cur = -1;
    if (cudaGetDevice(&cur) != cudaSuccess) return;
    for (int dev = 0; dev < 64; ++dev) {
        if (!g_pool[dev]) continue;
        if (cudaSetDevice(dev) == cudaSuccess) (void)cudaFree(g_pool[dev]);
        g_pool[dev] = nullptr;
    }
    (void)cudaSetDevice(cur);
    (void)cudaGetLastError();
}

// Scratch of the allocation-free entry point: one operand-set ring per cluster for at
// most kNoAllocMaxUnits clusters (15.4 MiB). It is part of the module image, so it
// exists as soon as the module is loaded and nothing is allocated when it is used.
// Nothing in it has to start at zero: a prep CTA writes every ring slot before it
// signals the chain CTA to read it.
static __device__ __align__(256) unsigned char g_noalloc_rings[kNoAllocMaxUnits * tc::RING_BYTES];

std::mutex g_noalloc_mu;
unsigned char *g_noalloc_addr[64] = {};

// Device address of g_noalloc_rings on `dev` (the current device), looked up once.
cudaError_t noalloc_scratch(int dev, unsigned char **out) {
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_addr[dev]) {
        void *ptr = nullptr;
        const cudaError_t err = cudaGetSymbolAddress(&ptr, g_noalloc_rings);
        if (err != cudaSuccess) return err;
        g_noalloc_addr[dev] = static_cast<unsigned char *>(ptr);
    }
    *out = g_noalloc_addr[dev];
    return cudaSuccess;
}

// Encode the tensor maps and launch one 4-CTA cluster per (sequence, head).
template <bool kRingPerCluster, int kGate, bool kNorm, bool kSeg = false>
cudaError_t launch_clusters(const FwdParams &p, int64_t rows, int64_t grid, unsigned char *rings,
                            cudaStream_t stream) {
    tc::TmaMaps maps;
    memset(&maps, 0, sizeof(maps));
    if (rows > 0) {
        if (rows > 0x7fffffffLL) return cudaErrorInvalidValue;
        if (!encode3d(&maps.q, p.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.num_heads, rows, 128,
                      CU_TENSOR_MAP_SWIZZLE_NONE) ||
            !encode3d(&maps.k, p.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.num_heads, rows, 128,
                      CU_TENSOR_MAP_SWIZZLE_NONE) ||
            (kGate == kGateF32 && !encode3d(&maps.g, p.g, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, p.num_heads,
                                            rows, 128, CU_TENSOR_MAP_SWIZZLE_NONE)) ||
            (kGate == kGateBF16 && !encode3d(&maps.g, p.g, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.num_heads,
                                             rows, 128, CU_TENSOR_MAP_SWIZZLE_NONE)) ||
            !encode3d(&maps.v, p.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.num_heads, rows, 64,
                      CU_TENSOR_MAP_SWIZZLE_128B) ||
            !encode3d(&maps.o, p.out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.num_heads, rows, 64,
                      CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
    }
    cudaError_t err = cudaFuncSetAttribute(tc::kda_fwd_tc_kernel<kRingPerCluster, kGate, kNorm, kSeg>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
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
    err = cudaLaunchKernelEx(&cfg, tc::kda_fwd_tc_kernel<kRingPerCluster, kGate, kNorm, kSeg>, p, maps, rings);
    if (err != cudaSuccess) return err;
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_tc(const FwdParams &p, int64_t rows, cudaStream_t stream) {
    const int64_t units = static_cast<int64_t>(p.num_seqs) * p.num_heads * (p.mode == kModeAffine ? 2 : 1);
    if (units == 0) return cudaSuccess;
    const int64_t grid = units * tc::NS;
    if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    unsigned char *rings = ring_pool(dev);
    if (!rings) return cudaErrorMemoryAllocation;
    const bool norm = (p.flags & kFlagL2NormQK) != 0;
    if (p.seg_len > 0 || p.mode != kModePlain) {
        // the segmented forward takes the plain gate only
        if (p.gate_mode != kGateF32 || p.flags != 0) return cudaErrorInvalidValue;
        return launch_clusters<false, kGateF32, false, true>(p, rows, grid, rings, stream);
    }
    switch (p.gate_mode) {
        case kGateF32:
            return norm ? launch_clusters<false, kGateF32, true>(p, rows, grid, rings, stream)
                        : launch_clusters<false, kGateF32, false>(p, rows, grid, rings, stream);
        case kGateBF16:
            return norm ? launch_clusters<false, kGateBF16, true>(p, rows, grid, rings, stream)
                        : launch_clusters<false, kGateBF16, false>(p, rows, grid, rings, stream);
        case kGateScalar:
            return norm ? launch_clusters<false, kGateScalar, true>(p, rows, grid, rings, stream)
                        : launch_clusters<false, kGateScalar, false>(p, rows, grid, rings, stream);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_fwd_tc_noalloc(const FwdParams &p, int64_t rows, cudaStream_t stream) {
    const int64_t units = static_cast<int64_t>(p.num_seqs) * p.num_heads;
    if (units == 0) return cudaSuccess;
    if (units > kNoAllocMaxUnits) return cudaErrorInvalidValue;
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    unsigned char *rings = nullptr;
    err = noalloc_scratch(dev, &rings);
    if (err != cudaSuccess) return err;
    if (p.gate_mode != kGateF32 || p.flags != 0) return cudaErrorInvalidValue;
    return launch_clusters<true, kGateF32, false>(p, rows, units * tc::NS, rings, stream);
}

#ifdef KDA_TEST_HOOKS
extern "C" int kda_test_set_skip_chunk(int chunk) {
    return static_cast<int>(cudaMemcpyToSymbol(g_kda_test_skip_chunk, &chunk, sizeof(int)));
}
#endif

#ifdef KDA_TRACE
extern "C" int kda_trace_read(unsigned long long *host) {
    return static_cast<int>(cudaMemcpyFromSymbol(host, g_kda_trace, sizeof(g_kda_trace)));
}
extern "C" int kda_trace_read_clusters(unsigned long long *host) {
    return static_cast<int>(cudaMemcpyFromSymbol(host, g_kda_cluster_trace, sizeof(g_kda_cluster_trace)));
}
#endif

cudaError_t read_and_clear_device_error(unsigned int *value) {
    cudaError_t err = cudaMemcpyFromSymbol(value, g_kda_device_error, sizeof(unsigned int));
    if (err != cudaSuccess) return err;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_kda_device_error, &zero, sizeof(unsigned int));
}

}  // namespace kda
