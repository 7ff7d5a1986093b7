// kda_api.cu -- C-ABI front end: argument validation and kernel dispatch.
#include <cuda_runtime.h>

#include "../../include/kda.h"
#include "kda_internal.h"
#include "kda_decode.h"

static_assert(kda::kNoAllocMaxUnits == KDA_NOALLOC_MAX_UNITS, "scratch limit of kda_fwd_noalloc");

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool device_is_sm100(int *err) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) { *err = 1; return false; }
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
        *err = 1;
        return false;
    }
    *err = 0;
    return major == 10;
}

// Validate the arguments of kda_fwd / kda_fwd_noalloc and fill the kernel parameters.
// Returns KDA_OK with p->num_seqs == 0 when there is nothing to do.
kda_status prepare(const void *q, const void *k, const void *v, const void *g, const float *beta, float scale,
                   const int32_t *cu_seqlens, int32_t num_seqs, int32_t batch, int64_t seq_len,
                   int32_t num_heads, int32_t head_dim_k, int32_t head_dim_v, const void *initial_state,
                   kda_dtype initial_dtype, void *final_state, kda_dtype final_dtype, void *out,
                   bool noalloc, int32_t gate_kind, uint32_t flags, kda::FwdParams *p, int64_t *rows_out) {
    p->num_seqs = 0;
    if (gate_kind != KDA_GATE_FP32 && gate_kind != KDA_GATE_BF16 && gate_kind != KDA_GATE_SCALAR_FP32)
        return KDA_ERR_BAD_OPTION;
    if (flags & ~static_cast<uint32_t>(KDA_FLAG_L2NORM_QK | KDA_FLAG_GATE_LOGSIGMOID)) return KDA_ERR_BAD_OPTION;
    if (head_dim_k != kda::kHeadDim || head_dim_v != kda::kHeadDim) return KDA_ERR_BAD_SHAPE;
    if (batch < 0 || seq_len < 0 || num_heads < 1 || num_seqs < 0) return KDA_ERR_BAD_SHAPE;
    if (cu_seqlens && batch != 1) return KDA_ERR_VARLEN_BATCH;
    if (initial_state && initial_dtype != KDA_DTYPE_BF16 && initial_dtype != KDA_DTYPE_FP32)
        return KDA_ERR_STATE_DTYPE;
    if (final_state && final_dtype != KDA_DTYPE_BF16 && final_dtype != KDA_DTYPE_FP32)
        return KDA_ERR_STATE_DTYPE;
    if (initial_state && final_state && initial_dtype != final_dtype) return KDA_ERR_STATE_DTYPE;
    const int64_t n_seqs = cu_seqlens ? num_seqs : batch;
    const int64_t rows = cu_seqlens ? seq_len : static_cast<int64_t>(batch) * seq_len;
    if (rows > 0 && (!q || !k || !v || !g || !beta || !out)) return KDA_ERR_NULL_PTR;
    if (cu_seqlens && !(reinterpret_cast<uintptr_t>(cu_seqlens) % 4 == 0)) return KDA_ERR_BAD_ALIGNMENT;
    const bool g_ok = gate_kind == KDA_GATE_SCALAR_FP32 ? (reinterpret_cast<uintptr_t>(g) & 3u) == 0 : aligned16(g);
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !g_ok || !aligned16(out) ||
        !aligned16(initial_state) || !aligned16(final_state) ||
        (reinterpret_cast<uintptr_t>(beta) & 3u))
        return KDA_ERR_BAD_ALIGNMENT;
    // token offsets are formed as (row * H + h) * 128 in 64-bit; keep the product well inside
    if (rows > (int64_t(1) << 40) / (int64_t(num_heads) * kda::kHeadDim)) return KDA_ERR_TOO_LARGE;
    if (n_seqs * num_heads > (int64_t(1) << 29)) return KDA_ERR_TOO_LARGE;
    if (noalloc && n_seqs * num_heads > kda::kNoAllocMaxUnits) return KDA_ERR_NOALLOC_LIMIT;
    if (n_seqs == 0) return KDA_OK;

    int qerr = 0;
    if (!device_is_sm100(&qerr)) return qerr ? KDA_ERR_CUDA : KDA_ERR_UNSUPPORTED_DEVICE;

    p->q = static_cast<const uint16_t *>(q);
    p->k = static_cast<const uint16_t *>(k);
    p->v = static_cast<const uint16_t *>(v);
    p->g = g;
    p->beta = beta;
    p->scale = scale;
    p->cu_seqlens = cu_seqlens;
    p->seq_len = seq_len;
    p->num_seqs = static_cast<int32_t>(n_seqs);
    p->num_heads = num_heads;
    p->h0 = initial_state;
    p->h0_fp32 = initial_dtype == KDA_DTYPE_FP32;
    p->hT = final_state;
    p->hT_fp32 = final_dtype == KDA_DTYPE_FP32;
    p->out = static_cast<uint16_t *>(out);
    p->gate_mode = gate_kind;
    p->flags = flags;
    p->seg_len = 0;
    p->seg_count = 0;
    p->mode = kda::kModePlain;
    p->hT_aux = nullptr;
    *rows_out = rows;
    return KDA_OK;
}

}  // namespace

extern "C" {

const char *kda_status_string(kda_status s) {
    switch (s) {
        case KDA_OK: return "KDA_OK";
        case KDA_ERR_NULL_PTR: return "KDA_ERR_NULL_PTR: a required pointer is NULL";
        case KDA_ERR_BAD_SHAPE: return "KDA_ERR_BAD_SHAPE: head dims must be 128 and sizes non-negative";
        case KDA_ERR_VARLEN_BATCH: return "KDA_ERR_VARLEN_BATCH: cu_seqlens requires batch == 1";
        case KDA_ERR_STATE_DTYPE: return "KDA_ERR_STATE_DTYPE: states must be bf16 or fp32 and match";
        case KDA_ERR_CUDA: return "KDA_ERR_CUDA: a CUDA call failed";
        case KDA_ERR_UNSUPPORTED_DEVICE: return "KDA_ERR_UNSUPPORTED_DEVICE: needs an sm_100 (B200) device";
        case KDA_ERR_BAD_ALIGNMENT: return "KDA_ERR_BAD_ALIGNMENT: tensor pointers must be 16-byte aligned";
        case KDA_ERR_TOO_LARGE: return "KDA_ERR_TOO_LARGE: sizes exceed the library's index range";
        case KDA_ERR_TIMEOUT: return "KDA_ERR_TIMEOUT: a kernel gave up waiting on a barrier and stopped";
        case KDA_ERR_NOALLOC_LIMIT:
            return "KDA_ERR_NOALLOC_LIMIT: kda_fwd_noalloc takes at most 32 (sequence, head) pairs per call";
        case KDA_ERR_STATE_OVERLAP:
            return "KDA_ERR_STATE_OVERLAP: kda_decode state_in and state_out overlap without being the same buffer";
        case KDA_ERR_BAD_CU_SEQLENS:
            return "KDA_ERR_BAD_CU_SEQLENS: cu_seqlens must run 0, ..., seq_len without decreasing";
        case KDA_ERR_INTERNAL:
            return "KDA_ERR_INTERNAL: a kernel ran on an SM beyond its scratch pool and stopped";
        case KDA_ERR_BAD_OPTION:
            return "KDA_ERR_BAD_OPTION: unknown gate kind or flag";
        case KDA_ERR_WORKSPACE:
            return "KDA_ERR_WORKSPACE: the workspace is smaller than kda_fwd_segmented_workspace() asks";
    }
    return "KDA_ERR_UNKNOWN";
}

int32_t kda_version(void) { return (1 << 16) | 3; }

kda_status kda_fwd(const void *q, const void *k, const void *v, const float *g,
                   const float *beta, float scale, const int32_t *cu_seqlens,
                   int32_t num_seqs, int32_t batch, int64_t seq_len, int32_t num_heads,
                   int32_t head_dim_k, int32_t head_dim_v, const void *initial_state,
                   kda_dtype initial_dtype, void *final_state, kda_dtype final_dtype,
                   void *out, kda_stream_t stream) {
    kda::FwdParams p;
    int64_t rows = 0;
    const kda_status st = prepare(q, k, v, g, beta, scale, cu_seqlens, num_seqs, batch, seq_len, num_heads,
                                  head_dim_k, head_dim_v, initial_state, initial_dtype, final_state,
                                  final_dtype, out, false, KDA_GATE_FP32, 0u, &p, &rows);
    if (st != KDA_OK || p.num_seqs == 0) return st;
    const cudaError_t err = kda::launch_fwd_tc(p, rows, reinterpret_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status kda_fwd_ex(const void *q, const void *k, const void *v, const void *g, int32_t gate_kind,
                      const float *beta, float scale, const int32_t *cu_seqlens, int32_t num_seqs,
                      int32_t batch, int64_t seq_len, int32_t num_heads, int32_t head_dim_k,
                      int32_t head_dim_v, const void *initial_state, kda_dtype initial_dtype,
                      void *final_state, kda_dtype final_dtype, void *out, uint32_t flags,
                      kda_stream_t stream) {
    kda::FwdParams p;
    int64_t rows = 0;
    const kda_status st = prepare(q, k, v, g, beta, scale, cu_seqlens, num_seqs, batch, seq_len, num_heads,
                                  head_dim_k, head_dim_v, initial_state, initial_dtype, final_state,
                                  final_dtype, out, false, gate_kind, flags, &p, &rows);
    if (st != KDA_OK || p.num_seqs == 0) return st;
    const cudaError_t err = kda::launch_fwd_tc(p, rows, reinterpret_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

size_t kda_fwd_segmented_workspace(int32_t batch, int64_t seq_len, int32_t num_heads, int64_t segment_len) {
    if (batch < 0 || seq_len < 0 || num_heads < 1 || segment_len < kda::kChunk || segment_len % kda::kChunk)
        return 0;
    const int64_t pieces = (seq_len + segment_len - 1) / segment_len;
    return static_cast<size_t>(3) * static_cast<size_t>(batch) * static_cast<size_t>(pieces) *
           static_cast<size_t>(num_heads) * kda::kHeadDim * kda::kHeadDim * sizeof(float);
}

kda_status kda_fwd_segmented(const void *q, const void *k, const void *v, const float *g,
                             const float *beta, float scale, int32_t batch, int64_t seq_len,
                             int32_t num_heads, int32_t head_dim_k, int32_t head_dim_v,
                             const void *initial_state, kda_dtype initial_dtype, void *final_state,
                             kda_dtype final_dtype, void *out, int64_t segment_len, void *workspace,
                             size_t workspace_bytes, kda_stream_t stream) {
    if (segment_len < kda::kChunk || segment_len % kda::kChunk) return KDA_ERR_BAD_SHAPE;
    kda::FwdParams p;
    int64_t rows = 0;
    kda_status st = prepare(q, k, v, g, beta, scale, nullptr, 0, batch, seq_len, num_heads, head_dim_k,
                            head_dim_v, initial_state, initial_dtype, final_state, final_dtype, out, false,
                            KDA_GATE_FP32, 0u, &p, &rows);
    if (st != KDA_OK || p.num_seqs == 0) return st;
    const int64_t pieces = (seq_len + segment_len - 1) / segment_len;
    if (pieces <= 1) {
        const cudaError_t err = kda::launch_fwd_tc(p, rows, reinterpret_cast<cudaStream_t>(stream));
        return err == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
    }
    const int64_t units = static_cast<int64_t>(batch) * pieces;
    if (units * num_heads > (int64_t(1) << 28) || units > 0x7fffffffLL) return KDA_ERR_TOO_LARGE;
    const size_t need = kda_fwd_segmented_workspace(batch, seq_len, num_heads, segment_len);
    if (!workspace) return KDA_ERR_NULL_PTR;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return KDA_ERR_BAD_ALIGNMENT;
    if (workspace_bytes < need) return KDA_ERR_WORKSPACE;
    const size_t per = need / 3 / sizeof(float);
    float *Mb = static_cast<float *>(workspace), *Bb = Mb + per, *Sin = Bb + per;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // 1. every piece's affine map: B from a zero state, M from the identity with v = 0
    kda::FwdParams pa = p;
    pa.num_seqs = static_cast<int32_t>(units);
    pa.seg_len = segment_len;
    pa.seg_count = static_cast<int32_t>(pieces);
    pa.mode = kda::kModeAffine;
    pa.h0 = nullptr;
    pa.hT = Bb;
    pa.hT_fp32 = 1;
    pa.hT_aux = Mb;
    cudaError_t err = kda::launch_fwd_tc(pa, rows, s);
    // 2. the states entering the pieces
    if (err == cudaSuccess)
        err = kda::launch_segment_scan(initial_state, initial_dtype == KDA_DTYPE_FP32, Mb, Bb, Sin, batch,
                                       static_cast<int32_t>(pieces), num_heads, s);
    // 3. every piece from its entering state: the outputs, and each row's final state
    if (err == cudaSuccess) {
        kda::FwdParams pp = pa;
        pp.mode = kda::kModePlain;
        pp.h0 = Sin;
        pp.h0_fp32 = 1;
        pp.hT = final_state;
        pp.hT_fp32 = final_dtype == KDA_DTYPE_FP32;
        pp.hT_aux = nullptr;
        err = kda::launch_fwd_tc(pp, rows, s);
    }
    return err == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

size_t kda_bwd_workspace(int64_t total_tokens, int32_t num_seqs, int32_t num_heads) {
    if (total_tokens < 0 || num_seqs < 0 || num_heads < 1) return 0;
    return kda::bwd_workspace_bytes(total_tokens, num_seqs, num_heads);
}

kda_status kda_bwd(const void *q, const void *k, const void *v, const float *g, const float *beta, float scale,
                   const int32_t *cu_seqlens, int32_t num_seqs, int32_t batch, int64_t seq_len, int32_t num_heads,
                   int32_t head_dim_k, int32_t head_dim_v, const void *initial_state, kda_dtype initial_dtype,
                   const void *dout, const float *dfinal_state, float *dq, float *dk, float *dv, float *dg,
                   float *dbeta, float *dinitial_state, void *workspace, size_t workspace_bytes,
                   kda_stream_t stream) {
    // the forward's argument rules (no final state here; dinitial_state takes its place)
    kda::FwdParams fp;
    int64_t rows = 0;
    kda_status st = prepare(q, k, v, g, beta, scale, cu_seqlens, num_seqs, batch, seq_len, num_heads, head_dim_k,
                            head_dim_v, initial_state, initial_dtype, nullptr, KDA_DTYPE_NONE, dq, false,
                            KDA_GATE_FP32, 0u, &fp, &rows);
    if (st != KDA_OK) return st;
    if (rows > 0 && (!dout || !dk || !dv || !dg || !dbeta)) return KDA_ERR_NULL_PTR;
    if (!aligned16(dout) || !aligned16(dk) || !aligned16(dv) || !aligned16(dg) || !aligned16(dfinal_state) ||
        !aligned16(dinitial_state) || (reinterpret_cast<uintptr_t>(dbeta) & 3u))
        return KDA_ERR_BAD_ALIGNMENT;
    if (fp.num_seqs == 0) return KDA_OK;
    const size_t need = kda::bwd_workspace_bytes(rows, fp.num_seqs, num_heads);
    if (!workspace) return KDA_ERR_NULL_PTR;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return KDA_ERR_BAD_ALIGNMENT;
    if (workspace_bytes < need) return KDA_ERR_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // dq, dk, dg and dbeta gather the value-column slices' shares; dv too is cleared, for tokens
    // that no sequence covers
    const size_t elems = static_cast<size_t>(rows) * num_heads * kda::kHeadDim;
    cudaError_t err = cudaSuccess;
    if (rows > 0) {
        if (err == cudaSuccess) err = cudaMemsetAsync(dq, 0, elems * sizeof(float), s);
        if (err == cudaSuccess) err = cudaMemsetAsync(dk, 0, elems * sizeof(float), s);
        if (err == cudaSuccess) err = cudaMemsetAsync(dv, 0, elems * sizeof(float), s);
        if (err == cudaSuccess) err = cudaMemsetAsync(dg, 0, elems * sizeof(float), s);
        if (err == cudaSuccess)
            err = cudaMemsetAsync(dbeta, 0, static_cast<size_t>(rows) * num_heads * sizeof(float), s);
    }
    if (err != cudaSuccess) return KDA_ERR_CUDA;
    kda::BwdParams p;
    p.q = fp.q;
    p.k = fp.k;
    p.v = fp.v;
    p.g = static_cast<const float *>(fp.g);
    p.beta = fp.beta;
    p.scale = scale;
    p.cu_seqlens = cu_seqlens;
    p.seq_len = seq_len;
    p.num_seqs = fp.num_seqs;
    p.num_heads = num_heads;
    p.h0 = initial_state;
    p.h0_fp32 = initial_dtype == KDA_DTYPE_FP32;
    p.dout = static_cast<const uint16_t *>(dout);
    p.dhT = dfinal_state;
    p.dq = dq;
    p.dk = dk;
    p.dv = dv;
    p.dg = dg;
    p.dbeta = dbeta;
    p.dh0 = dinitial_state;
    p.workspace = static_cast<float *>(workspace);
    err = kda::launch_bwd(p, s);
    return err == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status kda_fwd_noalloc(const void *q, const void *k, const void *v, const float *g,
                           const float *beta, float scale, const int32_t *cu_seqlens,
                           int32_t num_seqs, int32_t batch, int64_t seq_len, int32_t num_heads,
                           int32_t head_dim_k, int32_t head_dim_v, const void *initial_state,
                           kda_dtype initial_dtype, void *final_state, kda_dtype final_dtype,
                           void *out, kda_stream_t stream) {
    kda::FwdParams p;
    int64_t rows = 0;
    const kda_status st = prepare(q, k, v, g, beta, scale, cu_seqlens, num_seqs, batch, seq_len, num_heads,
                                  head_dim_k, head_dim_v, initial_state, initial_dtype, final_state,
                                  final_dtype, out, true, KDA_GATE_FP32, 0u, &p, &rows);
    if (st != KDA_OK || p.num_seqs == 0) return st;
    const cudaError_t err = kda::launch_fwd_tc_noalloc(p, rows, reinterpret_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status kda_decode(const void *q, const void *k, const void *v, const float *g,
                      const float *beta, float scale, int32_t batch, int32_t num_heads,
                      int32_t head_dim_k, int32_t head_dim_v, const void *state_in,
                      void *state_out, kda_dtype state_dtype, void *out, kda_stream_t stream) {
    if (head_dim_k != kda::kHeadDim || head_dim_v != kda::kHeadDim) return KDA_ERR_BAD_SHAPE;
    if (batch < 0 || num_heads < 1) return KDA_ERR_BAD_SHAPE;
    if ((state_in || state_out) && state_dtype != KDA_DTYPE_BF16 && state_dtype != KDA_DTYPE_FP32)
        return KDA_ERR_STATE_DTYPE;
    const int64_t units = static_cast<int64_t>(batch) * num_heads;
    if (units > 0 && (!q || !k || !v || !g || !beta || !out)) return KDA_ERR_NULL_PTR;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(g) || !aligned16(out) ||
        !aligned16(state_in) || !aligned16(state_out) || (reinterpret_cast<uintptr_t>(beta) & 3u))
        return KDA_ERR_BAD_ALIGNMENT;
    if (units > 0x7fffffffLL) return KDA_ERR_TOO_LARGE;
    if (state_in && state_out && state_in != state_out) {
        // distinct state buffers must not overlap
        const uintptr_t a = reinterpret_cast<uintptr_t>(state_in), b = reinterpret_cast<uintptr_t>(state_out);
        const uintptr_t bytes = static_cast<uintptr_t>(units) * kda::kHeadDim * kda::kHeadDim *
                                (state_dtype == KDA_DTYPE_FP32 ? 4u : 2u);
        if (a < b + bytes && b < a + bytes) return KDA_ERR_STATE_OVERLAP;
    }
    if (units == 0) return KDA_OK;
    int qerr = 0;
    if (!device_is_sm100(&qerr)) return qerr ? KDA_ERR_CUDA : KDA_ERR_UNSUPPORTED_DEVICE;
    kda::DecodeParams p;
    p.q = static_cast<const uint16_t *>(q);
    p.k = static_cast<const uint16_t *>(k);
    p.v = static_cast<const uint16_t *>(v);
    p.g = g;
    p.beta = beta;
    p.scale = scale;
    p.state_in = state_in;
    p.state_out = state_out;
    p.state_fp32 = state_dtype == KDA_DTYPE_FP32;
    p.out = static_cast<uint16_t *>(out);
    const cudaError_t err = kda::launch_decode(p, units, reinterpret_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status kda_device_error(void) {
    if (cudaDeviceSynchronize() != cudaSuccess) return KDA_ERR_CUDA;
    unsigned int v = 0;
    if (kda::read_and_clear_device_error(&v) != cudaSuccess) return KDA_ERR_CUDA;
    if (v & kda::kErrCuSeqlens) return KDA_ERR_BAD_CU_SEQLENS;
    if (v & kda::kErrTimeout) return KDA_ERR_TIMEOUT;
    if (v & kda::kErrRingIndex) return KDA_ERR_INTERNAL;
    return KDA_OK;
}

}  // extern "C"
