// fa_api.cu -- the C ABI (include/fa.h): argument checks, launch set-up,
// status strings and the device error word.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "../../include/fa.h"
#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {

int device_sm_count() {
    static std::atomic<int> cached[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 1;
    if (dev >= 0 && dev < 64) {
        int v = cached[dev].load(std::memory_order_relaxed);
        if (v > 0) return v;
    }
    int n = 1;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n < 1) n = 1;
    if (dev >= 0 && dev < 64) cached[dev].store(n, std::memory_order_relaxed);
    return n;
}

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

int encode_tensor_map_3d(void *map, const void *base, int elem_bytes, uint64_t dim0,
                         uint64_t dim1, uint64_t dim2, uint64_t stride1_bytes,
                         uint64_t stride2_bytes, uint32_t box0, uint32_t box1, uint32_t box2,
                         int swizzle_bytes) {
    auto fn = encode_fn();
    if (!fn) return -1;
    CUtensorMapDataType dt;
    switch (elem_bytes) {
    case 1: dt = CU_TENSOR_MAP_DATA_TYPE_UINT8; break;
    case 2: dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16; break;
    case 4: dt = CU_TENSOR_MAP_DATA_TYPE_FLOAT32; break;
    default: return -1;
    }
    CUtensorMapSwizzle sw;
    switch (swizzle_bytes) {
    case 0: sw = CU_TENSOR_MAP_SWIZZLE_NONE; break;
    case 32: sw = CU_TENSOR_MAP_SWIZZLE_32B; break;
    case 64: sw = CU_TENSOR_MAP_SWIZZLE_64B; break;
    case 128: sw = CU_TENSOR_MAP_SWIZZLE_128B; break;
    default: return -1;
    }
    cuuint64_t dims[3] = {dim0, dim1, dim2};
    cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
    cuuint32_t box[3] = {box0, box1, box2};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(static_cast<CUtensorMap *>(map), dt, 3,
                    const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE,
                    sw,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? 0 : -1;
}

// Diagnostic kernel for the watchdog: waits on a barrier that nothing ever
// arrives on.  The bounded wait gives up after ~1 s, records the timeout in
// the device error word and the kernel returns normally.
__global__ void watchdog_probe_kernel() {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag);
}

}  // namespace fa

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

int map_rc(int rc) {
    switch (rc) {
    case 0: return FA_OK;
    case -2: return FA_ERR_UNSUPPORTED;
    case -4: return FA_ERR_WORKSPACE;
    default: return FA_ERR_CUDA;
    }
}

int check_common(int Hq, int Hkv, int d, int causal, int window, float scale, int o_dtype) {
    if (Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
    if (!(scale > 0.f) || !std::isfinite(scale)) return FA_ERR_INVALID_ARG;
    if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
    if (o_dtype != FA_OUT_BF16 && o_dtype != FA_OUT_FP32) return FA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
    if (window > 0 && !causal) return FA_ERR_UNSUPPORTED;
    return FA_OK;
}

}  // namespace

extern "C" {

}  // extern "C"

namespace {

int fwd_dense(const void *q, const void *k, const void *v, void *o, float *lse,
              const float *sinks, int B, int Hq, int Hkv, int N, int d, int causal, int window,
              float scale, int o_dtype, void *stream, const int *doc = nullptr,
              int n_sink = 0) {
    if (B < 0 || N < 0) return FA_ERR_INVALID_ARG;
    int rc = check_common(Hq, Hkv, d, causal, window, scale, o_dtype);
    if (rc) return rc;
    if (B == 0 || N == 0) return FA_OK;
    if (!q || !k || !v || !o) return FA_ERR_INVALID_ARG;
    if ((long long)B * N > INT32_MAX / 2) return FA_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
        (lse && (reinterpret_cast<uintptr_t>(lse) & 3)))
        return FA_ERR_ALIGNMENT;
    fa::PrefillArgs a{};
    a.q = q; a.k = k; a.v = v; a.o = o; a.lse = lse;
    a.cu_seqlens = nullptr;
    a.num_seqs = B;
    a.seqlen = N;
    a.total_tokens = B * N;
    a.max_seqlen = N;
    a.Hq = Hq; a.Hkv = Hkv; a.d = d;
    a.causal = causal;
    a.window = window > 0 ? window : 0;
    a.scale = scale;
    a.o_fp32 = o_dtype == FA_OUT_FP32;
    a.sinks = sinks;
    a.doc = doc;
    a.n_sink = n_sink;
    return map_rc(fa::launch_prefill(a, static_cast<cudaStream_t>(stream)));
}

int fwd_varlen(const void *q, const void *k, const void *v, void *o, float *lse,
               const float *sinks, const int *cu_seqlens, int num_seqs, int total_tokens,
               int max_seqlen, int Hq, int Hkv, int d, int causal, int window, float scale,
               int o_dtype, void *stream, int n_sink = 0) {
    if (num_seqs < 0 || total_tokens < 0 || max_seqlen < 0) return FA_ERR_INVALID_ARG;
    int rc = check_common(Hq, Hkv, d, causal, window, scale, o_dtype);
    if (rc) return rc;
    if (num_seqs == 0 || total_tokens == 0 || max_seqlen == 0) return FA_OK;
    if (!q || !k || !v || !o || !cu_seqlens) return FA_ERR_INVALID_ARG;
    if (total_tokens > INT32_MAX / 2) return FA_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
        (reinterpret_cast<uintptr_t>(cu_seqlens) & 3) ||
        (lse && (reinterpret_cast<uintptr_t>(lse) & 3)))
        return FA_ERR_ALIGNMENT;
    fa::PrefillArgs a{};
    a.q = q; a.k = k; a.v = v; a.o = o; a.lse = lse;
    a.cu_seqlens = cu_seqlens;
    a.num_seqs = num_seqs;
    a.seqlen = 0;
    a.total_tokens = total_tokens;
    a.max_seqlen = max_seqlen;
    a.Hq = Hq; a.Hkv = Hkv; a.d = d;
    a.causal = causal;
    a.window = window > 0 ? window : 0;
    a.scale = scale;
    a.o_fp32 = o_dtype == FA_OUT_FP32;
    a.sinks = sinks;
    a.n_sink = n_sink;
    return map_rc(fa::launch_prefill(a, static_cast<cudaStream_t>(stream)));
}

}  // namespace

extern "C" {

int fa_fwd(const void *q, const void *k, const void *v, void *o, float *lse, int B, int Hq,
           int Hkv, int N, int d, int causal, int window, float scale, int o_dtype,
           void *stream) {
    return fwd_dense(q, k, v, o, lse, nullptr, B, Hq, Hkv, N, d, causal, window, scale,
                     o_dtype, stream);
}

int fa_fwd_sink_tokens(const void *q, const void *k, const void *v, void *o, float *lse,
                       int B, int Hq, int Hkv, int N, int d, int window, int n_sink,
                       float scale, int o_dtype, void *stream) {
    if (window <= 0 || n_sink < 0) return FA_ERR_INVALID_ARG;
    return fwd_dense(q, k, v, o, lse, nullptr, B, Hq, Hkv, N, d, 1, window, scale, o_dtype,
                     stream, nullptr, n_sink);
}

int fa_fwd_varlen_sink_tokens(const void *q, const void *k, const void *v, void *o, float *lse,
                              const int *cu_seqlens, int num_seqs, int total_tokens,
                              int max_seqlen, int Hq, int Hkv, int d, int window, int n_sink,
                              float scale, int o_dtype, void *stream) {
    if (window <= 0 || n_sink < 0) return FA_ERR_INVALID_ARG;
    return fwd_varlen(q, k, v, o, lse, nullptr, cu_seqlens, num_seqs, total_tokens, max_seqlen,
                      Hq, Hkv, d, 1, window, scale, o_dtype, stream, n_sink);
}

int fa_fwd_sinks(const void *q, const void *k, const void *v, void *o, float *lse,
                 const float *sinks, int B, int Hq, int Hkv, int N, int d, int causal,
                 int window, float scale, int o_dtype, void *stream) {
    if (!sinks) return FA_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(sinks) & 3) return FA_ERR_ALIGNMENT;
    return fwd_dense(q, k, v, o, lse, sinks, B, Hq, Hkv, N, d, causal, window, scale,
                     o_dtype, stream);
}

int fa_fwd_doc(const void *q, const void *k, const void *v, void *o, float *lse,
               const int *doc_ids, int B, int Hq, int Hkv, int N, int d, int causal,
               int window, float scale, int o_dtype, void *stream) {
    if (!doc_ids) return FA_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(doc_ids) & 3) return FA_ERR_ALIGNMENT;
    return fwd_dense(q, k, v, o, lse, nullptr, B, Hq, Hkv, N, d, causal, window, scale,
                     o_dtype, stream, doc_ids);
}

int fa_fwd_varlen(const void *q, const void *k, const void *v, void *o, float *lse,
                  const int *cu_seqlens, int num_seqs, int total_tokens, int max_seqlen,
                  int Hq, int Hkv, int d, int causal, int window, float scale, int o_dtype,
                  void *stream) {
    return fwd_varlen(q, k, v, o, lse, nullptr, cu_seqlens, num_seqs, total_tokens,
                      max_seqlen, Hq, Hkv, d, causal, window, scale, o_dtype, stream);
}

int fa_fwd_varlen_sinks(const void *q, const void *k, const void *v, void *o, float *lse,
                        const float *sinks, const int *cu_seqlens, int num_seqs,
                        int total_tokens, int max_seqlen, int Hq, int Hkv, int d, int causal,
                        int window, float scale, int o_dtype, void *stream) {
    if (!sinks) return FA_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(sinks) & 3) return FA_ERR_ALIGNMENT;
    return fwd_varlen(q, k, v, o, lse, sinks, cu_seqlens, num_seqs, total_tokens,
                      max_seqlen, Hq, Hkv, d, causal, window, scale, o_dtype, stream);
}

int fa_fwd_paged(const void *q, const void *k_cache, const void *v_cache,
                 const int *block_table, const int *cu_seqlens_q, const int *seq_lens_k,
                 void *o, float *lse, const float *sinks, int num_seqs, int total_q,
                 int max_seqlen_q, int num_pages, int Hq, int Hkv, int d, int page_size,
                 int max_pages_per_seq, int causal, int window, float scale, int o_dtype,
                 void *stream) {
    if (num_seqs < 0 || total_q < 0 || max_seqlen_q < 0 || num_pages < 0 ||
        max_pages_per_seq <= 0)
        return FA_ERR_INVALID_ARG;
    int rc = check_common(Hq, Hkv, d, causal, window, scale, o_dtype);
    if (rc) return rc;
    if (page_size != 16) return FA_ERR_UNSUPPORTED;
    if (num_seqs == 0 || total_q == 0 || max_seqlen_q == 0) return FA_OK;
    if (num_pages == 0) return FA_ERR_INVALID_ARG;
    if (!q || !k_cache || !v_cache || !block_table || !cu_seqlens_q || !seq_lens_k || !o)
        return FA_ERR_INVALID_ARG;
    if (total_q > INT32_MAX / 2 || (long long)num_pages * page_size > INT32_MAX / 2 ||
        (long long)max_pages_per_seq * page_size > INT32_MAX / 2)
        return FA_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o) ||
        (reinterpret_cast<uintptr_t>(block_table) & 3) ||
        (reinterpret_cast<uintptr_t>(cu_seqlens_q) & 3) ||
        (reinterpret_cast<uintptr_t>(seq_lens_k) & 3) ||
        (lse && (reinterpret_cast<uintptr_t>(lse) & 3)) ||
        (sinks && (reinterpret_cast<uintptr_t>(sinks) & 3)))
        return FA_ERR_ALIGNMENT;
    fa::PrefillArgs a{};
    a.q = q; a.k = k_cache; a.v = v_cache; a.o = o; a.lse = lse;
    a.cu_seqlens = cu_seqlens_q;
    a.num_seqs = num_seqs;
    a.seqlen = 0;
    a.total_tokens = total_q;
    a.max_seqlen = max_seqlen_q;
    a.Hq = Hq; a.Hkv = Hkv; a.d = d;
    a.causal = causal;
    a.window = window > 0 ? window : 0;
    a.scale = scale;
    a.o_fp32 = o_dtype == FA_OUT_FP32;
    a.sinks = sinks;
    a.paged = 1;
    a.block_table = block_table;
    a.seq_lens_k = seq_lens_k;
    a.max_pages = max_pages_per_seq;
    a.num_pages = num_pages;
    return map_rc(fa::launch_prefill(a, static_cast<cudaStream_t>(stream)));
}

size_t fa_bwd_workspace_bytes(int total_tokens, int Hq, int d) {
    return fa::bwd_workspace_bytes(total_tokens, Hq, d);
}

}  // extern "C"

namespace {

int bwd_common(const void *q, const void *k, const void *v, const void *o, const void *dout,
               const float *lse, void *dq, void *dk, void *dv, int Hq, int Hkv, int d,
               int causal, int window, float scale, long long total, void *workspace,
               size_t workspace_bytes) {
    int rc = check_common(Hq, Hkv, d, causal, window, scale, FA_OUT_BF16);
    if (rc) return rc;
    if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
    if (total > INT32_MAX / 2 || total * Hq > INT32_MAX / 2) return FA_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) ||
        !aligned16(dq) || !aligned16(dk) || !aligned16(dv) ||
        (reinterpret_cast<uintptr_t>(lse) & 3))
        return FA_ERR_ALIGNMENT;
    const size_t need = fa::bwd_workspace_bytes(total, Hq, d);
    if (!workspace || workspace_bytes < need) return FA_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255) return FA_ERR_ALIGNMENT;
    return FA_OK;
}

}  // namespace

extern "C" {

}  // extern "C"

namespace {

int bwd_dense_call(const void *q, const void *k, const void *v, const void *o,
                   const void *dout, const float *lse, const float *sinks, void *dq, void *dk,
                   void *dv, float *dsinks, int B, int Hq, int Hkv, int N, int d, int causal,
                   int window, float scale, void *workspace, size_t workspace_bytes,
                   void *stream) {
    if (B < 0 || N < 0) return FA_ERR_INVALID_ARG;
    int rc = check_common(Hq, Hkv, d, causal, window, scale, FA_OUT_BF16);
    if (rc) return rc;
    if (B == 0 || N == 0) return FA_OK;
    rc = bwd_common(q, k, v, o, dout, lse, dq, dk, dv, Hq, Hkv, d, causal, window, scale,
                    (long long)B * N, workspace, workspace_bytes);
    if (rc) return rc;
    fa::BwdArgs a{};
    a.q = q; a.k = k; a.v = v; a.o = o; a.dout = dout; a.lse = lse;
    a.dq = dq; a.dk = dk; a.dv = dv;
    a.cu_seqlens = nullptr;
    a.num_seqs = B;
    a.seqlen = N;
    a.total_tokens = B * N;
    a.max_seqlen = N;
    a.Hq = Hq; a.Hkv = Hkv; a.d = d;
    a.causal = causal;
    a.window = window > 0 ? window : 0;
    a.scale = scale;
    a.workspace = workspace;
    a.sinks = sinks;
    a.dsinks = dsinks;
    return map_rc(fa::launch_bwd(a, static_cast<cudaStream_t>(stream)));
}

int bwd_varlen_call(const void *q, const void *k, const void *v, const void *o,
                    const void *dout, const float *lse, const float *sinks, void *dq, void *dk,
                    void *dv, float *dsinks, const int *cu_seqlens, int num_seqs,
                    int total_tokens, int max_seqlen, int Hq, int Hkv, int d, int causal,
                    int window, float scale, void *workspace, size_t workspace_bytes,
                    void *stream) {
    if (num_seqs < 0 || total_tokens < 0 || max_seqlen < 0) return FA_ERR_INVALID_ARG;
    int rc = check_common(Hq, Hkv, d, causal, window, scale, FA_OUT_BF16);
    if (rc) return rc;
    if (num_seqs == 0 || total_tokens == 0 || max_seqlen == 0) return FA_OK;
    if (!cu_seqlens) return FA_ERR_INVALID_ARG;
    rc = bwd_common(q, k, v, o, dout, lse, dq, dk, dv, Hq, Hkv, d, causal, window, scale,
                    total_tokens, workspace, workspace_bytes);
    if (rc) return rc;
    if (reinterpret_cast<uintptr_t>(cu_seqlens) & 3) return FA_ERR_ALIGNMENT;
    fa::BwdArgs a{};
    a.q = q; a.k = k; a.v = v; a.o = o; a.dout = dout; a.lse = lse;
    a.dq = dq; a.dk = dk; a.dv = dv;
    a.cu_seqlens = cu_seqlens;
    a.num_seqs = num_seqs;
    a.seqlen = 0;
    a.total_tokens = total_tokens;
    a.max_seqlen = max_seqlen;
    a.Hq = Hq; a.Hkv = Hkv; a.d = d;
    a.causal = causal;
    a.window = window > 0 ? window : 0;
    a.scale = scale;
    a.workspace = workspace;
    a.sinks = sinks;
    a.dsinks = dsinks;
    return map_rc(fa::launch_bwd(a, static_cast<cudaStream_t>(stream)));
}

int check_sink_pair(const float *sinks, const float *dsinks) {
    if (!sinks || !dsinks) return FA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(sinks) & 3) || (reinterpret_cast<uintptr_t>(dsinks) & 3))
        return FA_ERR_ALIGNMENT;
    return FA_OK;
}

}  // namespace

extern "C" {

int fa_bwd(const void *q, const void *k, const void *v, const void *o, const void *dout,
           const float *lse, void *dq, void *dk, void *dv, int B, int Hq, int Hkv, int N, int d,
           int causal, int window, float scale, void *workspace, size_t workspace_bytes,
           void *stream) {
    return bwd_dense_call(q, k, v, o, dout, lse, nullptr, dq, dk, dv, nullptr, B, Hq, Hkv, N,
                          d, causal, window, scale, workspace, workspace_bytes, stream);
}

int fa_bwd_sinks(const void *q, const void *k, const void *v, const void *o, const void *dout,
                 const float *lse, const float *sinks, void *dq, void *dk, void *dv,
                 float *dsinks, int B, int Hq, int Hkv, int N, int d, int causal, int window,
                 float scale, void *workspace, size_t workspace_bytes, void *stream) {
    const int rc = check_sink_pair(sinks, dsinks);
    if (rc) return rc;
    return bwd_dense_call(q, k, v, o, dout, lse, sinks, dq, dk, dv, dsinks, B, Hq, Hkv, N, d,
                          causal, window, scale, workspace, workspace_bytes, stream);
}

int fa_bwd_varlen(const void *q, const void *k, const void *v, const void *o,
                  const void *dout, const float *lse, void *dq, void *dk, void *dv,
                  const int *cu_seqlens, int num_seqs, int total_tokens, int max_seqlen,
                  int Hq, int Hkv, int d, int causal, int window, float scale, void *workspace,
                  size_t workspace_bytes, void *stream) {
    return bwd_varlen_call(q, k, v, o, dout, lse, nullptr, dq, dk, dv, nullptr, cu_seqlens,
                           num_seqs, total_tokens, max_seqlen, Hq, Hkv, d, causal, window,
                           scale, workspace, workspace_bytes, stream);
}

int fa_bwd_varlen_sinks(const void *q, const void *k, const void *v, const void *o,
                        const void *dout, const float *lse, const float *sinks, void *dq,
                        void *dk, void *dv, float *dsinks, const int *cu_seqlens, int num_seqs,
                        int total_tokens, int max_seqlen, int Hq, int Hkv, int d, int causal,
                        int window, float scale, void *workspace, size_t workspace_bytes,
                        void *stream) {
    const int rc = check_sink_pair(sinks, dsinks);
    if (rc) return rc;
    return bwd_varlen_call(q, k, v, o, dout, lse, sinks, dq, dk, dv, dsinks, cu_seqlens,
                           num_seqs, total_tokens, max_seqlen, Hq, Hkv, d, causal, window,
                           scale, workspace, workspace_bytes, stream);
}

size_t fa_decode_workspace_bytes(int num_seqs, int Hq, int d, int page_size,
                                 int max_pages_per_seq) {
    return fa::decode_workspace_bytes(num_seqs, Hq, d, page_size, max_pages_per_seq);
}

}  // extern "C"

namespace {

int decode_impl_call(const void *q, const void *k_cache, const void *v_cache,
                     const int *block_table, const int *seq_lens, void *o, float *lse,
                     const float *sinks, int num_seqs, int num_pages, int Hq, int Hkv, int d,
                     int page_size, int max_pages_per_seq, float scale, void *workspace,
                     size_t workspace_bytes, void *stream, const float *k_scale = nullptr,
                     const float *v_scale = nullptr) {
    if (num_seqs < 0 || num_pages < 0 || max_pages_per_seq <= 0) return FA_ERR_INVALID_ARG;
    int rc = check_common(Hq, Hkv, d, 0, 0, scale, FA_OUT_BF16);
    if (rc) return rc;
    if (page_size != 16) return FA_ERR_UNSUPPORTED;
    if (num_seqs == 0) return FA_OK;
    if (num_pages == 0) return FA_ERR_INVALID_ARG;
    if (!q || !k_cache || !v_cache || !block_table || !seq_lens || !o) return FA_ERR_INVALID_ARG;
    if ((long long)num_pages * page_size > INT32_MAX / 2) return FA_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o) ||
        (reinterpret_cast<uintptr_t>(block_table) & 3) ||
        (reinterpret_cast<uintptr_t>(seq_lens) & 3) ||
        (lse && (reinterpret_cast<uintptr_t>(lse) & 3)))
        return FA_ERR_ALIGNMENT;
    const size_t need = fa::decode_workspace_bytes(num_seqs, Hq, d, page_size, max_pages_per_seq);
    if (need == 0) return FA_ERR_UNSUPPORTED;
    if (!workspace || workspace_bytes < need) return FA_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255) return FA_ERR_ALIGNMENT;
    fa::DecodeArgs a{};
    a.q = q; a.k_cache = k_cache; a.v_cache = v_cache;
    a.block_table = block_table; a.seq_lens = seq_lens;
    a.o = o; a.lse = lse;
    a.num_seqs = num_seqs; a.num_pages = num_pages;
    a.Hq = Hq; a.Hkv = Hkv; a.d = d; a.page_size = page_size;
    a.max_pages = max_pages_per_seq;
    a.scale = scale;
    a.workspace = workspace;
    a.sinks = sinks;
    a.fp8 = k_scale != nullptr;
    a.k_scale = k_scale;
    a.v_scale = v_scale;
    a.workspace_bytes = workspace_bytes;
    return map_rc(fa::launch_decode(a, static_cast<cudaStream_t>(stream)));
}

}  // namespace

extern "C" {

int fa_decode_paged(const void *q, const void *k_cache, const void *v_cache,
                    const int *block_table, const int *seq_lens, void *o, float *lse,
                    int num_seqs, int num_pages, int Hq, int Hkv, int d, int page_size,
                    int max_pages_per_seq, float scale, void *workspace, size_t workspace_bytes,
                    void *stream) {
    return decode_impl_call(q, k_cache, v_cache, block_table, seq_lens, o, lse, nullptr,
                            num_seqs, num_pages, Hq, Hkv, d, page_size, max_pages_per_seq,
                            scale, workspace, workspace_bytes, stream);
}

int fa_decode_paged_fp8(const void *q, const void *k_cache, const void *v_cache,
                        const float *k_scale, const float *v_scale, const int *block_table,
                        const int *seq_lens, void *o, float *lse, const float *sinks,
                        int num_seqs, int num_pages, int Hq, int Hkv, int d, int page_size,
                        int max_pages_per_seq, float scale, void *workspace,
                        size_t workspace_bytes, void *stream) {
    if (!k_scale || !v_scale) return FA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(k_scale) & 3) || (reinterpret_cast<uintptr_t>(v_scale) & 3) ||
        (sinks && (reinterpret_cast<uintptr_t>(sinks) & 3)))
        return FA_ERR_ALIGNMENT;
    return decode_impl_call(q, k_cache, v_cache, block_table, seq_lens, o, lse, sinks,
                            num_seqs, num_pages, Hq, Hkv, d, page_size, max_pages_per_seq,
                            scale, workspace, workspace_bytes, stream, k_scale, v_scale);
}

int fa_decode_paged_sinks(const void *q, const void *k_cache, const void *v_cache,
                          const int *block_table, const int *seq_lens, void *o, float *lse,
                          const float *sinks, int num_seqs, int num_pages, int Hq, int Hkv,
                          int d, int page_size, int max_pages_per_seq, float scale,
                          void *workspace, size_t workspace_bytes, void *stream) {
    if (!sinks) return FA_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(sinks) & 3) return FA_ERR_ALIGNMENT;
    return decode_impl_call(q, k_cache, v_cache, block_table, seq_lens, o, lse, sinks,
                            num_seqs, num_pages, Hq, Hkv, d, page_size, max_pages_per_seq,
                            scale, workspace, workspace_bytes, stream);
}

size_t fa_fp8_workspace_bytes(int B, int N, int Hkv) {
    if (B <= 0 || N <= 0 || Hkv <= 0) return 0;
    return (size_t)B * Hkv * (size_t)((N + 127) / 128) * sizeof(float);
}

int fa_fp8_prepare(const void *q, const void *k, const void *v, const float *signs,
                   void *q8, void *k8, void *vt8, float *q_scale, float *k_scale,
                   float *v_scale, int B, int N, int Hq, int Hkv, int d, void *workspace,
                   size_t workspace_bytes, void *stream) {
    if (B < 0 || N < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
    if (d != 128) return (d == 64) ? FA_ERR_UNSUPPORTED : FA_ERR_INVALID_ARG;
    if (B == 0 || N == 0) return FA_OK;
    if (!q || !k || !v || !q8 || !k8 || !vt8 || !q_scale || !k_scale || !v_scale)
        return FA_ERR_INVALID_ARG;
    if ((long long)B * N > INT32_MAX / 2) return FA_ERR_UNSUPPORTED;
    const size_t need = fa_fp8_workspace_bytes(B, N, Hkv);
    if (!workspace || workspace_bytes < need) return FA_ERR_WORKSPACE;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(q8) || !aligned16(k8) ||
        !aligned16(vt8) || (signs && !aligned16(signs)) ||
        (reinterpret_cast<uintptr_t>(q_scale) & 3) || (reinterpret_cast<uintptr_t>(k_scale) & 3) ||
        (reinterpret_cast<uintptr_t>(v_scale) & 3) || (reinterpret_cast<uintptr_t>(workspace) & 3))
        return FA_ERR_ALIGNMENT;
    fa::Fp8PrepArgs a{};
    a.q = q; a.k = k; a.v = v; a.signs = signs;
    a.q8 = q8; a.k8 = k8; a.vt8 = vt8;
    a.q_scale = q_scale; a.k_scale = k_scale; a.v_scale = v_scale;
    a.v_block_max = static_cast<float *>(workspace);
    a.B = B; a.N = N; a.Hq = Hq; a.Hkv = Hkv; a.d = d;
    a.vt_stride = (N + 15) / 16 * 16;
    return map_rc(fa::launch_fp8_prepare(a, static_cast<cudaStream_t>(stream)));
}

int fa_fwd_fp8(const void *q8, const void *k8, const void *vt8, const float *q_scale,
               const float *k_scale, const float *v_scale, void *o, float *lse, int B,
               int Hq, int Hkv, int N, int d, int causal, int window, float scale,
               int o_dtype, void *stream) {
    if (B < 0 || N < 0) return FA_ERR_INVALID_ARG;
    int rc = check_common(Hq, Hkv, d, causal, window, scale, o_dtype);
    if (rc) return rc;
    if (d != 128) return FA_ERR_UNSUPPORTED;
    if (B == 0 || N == 0) return FA_OK;
    if (!q8 || !k8 || !vt8 || !o || !q_scale || !k_scale || !v_scale) return FA_ERR_INVALID_ARG;
    if ((long long)B * N > INT32_MAX / 2) return FA_ERR_UNSUPPORTED;
    if (!aligned16(q8) || !aligned16(k8) || !aligned16(vt8) || !aligned16(o) ||
        (lse && (reinterpret_cast<uintptr_t>(lse) & 3)) ||
        (reinterpret_cast<uintptr_t>(q_scale) & 3) || (reinterpret_cast<uintptr_t>(k_scale) & 3) ||
        (reinterpret_cast<uintptr_t>(v_scale) & 3))
        return FA_ERR_ALIGNMENT;
    fa::PrefillArgs a{};
    a.q = q8; a.k = k8; a.v = vt8; a.o = o; a.lse = lse;
    a.cu_seqlens = nullptr;
    a.num_seqs = B;
    a.seqlen = N;
    a.total_tokens = B * N;
    a.max_seqlen = N;
    a.Hq = Hq; a.Hkv = Hkv; a.d = d;
    a.causal = causal;
    a.window = window > 0 ? window : 0;
    a.scale = scale;
    a.o_fp32 = o_dtype == FA_OUT_FP32;
    a.q_scale = q_scale; a.k_scale = k_scale; a.v_scale = v_scale;
    a.vt_stride = (N + 15) / 16 * 16;
    return map_rc(fa::launch_prefill_fp8(a, static_cast<cudaStream_t>(stream)));
}

const char *fa_status_string(int status) {
    switch (status) {
    case FA_OK: return "ok";
    case FA_ERR_INVALID_ARG: return "invalid argument";
    case FA_ERR_UNSUPPORTED: return "unsupported configuration";
    case FA_ERR_ALIGNMENT: return "pointer not aligned";
    case FA_ERR_WORKSPACE: return "workspace missing or too small";
    case FA_ERR_CUDA: return "CUDA runtime error";
    case FA_ERR_TIMEOUT: return "device-side wait timed out";
    default: return "unknown status";
    }
}

int fa_check_device_error(void *stream) {
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return FA_ERR_CUDA;
    int word = 0;
    const int zero = 0;
    if (cudaMemcpyFromSymbol(&word, fa::g_device_error, sizeof word) != cudaSuccess)
        return FA_ERR_CUDA;
    if (word && cudaMemcpyToSymbol(fa::g_device_error, &zero, sizeof zero) != cudaSuccess)
        return FA_ERR_CUDA;
    if (word == fa::kDevErrTimeout) return FA_ERR_TIMEOUT;
    if (word == fa::kDevErrInput) return FA_ERR_INVALID_ARG;
    return word ? FA_ERR_CUDA : FA_OK;
}

int fa_selftest_watchdog(void *stream) {
    fa::watchdog_probe_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>();
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

int fa_version(void) { return 100; }

}  // extern "C"
