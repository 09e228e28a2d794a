// fa_internal.h -- host-side declarations shared by the library's .cu files.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace fa {

// Sizes the prefill launch needs; validated by the public entry points.
struct PrefillArgs {
    const void *q, *k, *v;
    void *o;
    float *lse;
    const int *cu_seqlens;  // device; nullptr = dense batch
    int num_seqs;           // B (dense) or number of packed sequences
    int seqlen;             // N (dense only)
    int total_tokens;
    int max_seqlen;
    int Hq, Hkv, d;
    int causal, window;
    float scale;
    int o_fp32;
    const float *sinks;     // device [Hq] learned sink logits; nullptr = none
    // chunked prefill over a paged cache (k, v are the caches)
    int paged;
    const int *block_table, *seq_lens_k;
    int max_pages, num_pages;
    // document mask: one id per token; nullptr = none
    const int *doc;
    // sink tokens kept visible beside a causal window (0 = none)
    int n_sink;
    // FP8 operands (launch_prefill_fp8): q, k hold E4M3 codes, v the
    // transposed V codes [B, Hkv, d, vt_stride]; scales per (sequence, head,
    // 128-token block) for Q and K, per (sequence, KV head) for V
    const float *q_scale, *k_scale, *v_scale;
    int vt_stride;
};

int launch_prefill(const PrefillArgs &a, cudaStream_t stream);
int launch_prefill_fp8(const PrefillArgs &a, cudaStream_t stream);

// Rotation and E4M3 quantisation of the FP8 prefill's operands.
struct Fp8PrepArgs {
    const void *q, *k, *v;      // bf16 [B*N, H, d]
    const float *signs;         // [d] +-1, or nullptr: no rotation
    void *q8, *k8, *vt8;        // codes; vt8 [B, Hkv, d, vt_stride]
    float *q_scale, *k_scale, *v_scale;
    float *v_block_max;         // workspace [B, Hkv, nblk]
    int B, N, Hq, Hkv, d, vt_stride;
};

int launch_fp8_prepare(const Fp8PrepArgs &a, cudaStream_t stream);

struct DecodeArgs {
    const void *q, *k_cache, *v_cache;
    const int *block_table, *seq_lens;
    void *o;
    float *lse;
    int num_seqs, num_pages, Hq, Hkv, d, page_size, max_pages;
    float scale;
    void *workspace;
    size_t workspace_bytes;
    const float *sinks;     // device [Hq] learned sink logits; nullptr = none
    int fp8;                // caches hold FP8 E4M3 codes (1 byte) instead of bf16
    const float *k_scale, *v_scale;  // FP8: device [num_pages][Hkv] scales
};

size_t decode_workspace_bytes(int num_seqs, int Hq, int d, int page_size, int max_pages);
int launch_decode(const DecodeArgs &a, cudaStream_t stream);

// Split-KV decode of an FP8 cache on the tensor core (decode_tc_sm100.cu):
// group sizes 1, 2, 4, 8 and d = 128; writes the same chunk partials as the
// CUDA-core split kernel.
bool decode_tc_supported(const DecodeArgs &a);
int launch_decode_split_tc(const DecodeArgs &a, float *part_o, float *part_lse, int max_chunks,
                           cudaStream_t stream);

// Sizes the backward launch needs; validated by the public entry points.
struct BwdArgs {
    const void *q, *k, *v, *o, *dout;
    const float *lse;
    void *dq, *dk, *dv;
    const int *cu_seqlens;  // device; nullptr = dense batch
    int num_seqs, seqlen, total_tokens, max_seqlen;
    int Hq, Hkv, d;
    int causal, window;
    float scale;
    void *workspace;
    const float *sinks;     // [Hq] learned sink logits, or nullptr
    float *dsinks;          // [Hq] their gradient (written when sinks is set)
};

size_t bwd_workspace_bytes(long long total_tokens, int Hq, int d);
int launch_bwd(const BwdArgs &a, cudaStream_t stream);

// Number of SMs of the current device (cached per device).
int device_sm_count();

// cuTensorMapEncodeTiled through the runtime's driver entry point.
int encode_tensor_map_3d(void *map, const void *base, int elem_bytes,
                         uint64_t dim0, uint64_t dim1, uint64_t dim2,
                         uint64_t stride1_bytes, uint64_t stride2_bytes,
                         uint32_t box0, uint32_t box1, uint32_t box2, int swizzle_bytes);

}  // namespace fa
