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
};

int launch_prefill(const PrefillArgs &a, cudaStream_t stream);

struct DecodeArgs {
    const void *q, *k_cache, *v_cache;
    const int *block_table, *seq_lens;
    void *o;
    float *lse;
    int num_seqs, num_pages, Hq, Hkv, d, page_size, max_pages;
    float scale;
    void *workspace;
    size_t workspace_bytes;
};

size_t decode_workspace_bytes(int num_seqs, int Hq, int d, int page_size, int max_pages);
int launch_decode(const DecodeArgs &a, cudaStream_t stream);

// Number of SMs of the current device (cached per device).
int device_sm_count();

// cuTensorMapEncodeTiled through the runtime's driver entry point.
int encode_tensor_map_3d(void *map, const void *base, int elem_bytes,
                         uint64_t dim0, uint64_t dim1, uint64_t dim2,
                         uint64_t stride1_bytes, uint64_t stride2_bytes,
                         uint32_t box0, uint32_t box1, uint32_t box2, bool swizzle128);

}  // namespace fa
