// kernels.h -- launcher interface between the C-ABI layer (api.cu) and the
// kernel translation units.  Host-only structs of plain pointers and sizes;
// all arguments have been validated by api.cu before a launcher runs.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace pa {

struct WriteArgs {
    const void *k, *v;
    const int64_t *slots;
    int64_t num_tokens;
    void *k_cache, *v_cache;
    const float *k_scale, *v_scale;
    int64_t num_blocks;
    int Hkv, D;
    bool fp8;
    unsigned *err;
};

struct CopyArgs {
    void *k_cache, *v_cache;
    const int32_t *pairs;
    int32_t num_pairs;
    int64_t num_blocks;
    int Hkv, D, elem_bytes;
    unsigned *err;
};

struct DecodeArgs {
    void *out;
    const void *q;
    const void *k_cache, *v_cache;
    const int32_t *block_tables, *seq_lens;
    int B, max_blocks, Hq, Hkv, D;
    int64_t num_blocks;
    float scale;
    const float *k_scale, *v_scale;
    int partition_tokens;  // multiple of 16
    int max_parts;         // partitions of the longest possible sequence
    float *ws_o;           // [B][Hq][max_parts][D]
    float *ws_lse;         // [B][Hq][max_parts]
    bool fp8;
    unsigned *err;
};

struct PrefillArgs {
    void *out;
    const void *q;
    const int32_t *cu_q, *prefix_lens, *block_tables;
    int n_chunks, max_blocks, Hq, Hkv, D, max_q_len, total_q;
    int64_t num_blocks;
    const void *k_cache, *v_cache;
    float scale;
    unsigned *err;
};

cudaError_t launch_write_kv(const WriteArgs &a, cudaStream_t st);
cudaError_t launch_copy_blocks(const CopyArgs &a, cudaStream_t st);
// Returns cudaErrorNotSupported for a (head_dim, group, dtype) that is not built.
cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t st);
cudaError_t launch_prefill(const PrefillArgs &a, cudaStream_t st);

// Workspace layout shared by pa_decode_workspace_size and pa_decode.
size_t decode_ws_o_bytes(int B, int Hq, int D, int max_parts);
size_t decode_ws_bytes(int B, int Hq, int D, int max_parts);

}  // namespace pa
