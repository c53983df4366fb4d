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
    int partition_tokens;  // 0: balanced split; else a multiple of 16 (fixed partitions)
    int max_parts;         // most pieces one (sequence, kv head) can be cut into
    int *ws_np;            // [B][Hkv] pieces of each (sequence, kv head), written by every call
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

// Device address of the status word on the current device (nullptr if unknown).
unsigned *status_word();

// Workspace layout shared by pa_decode_workspace_size, pa_decode and
// pa_decode_noalloc: [piece counts | partial outputs | partial log2-sum-exp],
// each region 256-byte aligned.  Every call writes what it reads (the decode
// kernel writes the piece counts and partials, the merge kernel reads them),
// so the workspace needs no initialisation and keeps nothing between calls.
constexpr int kMaxDecodeSeqs = 2048;
constexpr int kMinShareBlocks = 16;  // balanced split: smallest per-warp share, in cost units
constexpr int kMaxDecodeKvHeads = 128;
// Pieces one (sequence, kv head) of max_blocks blocks can be cut into.
inline int decode_max_parts(int max_blocks, int partition_tokens) {
    return partition_tokens == 0 ? max_blocks / kMinShareBlocks + 2
                                 : (max_blocks * 16 + partition_tokens - 1) / partition_tokens;
}
size_t decode_ws_bytes(int B, int Hq, int D, int max_parts);
// Points a.ws_np / a.ws_o / a.ws_lse into a workspace of decode_ws_bytes().
void decode_ws_carve(void *base, int B, int Hq, int D, int max_parts, DecodeArgs &a);

}  // namespace pa
