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
    int prefix_blocks;     // cascade: the first prefix_blocks of every row are attended elsewhere (pieces
                           // 0..prefix_pieces-1); this launch attends the rest as the pieces after them (0: off)
    int prefix_pieces;
    int merge_spec;        // pieces the merge kernel loads per row before it has read the row's piece count
                           // (set by the decode launcher)
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
    // Shared-prefix mode (shared_len > 0): one "chunk" of total_q decode
    // sequences (q is the decode q [total_q][Hq][D]) that all attend keys
    // [0, shared_len) through block_tables row 0, without causal extension,
    // split over key_splits ranges of whole key tiles (at most one range per
    // tile); instead of bf16 out, each row's normalised fp32 output and
    // log2-sum-exp over range z become split-K piece z of that row in ws_o /
    // ws_lse.  Scores are scaled by k_scale[kv head] and outputs by
    // v_scale[kv head] when given.
    int shared_len;
    const float *k_scale, *v_scale;
    float *ws_o, *ws_lse;
    int max_parts;
    int key_splits;
    // E4M3 cache (k_scale / v_scale required): K/V tiles are widened to f16
    // on the way into shared memory and the MMAs take f16 operands
    bool fp8;
};

cudaError_t launch_write_kv(const WriteArgs &a, cudaStream_t st);
cudaError_t launch_copy_blocks(const CopyArgs &a, cudaStream_t st);
// Returns cudaErrorNotSupported for a (head_dim, group, dtype) that is not built.
cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t st);
cudaError_t launch_prefill(const PrefillArgs &a, cudaStream_t st);

// Device address of the status word on the current device (nullptr if unknown).
unsigned *status_word();

// Streaming multiprocessors of the current device (queried once per device
// and cached; 148 on a B200).  Grids are sized in multiples of it.
int sm_count();

// Workspace layout shared by pa_decode_workspace_size, pa_decode and
// pa_decode_noalloc: [piece counts | partial outputs | partial log2-sum-exp],
// each region 256-byte aligned.  Every call writes what it reads (the decode
// kernel writes the piece counts and partials, the merge kernel reads them),
// so the workspace needs no initialisation and keeps nothing between calls.
constexpr int kMaxDecodeSeqs = 2048;
constexpr int kMinShareBlocks = 16;  // balanced split: smallest per-warp share, in cost units
constexpr int kMaxDecodeKvHeads = 128;
// Widest block table any entry point accepts (PA_MAX_BLOCKS_PER_SEQ): token
// positions (16 * max_blocks) and piece counts stay far inside int32.
constexpr int kMaxBlocksPerSeq = PA_MAX_BLOCKS_PER_SEQ;
// Pieces one (sequence, kv head) of max_blocks blocks can be cut into
// (max_blocks in [1, kMaxBlocksPerSeq], checked by every entry point).
inline int decode_max_parts(int max_blocks, int partition_tokens) {
    const int64_t mb = max_blocks;
    return (int)(partition_tokens == 0 ? mb / kMinShareBlocks + 2 : (mb * 16 + partition_tokens - 1) / partition_tokens);
}
size_t decode_ws_bytes(int B, int Hq, int D, int max_parts);
// Points a.ws_np / a.ws_o / a.ws_lse into a workspace of decode_ws_bytes().
void decode_ws_carve(void *base, int B, int Hq, int D, int max_parts, DecodeArgs &a);

// Cascade decode (cascade.cu): rows share their first prefix_blocks blocks.
// The workspace is the decode workspace for cascade_max_parts() pieces,
// followed (fp8 caches) by an identity block table and bf16 copies of the
// shared prefix of both caches.
constexpr int kMaxPrefixSplits = 4;  // key ranges the shared prefix is split into
int cascade_max_parts(int max_blocks, int prefix_blocks);
size_t cascade_ws_bytes(int B, int Hq, int Hkv, int D, int max_blocks, int prefix_blocks, bool fp8);
cudaError_t launch_decode_cascade(const DecodeArgs &a, void *workspace, cudaStream_t st);

}  // namespace pa
