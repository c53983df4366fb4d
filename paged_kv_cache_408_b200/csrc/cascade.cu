// cascade.cu -- decode of a batch whose sequences all begin with the same
// physical blocks (a shared prompt, sequences forked from one parent).
//
// What is computed is pa_decode's result ("Production Serving: Continuous
// Batching and PagedAttention", Step 6; per query head): softmax over every
// cached token of the sequence, applied to V.  How: the keys split into the
// shared prefix [0, P) and the sequence's own suffix [P, len), and
//   * the shared prefix is attended ONCE per kv head for all sequences: its
//     K/V are read once and the queries of every sequence and head of the
//     kv head form the rows of a dense attention on the tensor cores (the
//     prefill kernel in its shared-prefix mode), split over key ranges so
//     that it fills the SMs, giving split-K pieces 0..S-1 of every row;
//   * the decode kernel attends each suffix (pieces S..);
//   * the log-sum-exp merge combines the pieces (the same merge as split-K).
// An E4M3 prefix goes to the prefill kernel as it is: its converter warps
// widen each K/V tile to f16 on the way into shared memory (exact), and the
// per-head scales are applied to the scores and outputs as in decode.
// The three launches are chained as programmatic dependents.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace pa {

int cascade_max_parts(int max_blocks, int prefix_blocks) {
    return decode_max_parts(max_blocks - prefix_blocks, 0) + kMaxPrefixSplits;
}

size_t cascade_ws_bytes(int B, int Hq, int Hkv, int D, int max_blocks, int prefix_blocks, bool fp8) {
    (void)Hkv;
    (void)fp8;  // an E4M3 prefix is widened inside the prefill kernel: no scratch copy
    return decode_ws_bytes(B, Hq, D, cascade_max_parts(max_blocks, prefix_blocks));
}

cudaError_t launch_decode_cascade(const DecodeArgs &d, void *workspace, cudaStream_t st) {
    DecodeArgs a = d;
    a.partition_tokens = 0;
    a.max_parts = cascade_max_parts(a.max_blocks, a.prefix_blocks);
    decode_ws_carve(workspace, a.B, a.Hq, a.D, a.max_parts, a);
    PrefillArgs p{};
    p.q = a.q;
    p.n_chunks = 1;
    p.Hq = a.Hq;
    p.Hkv = a.Hkv;
    p.D = a.D;
    p.max_q_len = a.B;  // rows are sequences
    p.total_q = a.B;
    p.scale = a.scale;
    p.err = a.err;
    p.shared_len = a.prefix_blocks * 16;
    p.ws_o = a.ws_o;
    p.ws_lse = a.ws_lse;
    p.max_parts = a.max_parts;
    // split the prefix's keys so that the prefix attention fills the SMs:
    // CTAs per split = kv heads x query tiles of 256 rows (rows = sequences x
    // group), at most one split per 128-key tile
    {
        const int ctas = a.Hkv * ((a.B * (a.Hq / a.Hkv) + 255) / 256);
        const int tiles = (p.shared_len + 127) / 128;
        p.key_splits = std::max(1, std::min({sm_count() / std::max(ctas, 1), kMaxPrefixSplits, tiles}));
    }
    a.prefix_pieces = p.key_splits;
    p.block_tables = a.block_tables;  // row 0 holds the shared blocks
    p.max_blocks = a.max_blocks;
    p.num_blocks = a.num_blocks;
    p.k_cache = a.k_cache;
    p.v_cache = a.v_cache;
    if (a.fp8) {
        p.fp8 = true;
        p.k_scale = a.k_scale;
        p.v_scale = a.v_scale;
    }
    cudaError_t e = launch_prefill(p, st);
    if (e != cudaSuccess) return e;
    return launch_decode(a, st);
}

}  // namespace pa
