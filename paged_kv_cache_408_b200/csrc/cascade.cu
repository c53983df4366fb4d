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
// An E4M3 prefix is first widened to bf16 (exactly: every E4M3 value is a
// bf16 value) into workspace scratch with an identity block table, and the
// per-head scales are applied to the scores and outputs as in decode.  (The
// prefill kernel can also widen E4M3 tiles itself, on the way into shared
// memory, as chunked prefill over an E4M3 cache does; for the shared
// prefix, whose CTAs each run only a few key tiles, that measured 60.0
// against 40.2 us for the widening kernel plus the bf16 tiles on the
// 256-sequence, 2048-token-prefix batch, so the prefix is widened first.)
// The launches are chained as programmatic dependents.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace pa {
namespace {

size_t round256(size_t n) { return (n + 255) & ~(size_t)255; }

// Widen the prefix blocks of both caches (block_tables row 0) to bf16 into
// [prefix_blocks][Hkv][16][D] scratch and write the identity table.  One
// thread per 8 elements.
__global__ void __launch_bounds__(256) widen_prefix_kernel(const uint8_t *__restrict__ kc, const uint8_t *__restrict__ vc,
                                                           const int32_t *__restrict__ bt, int prefix_blocks,
                                                           int64_t num_blocks, int64_t block_elems,
                                                           uint4 *__restrict__ kout, uint4 *__restrict__ vout,
                                                           int32_t *__restrict__ ident, unsigned *err) {
    pdl_trigger();
    pdl_wait();
    const int64_t n8 = (int64_t)prefix_blocks * block_elems / 8;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n8; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t e = i * 8, j = e / block_elems, within = e - j * block_elems;
        int64_t phys = bt[j];
        if (phys < 0 || phys >= num_blocks) {
            if (within == 0) flag_error(err, PA_DEVERR_BAD_BLOCK);
            phys = 0;
        }
        const uint2 kw = *reinterpret_cast<const uint2 *>(kc + phys * block_elems + within);
        const uint2 vw = *reinterpret_cast<const uint2 *>(vc + phys * block_elems + within);
        const uint32_t kin[2] = {kw.x, kw.y}, vin[2] = {vw.x, vw.y};
        uint32_t ko[4], vo[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const float2 kf = e4m3x2_to_float2((uint16_t)(kin[p / 2] >> (16 * (p % 2))));
            const float2 vf = e4m3x2_to_float2((uint16_t)(vin[p / 2] >> (16 * (p % 2))));
            const __nv_bfloat162 kb = __floats2bfloat162_rn(kf.x, kf.y), vb = __floats2bfloat162_rn(vf.x, vf.y);
            ko[p] = *reinterpret_cast<const uint32_t *>(&kb);
            vo[p] = *reinterpret_cast<const uint32_t *>(&vb);
        }
        kout[i] = make_uint4(ko[0], ko[1], ko[2], ko[3]);
        vout[i] = make_uint4(vo[0], vo[1], vo[2], vo[3]);
    }
    for (int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; j < prefix_blocks;
         j += (int64_t)gridDim.x * blockDim.x)
        ident[j] = (int32_t)j;
}

}  // namespace

int cascade_max_parts(int max_blocks, int prefix_blocks) {
    return decode_max_parts(max_blocks - prefix_blocks, 0) + kMaxPrefixSplits;
}

size_t cascade_ws_bytes(int B, int Hq, int Hkv, int D, int max_blocks, int prefix_blocks, bool fp8) {
    size_t n = decode_ws_bytes(B, Hq, D, cascade_max_parts(max_blocks, prefix_blocks));
    if (fp8) n += round256((size_t)prefix_blocks * 4) + 2 * round256((size_t)prefix_blocks * Hkv * 16 * D * 2);
    return n;
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
    cudaError_t e = cudaSuccess;
    if (a.fp8) {
        char *sc = static_cast<char *>(workspace) + decode_ws_bytes(a.B, a.Hq, a.D, a.max_parts);
        int32_t *ident = reinterpret_cast<int32_t *>(sc);
        const int64_t block_elems = (int64_t)a.Hkv * 16 * a.D;
        uint4 *kout = reinterpret_cast<uint4 *>(sc + round256((size_t)a.prefix_blocks * 4));
        uint4 *vout = reinterpret_cast<uint4 *>(reinterpret_cast<char *>(kout) +
                                               round256((size_t)a.prefix_blocks * block_elems * 2));
        const int64_t n8 = (int64_t)a.prefix_blocks * block_elems / 8;
        const unsigned grid = (unsigned)std::min<int64_t>((n8 + 255) / 256, (int64_t)sm_count() * 8);
        e = launch_pdl(widen_prefix_kernel, dim3(grid), dim3(256), 0, st, static_cast<const uint8_t *>(a.k_cache),
                       static_cast<const uint8_t *>(a.v_cache), a.block_tables, a.prefix_blocks, a.num_blocks,
                       block_elems, kout, vout, ident, a.err);
        if (e != cudaSuccess) return e;
        p.block_tables = ident;
        p.max_blocks = a.prefix_blocks;
        p.num_blocks = a.prefix_blocks;
        p.k_cache = kout;
        p.v_cache = vout;
        p.k_scale = a.k_scale;  // bf16 tiles of E4M3 values: scale the scores and outputs
        p.v_scale = a.v_scale;
    } else {
        p.block_tables = a.block_tables;  // row 0 holds the shared blocks
        p.max_blocks = a.max_blocks;
        p.num_blocks = a.num_blocks;
        p.k_cache = a.k_cache;
        p.v_cache = a.v_cache;
    }
    e = launch_prefill(p, st);
    if (e != cudaSuccess) return e;
    return launch_decode(a, st);
}

}  // namespace pa
