// decode_noalloc.cu -- pa_decode_noalloc: paged decode whose split-K scratch
// is a fixed device array inside the library, for callers that cannot
// allocate device memory (see include/pa.h).  No cudaMalloc, cudaFree or
// allocating library routine is called anywhere on this path.
#include <mutex>

#include "common.cuh"
#include "kernels.h"

// The scratch: piece counts, partial outputs and partial log-sum-exps of the
// split-K merge.  Every GPU that loads the library holds it
// until the process exits.  Host code must not use this name as an address
// (on the host it is only a stand-in); it uses the address looked up below.
static __device__ __align__(256) unsigned char pa_noalloc_scratch[PA_DECODE_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;

// Device address of the scratch on the current device, looked up once per
// device (with that device current) and cached.
int scratch_address(void **out) {
    static std::mutex mu;
    static void *addr[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, pa_noalloc_scratch) != cudaSuccess || !p) return PA_ERR_CUDA;
        addr[dev] = p;
    }
    *out = addr[dev];
    return PA_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

extern "C" int pa_decode_noalloc(void *out, const void *q, const void *k_cache, const void *v_cache,
                                 const int32_t *block_tables, const int32_t *seq_lens, int32_t num_seqs,
                                 int32_t max_blocks_per_seq, int32_t num_q_heads, float scale,
                                 const float *k_scale, const float *v_scale, int32_t partition_tokens,
                                 const pa_cache_desc *desc, pa_stream_t stream) {
    // argument checks (the same rules as pa_decode)
    if (!desc || desc->block_size != PA_BLOCK_SIZE || desc->num_blocks <= 0 || desc->num_kv_heads <= 0)
        return PA_ERR_INVALID_ARG;
    if (desc->dtype != PA_DTYPE_BF16 && desc->dtype != PA_DTYPE_FP8_E4M3) return PA_ERR_INVALID_ARG;
    if (desc->head_dim != 64 && desc->head_dim != 128) return PA_ERR_UNSUPPORTED;
    if (num_seqs < 0 || num_seqs > pa::kMaxDecodeSeqs || max_blocks_per_seq <= 0 ||
        max_blocks_per_seq > pa::kMaxBlocksPerSeq || num_q_heads <= 0)
        return PA_ERR_INVALID_ARG;
    if (num_q_heads % desc->num_kv_heads != 0) return PA_ERR_INVALID_ARG;
    if (desc->num_kv_heads > pa::kMaxDecodeKvHeads) return PA_ERR_UNSUPPORTED;
    const int G = num_q_heads / desc->num_kv_heads;
    if (G != 1 && G != 2 && G != 4 && G != 8) return PA_ERR_UNSUPPORTED;
    if (partition_tokens != 0 && (partition_tokens < 16 || partition_tokens > 2048 || partition_tokens % 16))
        return PA_ERR_INVALID_ARG;
    if (num_seqs == 0) return PA_OK;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !seq_lens) return PA_ERR_INVALID_ARG;
    if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache)) return PA_ERR_INVALID_ARG;
    const bool fp8 = desc->dtype == PA_DTYPE_FP8_E4M3;
    if (fp8 && (!k_scale || !v_scale)) return PA_ERR_INVALID_ARG;

    // the shape must fit the fixed scratch
    const int P = partition_tokens;
    const int max_parts = pa::decode_max_parts(max_blocks_per_seq, P);
    const size_t need = max_parts > 1 ? pa::decode_ws_bytes(num_seqs, num_q_heads, desc->head_dim, max_parts) : 0;
    if (need > PA_DECODE_NOALLOC_SCRATCH_BYTES) return PA_ERR_WORKSPACE;

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    pa::DecodeArgs a{out, q, k_cache, v_cache, block_tables, seq_lens, num_seqs, max_blocks_per_seq,
                     num_q_heads, desc->num_kv_heads, desc->head_dim, desc->num_blocks, scale, k_scale, v_scale,
                     P, max_parts, nullptr, nullptr, nullptr, fp8, pa::status_word()};
    if (max_parts > 1) {
        void *scratch = nullptr;
        const int rc = scratch_address(&scratch);
        if (rc != PA_OK) return rc;
        pa::decode_ws_carve(scratch, num_seqs, num_q_heads, desc->head_dim, max_parts, a);
    }
    const cudaError_t e = pa::launch_decode(a, st);
    if (e == cudaSuccess) return PA_OK;
    return e == cudaErrorNotSupported ? PA_ERR_UNSUPPORTED : PA_ERR_CUDA;
}
