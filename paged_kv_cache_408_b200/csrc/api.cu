// api.cu -- the extern "C" entry points declared in include/pa.h: argument
// validation on the host, then one or two kernel launches on the caller's
// stream.  No allocation, no synchronisation (except the explicit status
// query).
#include <mutex>

#include "common.cuh"
#include "kernels.h"

// Device status word: kernels OR PA_DEVERR_* bits into it.  One copy per
// device that loads the library.
__device__ unsigned pa_device_status_word;

namespace {

constexpr int kMaxDevices = 64;
constexpr int kMaxSeqs = pa::kMaxDecodeSeqs;

unsigned *status_word_ptr() {
    static std::mutex mu;
    static unsigned *ptr[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, pa_device_status_word) != cudaSuccess) return nullptr;
        ptr[dev] = static_cast<unsigned *>(p);
    }
    return ptr[dev];
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

int check_desc(const pa_cache_desc *d) {
    if (!d) return PA_ERR_INVALID_ARG;
    if (d->block_size != PA_BLOCK_SIZE || d->num_blocks <= 0 || d->num_kv_heads <= 0) return PA_ERR_INVALID_ARG;
    if (d->dtype != PA_DTYPE_BF16 && d->dtype != PA_DTYPE_FP8_E4M3) return PA_ERR_INVALID_ARG;
    if (d->head_dim != 64 && d->head_dim != 128) return PA_ERR_UNSUPPORTED;
    return PA_OK;
}

int elem_bytes(const pa_cache_desc *d) { return d->dtype == PA_DTYPE_BF16 ? 2 : 1; }

int from_cuda(cudaError_t e) {
    if (e == cudaSuccess) return PA_OK;
    if (e == cudaErrorNotSupported) return PA_ERR_UNSUPPORTED;
    return PA_ERR_CUDA;
}

// 0 selects the balanced split; otherwise fixed partitions of 16..2048 tokens.
int resolve_partition(int32_t partition_tokens, int *out) {
    const int p = partition_tokens;
    if (p != 0 && (p < 16 || p > 2048 || p % 16 != 0)) return PA_ERR_INVALID_ARG;
    *out = p;
    return PA_OK;
}

}  // namespace

unsigned *pa::status_word() { return status_word_ptr(); }

int pa::sm_count() {
    static std::mutex mu;
    static int n[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 1;
    std::lock_guard<std::mutex> lock(mu);
    if (!n[dev] && cudaDeviceGetAttribute(&n[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) n[dev] = 0;
    return n[dev] > 0 ? n[dev] : 1;
}

extern "C" {

int pa_version(void) { return 300; }

const char *pa_status_string(int status) {
    switch (status) {
        case PA_OK: return "PA_OK";
        case PA_ERR_INVALID_ARG: return "PA_ERR_INVALID_ARG";
        case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED";
        case PA_ERR_WORKSPACE: return "PA_ERR_WORKSPACE";
        case PA_ERR_CUDA: return "PA_ERR_CUDA";
        case PA_ERR_DEVICE: return "PA_ERR_DEVICE";
        case PA_ERR_TIMEOUT: return "PA_ERR_TIMEOUT";
        default: return "PA_ERR_UNKNOWN";
    }
}

int pa_write_kv(const void *k, const void *v, const int64_t *slot_mapping, int64_t num_tokens, void *k_cache,
                void *v_cache, const float *k_scale, const float *v_scale, const pa_cache_desc *desc,
                pa_stream_t stream) {
    int rc = check_desc(desc);
    if (rc != PA_OK) return rc;
    if (num_tokens < 0) return PA_ERR_INVALID_ARG;
    if (num_tokens == 0) return PA_OK;
    if (!k || !v || !slot_mapping || !k_cache || !v_cache) return PA_ERR_INVALID_ARG;
    if (!aligned16(k) || !aligned16(v) || !aligned16(k_cache) || !aligned16(v_cache)) return PA_ERR_INVALID_ARG;
    const bool fp8 = desc->dtype == PA_DTYPE_FP8_E4M3;
    if (fp8 && (!k_scale || !v_scale)) return PA_ERR_INVALID_ARG;
    pa::WriteArgs a{k, v, slot_mapping, num_tokens, k_cache, v_cache, k_scale, v_scale, desc->num_blocks,
                    desc->num_kv_heads, desc->head_dim, fp8, status_word_ptr()};
    return from_cuda(pa::launch_write_kv(a, static_cast<cudaStream_t>(stream)));
}

int pa_copy_blocks(void *k_cache, void *v_cache, const int32_t *src_dst_pairs, int32_t num_pairs,
                   const pa_cache_desc *desc, pa_stream_t stream) {
    int rc = check_desc(desc);
    if (rc != PA_OK) return rc;
    if (num_pairs < 0) return PA_ERR_INVALID_ARG;
    if (num_pairs == 0) return PA_OK;
    if (!k_cache || !v_cache || !src_dst_pairs) return PA_ERR_INVALID_ARG;
    if (!aligned16(k_cache) || !aligned16(v_cache)) return PA_ERR_INVALID_ARG;
    pa::CopyArgs a{k_cache, v_cache, src_dst_pairs, num_pairs, desc->num_blocks, desc->num_kv_heads,
                   desc->head_dim, elem_bytes(desc), status_word_ptr()};
    return from_cuda(pa::launch_copy_blocks(a, static_cast<cudaStream_t>(stream)));
}

int pa_decode_workspace_size(int32_t num_seqs, int32_t num_q_heads, int32_t head_dim, int32_t max_blocks_per_seq,
                             int32_t partition_tokens, size_t *bytes) {
    if (!bytes || num_seqs < 0 || num_q_heads <= 0 || max_blocks_per_seq <= 0 ||
        max_blocks_per_seq > pa::kMaxBlocksPerSeq)
        return PA_ERR_INVALID_ARG;
    if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
    int P = 0;
    int rc = resolve_partition(partition_tokens, &P);
    if (rc != PA_OK) return rc;
    const int max_parts = pa::decode_max_parts(max_blocks_per_seq, P);
    *bytes = max_parts > 1 ? pa::decode_ws_bytes(num_seqs, num_q_heads, head_dim, max_parts) : 0;
    return PA_OK;
}

int pa_decode(void *out, const void *q, const void *k_cache, const void *v_cache, const int32_t *block_tables,
              const int32_t *seq_lens, int32_t num_seqs, int32_t max_blocks_per_seq, int32_t num_q_heads,
              float scale, const float *k_scale, const float *v_scale, int32_t partition_tokens,
              void *workspace, size_t workspace_bytes, const pa_cache_desc *desc, pa_stream_t stream) {
    int rc = check_desc(desc);
    if (rc != PA_OK) return rc;
    if (num_seqs < 0 || num_seqs > kMaxSeqs || max_blocks_per_seq <= 0 ||
        max_blocks_per_seq > pa::kMaxBlocksPerSeq || num_q_heads <= 0)
        return PA_ERR_INVALID_ARG;
    if (num_q_heads % desc->num_kv_heads != 0) return PA_ERR_INVALID_ARG;
    if (desc->num_kv_heads > pa::kMaxDecodeKvHeads) return PA_ERR_UNSUPPORTED;
    const int G = num_q_heads / desc->num_kv_heads;
    if (G != 1 && G != 2 && G != 4 && G != 8) return PA_ERR_UNSUPPORTED;
    if (num_seqs == 0) return PA_OK;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !seq_lens) return PA_ERR_INVALID_ARG;
    if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache)) return PA_ERR_INVALID_ARG;
    const bool fp8 = desc->dtype == PA_DTYPE_FP8_E4M3;
    if (fp8 && (!k_scale || !v_scale)) return PA_ERR_INVALID_ARG;
    int P = 0;
    rc = resolve_partition(partition_tokens, &P);
    if (rc != PA_OK) return rc;
    const int max_parts = pa::decode_max_parts(max_blocks_per_seq, P);
    pa::DecodeArgs a{out, q, k_cache, v_cache, block_tables, seq_lens, num_seqs, max_blocks_per_seq,
                     num_q_heads, desc->num_kv_heads, desc->head_dim, desc->num_blocks, scale, k_scale, v_scale,
                     P, max_parts, nullptr, nullptr, nullptr, fp8, status_word_ptr()};
    if (max_parts > 1) {
        const size_t need = pa::decode_ws_bytes(num_seqs, num_q_heads, desc->head_dim, max_parts);
        if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255))
            return PA_ERR_WORKSPACE;
        pa::decode_ws_carve(workspace, num_seqs, num_q_heads, desc->head_dim, max_parts, a);
    }
    return from_cuda(pa::launch_decode(a, static_cast<cudaStream_t>(stream)));
}

int pa_decode_cascade_workspace_size(int32_t num_seqs, int32_t num_q_heads, int32_t max_blocks_per_seq,
                                     int32_t prefix_blocks, const pa_cache_desc *desc, size_t *bytes) {
    int rc = check_desc(desc);
    if (rc != PA_OK) return rc;
    if (!bytes || num_seqs < 0 || num_q_heads <= 0 || max_blocks_per_seq <= 0 ||
        max_blocks_per_seq > pa::kMaxBlocksPerSeq || prefix_blocks < 0 || prefix_blocks > max_blocks_per_seq)
        return PA_ERR_INVALID_ARG;
    *bytes = pa::cascade_ws_bytes(num_seqs, num_q_heads, desc->num_kv_heads, desc->head_dim, max_blocks_per_seq,
                                  prefix_blocks, desc->dtype == PA_DTYPE_FP8_E4M3);
    return PA_OK;
}

int pa_decode_cascade(void *out, const void *q, const void *k_cache, const void *v_cache,
                      const int32_t *block_tables, const int32_t *seq_lens, int32_t num_seqs,
                      int32_t max_blocks_per_seq, int32_t num_q_heads, float scale, const float *k_scale,
                      const float *v_scale, int32_t prefix_blocks, void *workspace, size_t workspace_bytes,
                      const pa_cache_desc *desc, pa_stream_t stream) {
    int rc = check_desc(desc);
    if (rc != PA_OK) return rc;
    if (num_seqs < 0 || num_seqs > kMaxSeqs || max_blocks_per_seq <= 0 ||
        max_blocks_per_seq > pa::kMaxBlocksPerSeq || num_q_heads <= 0)
        return PA_ERR_INVALID_ARG;
    if (prefix_blocks < 0 || prefix_blocks > max_blocks_per_seq) return PA_ERR_INVALID_ARG;
    if (prefix_blocks == 0)  // nothing shared: plain decode
        return pa_decode(out, q, k_cache, v_cache, block_tables, seq_lens, num_seqs, max_blocks_per_seq,
                         num_q_heads, scale, k_scale, v_scale, 0, workspace, workspace_bytes, desc, stream);
    if (num_q_heads % desc->num_kv_heads != 0) return PA_ERR_INVALID_ARG;
    if (desc->num_kv_heads > pa::kMaxDecodeKvHeads) return PA_ERR_UNSUPPORTED;
    const int G = num_q_heads / desc->num_kv_heads;
    if (G != 1 && G != 2 && G != 4 && G != 8) return PA_ERR_UNSUPPORTED;
    if (num_seqs == 0) return PA_OK;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !seq_lens) return PA_ERR_INVALID_ARG;
    if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache)) return PA_ERR_INVALID_ARG;
    const bool fp8 = desc->dtype == PA_DTYPE_FP8_E4M3;
    if (fp8 && (!k_scale || !v_scale)) return PA_ERR_INVALID_ARG;
    const size_t need = pa::cascade_ws_bytes(num_seqs, num_q_heads, desc->num_kv_heads, desc->head_dim,
                                             max_blocks_per_seq, prefix_blocks, fp8);
    if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255)) return PA_ERR_WORKSPACE;
    pa::DecodeArgs a{out, q, k_cache, v_cache, block_tables, seq_lens, num_seqs, max_blocks_per_seq,
                     num_q_heads, desc->num_kv_heads, desc->head_dim, desc->num_blocks, scale, k_scale, v_scale,
                     0, 0, nullptr, nullptr, nullptr, fp8, status_word_ptr(), prefix_blocks};
    return from_cuda(pa::launch_decode_cascade(a, workspace, static_cast<cudaStream_t>(stream)));
}

int pa_prefill_chunk(void *out, const void *q, const int32_t *cu_q_lens, const int32_t *prefix_lens,
                     const int32_t *block_tables, int32_t num_chunks, int32_t max_blocks_per_seq,
                     int32_t num_q_heads, int32_t max_q_len, int32_t total_q_tokens, const void *k_cache,
                     const void *v_cache, float scale, const float *k_scale, const float *v_scale,
                     const pa_cache_desc *desc, pa_stream_t stream) {
    int rc = check_desc(desc);
    if (rc != PA_OK) return rc;
    if (num_chunks < 0 || max_blocks_per_seq <= 0 || max_blocks_per_seq > pa::kMaxBlocksPerSeq ||
        num_q_heads <= 0 || max_q_len < 0 || total_q_tokens < 0)
        return PA_ERR_INVALID_ARG;
    if (num_q_heads % desc->num_kv_heads != 0) return PA_ERR_INVALID_ARG;
    const int G = num_q_heads / desc->num_kv_heads;
    if (G != 1 && G != 2 && G != 4 && G != 8) return PA_ERR_UNSUPPORTED;
    const bool fp8 = desc->dtype == PA_DTYPE_FP8_E4M3;
    if (fp8 && (!k_scale || !v_scale)) return PA_ERR_INVALID_ARG;
    if (num_chunks == 0 || max_q_len == 0 || total_q_tokens == 0) return PA_OK;
    if (!out || !q || !cu_q_lens || !prefix_lens || !block_tables || !k_cache || !v_cache) return PA_ERR_INVALID_ARG;
    if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache)) return PA_ERR_INVALID_ARG;
    pa::PrefillArgs a{out, q, cu_q_lens, prefix_lens, block_tables, num_chunks, max_blocks_per_seq, num_q_heads,
                      desc->num_kv_heads, desc->head_dim, max_q_len, total_q_tokens, desc->num_blocks, k_cache,
                      v_cache, scale, status_word_ptr()};
    if (fp8) {
        a.fp8 = true;
        a.k_scale = k_scale;
        a.v_scale = v_scale;
    }
    return from_cuda(pa::launch_prefill(a, static_cast<cudaStream_t>(stream)));
}

int pa_get_last_device_error(uint32_t *flags, pa_stream_t stream) {
    if (!flags) return PA_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    unsigned *p = status_word_ptr();
    if (!p) return PA_ERR_CUDA;
    unsigned v = 0;
    if (cudaStreamSynchronize(st) != cudaSuccess) return PA_ERR_CUDA;
    if (cudaMemcpy(&v, p, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) return PA_ERR_CUDA;
    if (cudaMemset(p, 0, sizeof v) != cudaSuccess) return PA_ERR_CUDA;
    *flags = v;
    return v ? PA_ERR_DEVICE : PA_OK;
}

}  // extern "C"
