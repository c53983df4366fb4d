/*
 * pa.h -- C ABI of libpa.so: paged-KV attention for continuous batching on
 * NVIDIA B200 (sm_100a).
 *
 * The operations follow three pages on continuous batching and
 * PagedAttention:
 *   [CB]  "Continuous batching and PagedAttention" (how-ai-works, chapter 7)
 *   [PS]  "Production Serving: Continuous Batching and PagedAttention"
 *         (llm-under-the-hood, project 17)
 *   [TR]  "Continuous batching and PagedAttention: serving many users from
 *         one GPU" (trefon.com notes)
 *
 * ---------------------------------------------------------------- layout --
 * KV cache: two device arrays, k_cache and v_cache, each
 *     [num_blocks][num_kv_heads][PA_BLOCK_SIZE = 16][head_dim]
 * row-major, element type bf16 or fp8 E4M3 (OCP "fn" variant).  Physical
 * block p of kv head h is one contiguous run of 16*head_dim elements
 * ([PS] "PagedAttention, the thing you build for memory": fixed 16-token
 * pages in one pre-allocated pool; [TR] "Fragmentation: PagedAttention").
 * The pages print two contradictory interleaved K/V layouts; this library
 * keeps K and V in separate arrays.
 *
 * Block table: int32 [num_seqs][max_blocks_per_seq]; entry [b][j] is the
 * physical block holding logical tokens 16j..16j+15 of sequence b ([PS]
 * Step 4 "Implement the paged KV cache": page table, logical block ->
 * physical page).  Entries at or past ceil(seq_len/16) are never read.
 *
 * Slot mapping: int64 [num_tokens]; slot = physical_block*16 + offset.
 * A negative slot marks a padding token that is skipped.
 *
 * Grouped-query attention: query head h reads kv head
 * floor(h * num_kv_heads / num_q_heads) (consecutive query heads share one
 * kv head).
 *
 * fp8 cache: one fp32 scale per kv head for K and one for V.  A stored code
 * c means the value e4m3(c) * scale[h].  Writing encodes
 *     c = e4m3_rn_satfinite(x * rn(1/scale[h]))
 * -- one IEEE fp32 multiply by the correctly rounded fp32 reciprocal, then
 * round-to-nearest-even to E4M3 with finite overflow and infinities clamped
 * to +-448.
 *
 * -------------------------------------------------------- conventions --
 * All array arguments are DEVICE pointers on the current device unless
 * stated otherwise.  The caller owns every buffer and the stream; the
 * library never allocates or frees memory and never synchronises, except
 * pa_get_last_device_error(), which reads a status word back.  Every call
 * enqueues its kernels on `stream` (a cudaStream_t; NULL = legacy default
 * stream) and returns at once.
 *
 * Every entry point returns a pa_status.  Argument errors are detected on
 * the host before anything is enqueued.  Metadata read on the device (block
 * ids, slots, lengths) is bounds-checked by the kernels: an out-of-range
 * value is skipped (treated as absent) and recorded in the device status
 * word, which pa_get_last_device_error() returns.
 */
#ifndef PA_H
#define PA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define PA_BLOCK_SIZE 16

/* Largest max_blocks_per_seq any call accepts (2^24 blocks = 2^28 tokens per
 * sequence); wider tables return PA_ERR_INVALID_ARG. */
#define PA_MAX_BLOCKS_PER_SEQ (1 << 24)

typedef enum pa_status {
    PA_OK = 0,
    PA_ERR_INVALID_ARG = -1, /* null pointer, bad size, Hq % Hkv != 0, block_size != 16 */
    PA_ERR_UNSUPPORTED = -2, /* valid but not built: head_dim not in {64,128}, group > 8, ... */
    PA_ERR_WORKSPACE = -3,   /* workspace missing or smaller than pa_decode_workspace_size() */
    PA_ERR_CUDA = -4,        /* a CUDA runtime call or kernel launch failed */
    PA_ERR_DEVICE = -5,      /* returned by pa_get_last_device_error when a kernel flagged bad metadata */
    PA_ERR_TIMEOUT = -6      /* reserved for host-side waits; device waits report PA_DEVERR_TIMEOUT */
} pa_status;

typedef enum pa_dtype {
    PA_DTYPE_BF16 = 0,
    PA_DTYPE_FP8_E4M3 = 1
} pa_dtype;

/* Bits of the device status word (pa_get_last_device_error). */
#define PA_DEVERR_BAD_BLOCK 0x1u  /* a block-table entry outside [0, num_blocks) was needed */
#define PA_DEVERR_BAD_SLOT 0x2u   /* a slot mapped past the last block */
#define PA_DEVERR_BAD_LEN 0x4u    /* seq_len < 0 or > 16 * max_blocks_per_seq (cascade: < 16 * prefix_blocks) */
#define PA_DEVERR_BAD_PAIR 0x8u   /* a copy pair outside [0, num_blocks) */
#define PA_DEVERR_TIMEOUT 0x10u   /* a bounded wait for an async copy or MMA gave up (results invalid) */
#define PA_DEVERR_LAYOUT 0x20u    /* prefill: the CTA's shared memory did not start on a 1 KB boundary (no output written) */

/* An opaque stream handle: pass a cudaStream_t. */
typedef void *pa_stream_t;

/* Shape of the paged cache.  block_size must be 16; head_dim 64 or 128;
 * dtype a pa_dtype. */
typedef struct pa_cache_desc {
    int64_t num_blocks;
    int32_t num_kv_heads;
    int32_t block_size;
    int32_t head_dim;
    int32_t dtype;
} pa_cache_desc;

/*
 * pa_write_kv -- slot-mapped write of new K/V ("reshape_and_cache").
 * [PS] Step 4 "Implement the paged KV cache": each new token's K and V land
 * in slot (length mod 16) of the sequence's current page; here the host
 * allocator has already turned that into one slot per token.
 *
 *   k, v          bf16 [num_tokens][num_kv_heads][head_dim], contiguous.
 *   slot_mapping  int64 [num_tokens]; slot < 0 skips the token.
 *   k_cache, v_cache  the cache (layout above), written in place.
 *   k_scale, v_scale  fp32 [num_kv_heads]; required for an fp8 cache,
 *                 ignored (may be NULL) for bf16.
 * For bf16 the cache receives the input bits unchanged.  Tokens must map to
 * distinct slots (otherwise which write wins is unspecified).
 * num_tokens == 0 enqueues nothing.
 */
int pa_write_kv(const void *k, const void *v, const int64_t *slot_mapping, int64_t num_tokens, void *k_cache,
                void *v_cache, const float *k_scale, const float *v_scale, const pa_cache_desc *desc,
                pa_stream_t stream);

/*
 * pa_copy_blocks -- copy-on-write block copy.
 * [CB] "PagedAttention: KV cache memory": blocks shared with copy-on-write
 * are copied when a sharer diverges; [TR] "Fragmentation: PagedAttention":
 * sequences with a common prefix point at the same blocks until they
 * diverge.
 *
 *   src_dst_pairs  int32 [num_pairs][2] = (src, dst) physical block ids.
 * Every element of block src (all kv heads, all 16 slots) is copied to block
 * dst in both caches.  Destinations must be distinct and no destination may
 * also be a source in the same call (pairs run concurrently).
 * Per-head fp8 scales are per cache, not per block: nothing else to copy.
 * num_pairs == 0 enqueues nothing.
 */
int pa_copy_blocks(void *k_cache, void *v_cache, const int32_t *src_dst_pairs, int32_t num_pairs,
                   const pa_cache_desc *desc, pa_stream_t stream);

/*
 * pa_decode_workspace_size -- bytes of device workspace pa_decode needs for
 * this shape (host function, no device work).  partition_tokens as for
 * pa_decode.  0 means no workspace is needed (every sequence fits one
 * partition).
 */
int pa_decode_workspace_size(int32_t num_seqs, int32_t num_q_heads, int32_t head_dim, int32_t max_blocks_per_seq,
                             int32_t partition_tokens, size_t *bytes);

/*
 * pa_decode -- paged decode attention, one query token per sequence.
 * [PS] Step 6 "Implement attention over paged storage", per query head:
 *     out[b][h] = sum_{t < seq_lens[b]} softmax_t(scale * q[b][h] . k_t) * v_t
 * with k_t, v_t stored at slot t%16 of block block_tables[b][t/16], kv head
 * floor(h*Hkv/Hq).  The sequence's own newest token must already be in the
 * cache (write first, then attend).
 *
 *   out           bf16 [num_seqs][num_q_heads][head_dim] (fp32 accumulation,
 *                 rounded to nearest-even bf16 once at the end).
 *   q             bf16 [num_seqs][num_q_heads][head_dim].
 *   block_tables  int32 [num_seqs][max_blocks_per_seq].
 *   seq_lens      int32 [num_seqs]; 0 gives an all-zero output row.
 *   scale         softmax scale (typically 1/sqrt(head_dim)).
 *   k_scale, v_scale  fp32 [num_kv_heads] for an fp8 cache, else ignored.
 *   partition_tokens  how a sequence's tokens are split across warps
 *                 (split-K; the pieces are combined by a log-sum-exp merge
 *                 kernel that the same call enqueues):
 *                 0  -- balanced: the (sequence, kv head, block) work of the
 *                       whole batch is cut into equal contiguous shares, one
 *                       per resident warp, so every SM streams the same
 *                       number of bytes whatever the length mix (fastest;
 *                       split points depend on the batch, so the last bits
 *                       of a result can differ between batch compositions);
 *                 16..2048, a multiple of 16 -- fixed partitions of that
 *                       many tokens: split points depend only on token
 *                       positions, so each sequence's result is bitwise
 *                       independent of the rest of the batch.
 *   workspace     device scratch of at least pa_decode_workspace_size()
 *                 bytes, 256-byte aligned: the split-K pieces (fp32
 *                 outputs, log2-sum-exps and piece counts) that a second
 *                 kernel, enqueued by the same call, merges.  Every call
 *                 writes all it reads, so it needs no initialisation and
 *                 keeps nothing between calls.  Calls that share one
 *                 workspace must not overlap on the GPU.
 * num_seqs must be in [0, 2048] (0 enqueues nothing); num_kv_heads <= 128;
 * num_q_heads / num_kv_heads in {1,2,4,8}.  With an fp8 cache and 8 q heads
 * per kv head the products run on the tensor cores (f16 operands: E4M3
 * exactly, q scaled by a power of two; fp32 accumulation), otherwise in fp32
 * on the CUDA cores.
 */
int pa_decode(void *out, const void *q, const void *k_cache, const void *v_cache, const int32_t *block_tables,
              const int32_t *seq_lens, int32_t num_seqs, int32_t max_blocks_per_seq, int32_t num_q_heads,
              float scale, const float *k_scale, const float *v_scale, int32_t partition_tokens,
              void *workspace, size_t workspace_bytes, const pa_cache_desc *desc, pa_stream_t stream);

/*
 * pa_decode_cascade -- pa_decode for a batch whose sequences all begin with
 * the same prefix_blocks physical blocks (a shared prompt; sequences forked
 * from one parent).  [PS] Step 6 defines the result (per query head, over
 * every cached token of the sequence), which equals pa_decode's; the pages
 * state that such blocks are shared ("Production Serving: Continuous
 * Batching and PagedAttention", Step 4; "Continuous batching and
 * PagedAttention", PagedAttention: KV cache memory) but give no kernel for
 * reading them once, so the split below is this library's.
 *
 * The keys of each sequence split into the shared prefix [0, 16*prefix_blocks)
 * and its own suffix.  The prefix is attended once per kv head for every
 * sequence at the same time (its K/V read once, all sequences' queries as
 * the rows of a tensor-core attention, cut into up to 4 key ranges so that
 * it fills the SMs; an fp8 prefix is first widened to bf16 exactly, into the
 * workspace), each suffix by the decode kernel, and all pieces are combined
 * by the split-K log-sum-exp merge.  Four launches (three for bf16), each a
 * programmatic dependent of the one before, all on `stream`.
 *
 * Arguments as pa_decode (balanced split; partition_tokens is not taken),
 * plus:
 *   prefix_blocks  number of leading block-table entries that every row
 *                  shares: entries 0..prefix_blocks-1 of every row must equal
 *                  those of row 0 (not checked; row 0's are used).  Range
 *                  [0, max_blocks_per_seq] (else PA_ERR_INVALID_ARG); 0 runs
 *                  pa_decode.  Every seq_lens[b] must be >= 16*prefix_blocks
 *                  (checked on the device: such a row is flagged
 *                  PA_DEVERR_BAD_LEN and gets the prefix's attention alone).
 *   workspace      device memory owned by the caller, at least
 *                  pa_decode_cascade_workspace_size() bytes, 256-byte
 *                  aligned (else PA_ERR_WORKSPACE), no initialisation needed
 *                  (every call writes all it reads).  Calls sharing one
 *                  workspace must not overlap on the GPU.
 * head_dim 64 or 128 (else PA_ERR_UNSUPPORTED); num_q_heads / num_kv_heads
 * in {1,2,4,8}; bf16 or fp8 E4M3 cache (fp8 needs k_scale, v_scale).
 *
 * pa_decode_cascade_workspace_size: bytes for num_seqs rows of num_q_heads
 * heads, tables of max_blocks_per_seq entries and prefix_blocks shared
 * blocks (an upper bound for any smaller num_seqs); host only.
 */
int pa_decode_cascade_workspace_size(int32_t num_seqs, int32_t num_q_heads, int32_t max_blocks_per_seq,
                                     int32_t prefix_blocks, const pa_cache_desc *desc, size_t *bytes);

int pa_decode_cascade(void *out, const void *q, const void *k_cache, const void *v_cache,
                      const int32_t *block_tables, const int32_t *seq_lens, int32_t num_seqs,
                      int32_t max_blocks_per_seq, int32_t num_q_heads, float scale, const float *k_scale,
                      const float *v_scale, int32_t prefix_blocks, void *workspace, size_t workspace_bytes,
                      const pa_cache_desc *desc, pa_stream_t stream);

/*
 * pa_prefill_chunk -- causal attention of prompt chunks over their paged
 * prefixes (chunked prefill).
 * [CB] "How the scheduler works": a long prompt is cut into chunks that fit
 * the per-step token budget; [TR] "Prefill gets in the way": chunks are
 * interleaved with decode steps.
 *
 *   out, q        bf16 [total_q][num_q_heads][head_dim].
 *   cu_q_lens     int32 [num_chunks+1]: chunk c owns rows
 *                 cu_q_lens[c]..cu_q_lens[c+1]-1.
 *   prefix_lens   int32 [num_chunks]: tokens already in the cache before the
 *                 chunk.  Row i of chunk c sits at position prefix_lens[c]+i
 *                 and attends keys 0..prefix_lens[c]+i inclusive.
 *   block_tables  int32 [num_chunks][max_blocks_per_seq].
 *   max_q_len     host upper bound on any chunk's length (sizes the grid).
 *   total_q_tokens  rows of q and out (= cu_q_lens[num_chunks]); chunks
 *                 reaching past it are rejected on the device.
 *   k_scale, v_scale  fp32 [num_kv_heads] for an fp8 cache (required;
 *                 PA_ERR_INVALID_ARG without them), ignored for bf16.
 * The chunk's own K/V must already be in the cache (pa_write_kv first).
 * bf16 cache: bf16 MMA operands.  fp8 E4M3 cache: each K/V tile is widened
 * exactly to f16 in shared memory on its way to the tensor cores, a query
 * row is scaled by a power of two into f16 range (exact for components
 * within 2^-28 of the row's largest), P enters P.V as f16; fp32
 * accumulation throughout.  head_dim 64 or 128; num_q_heads / num_kv_heads
 * in {1,2,4,8}.
 */
int pa_prefill_chunk(void *out, const void *q, const int32_t *cu_q_lens, const int32_t *prefix_lens,
                     const int32_t *block_tables, int32_t num_chunks, int32_t max_blocks_per_seq,
                     int32_t num_q_heads, int32_t max_q_len, int32_t total_q_tokens, const void *k_cache,
                     const void *v_cache, float scale,
                     const float *k_scale, const float *v_scale, const pa_cache_desc *desc, pa_stream_t stream);

/*
 * pa_decode_noalloc -- pa_decode for callers that cannot allocate device
 * memory.  There is no counterpart of this entry point in the source pages.
 *
 * Some callers cannot call cudaMalloc: a plugin hosted by a serving engine
 * whose memory pool has already claimed the device (engines typically
 * reserve nearly all HBM for the KV cache at start-up, so a late cudaMalloc
 * fails or fragments the pool), or an integration that must not trigger the
 * implicit device synchronisation cudaMalloc/cudaFree can cause.  This
 * variant takes the same arguments as pa_decode minus the workspace: its
 * split-K scratch lives in a fixed device array inside libpa.so,
 * PA_DECODE_NOALLOC_SCRATCH_BYTES (16 MiB) large, which every GPU that loads
 * the library holds until the process exits.  Nothing is allocated: no
 * cudaMalloc, cudaFree or allocating library routine is called.
 *
 *   - A shape whose pa_decode_workspace_size() exceeds the array returns
 *     PA_ERR_WORKSPACE before anything is enqueued (use pa_decode with a
 *     caller workspace, or fixed partitions, which need less scratch).
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress, once per device, with that device current);
 *     make that first call before any stream capture.
 *   - Every call on a device shares the one array and it keeps the last
 *     call's contents; a call writes every part it reads, so nothing is
 *     cleared between calls.  Calls that overlap on the GPU (on different
 *     streams without ordering) race on the array and give wrong results:
 *     order them.
 */
#define PA_DECODE_NOALLOC_SCRATCH_BYTES (16u << 20)

int pa_decode_noalloc(void *out, const void *q, const void *k_cache, const void *v_cache,
                      const int32_t *block_tables, const int32_t *seq_lens, int32_t num_seqs,
                      int32_t max_blocks_per_seq, int32_t num_q_heads, float scale, const float *k_scale,
                      const float *v_scale, int32_t partition_tokens, const pa_cache_desc *desc,
                      pa_stream_t stream);

/*
 * pa_get_last_device_error -- synchronise `stream`, return the device status
 * word (PA_DEVERR_* bits, 0 if clean) in *flags and clear it.  Returns
 * PA_ERR_DEVICE if any bit was set, PA_OK otherwise.
 */
int pa_get_last_device_error(uint32_t *flags, pa_stream_t stream);

/* Human-readable name of a pa_status value (static string). */
const char *pa_status_string(int status);

/* Library version as an integer (major*10000 + minor*100 + patch): 300 =
 * 0.3.0, which adds chunked prefill over an fp8 cache and the
 * PA_MAX_BLOCKS_PER_SEQ bound to 0.2.0 (pa_decode_cascade,
 * pa_decode_noalloc). */
int pa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PA_H */
