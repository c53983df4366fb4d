// write_copy.cu -- slot-mapped KV write ("reshape_and_cache") and the
// copy-on-write block copy.
//
// Write: "Production Serving: Continuous Batching and PagedAttention", The
// Build, Step 4 "Implement the paged KV cache" -- each new token's K and V
// land in one slot of a 16-token page; the host allocator has already turned
// (page table, length) into a flat slot per token.
// Copy: "Continuous batching and PagedAttention", PagedAttention: KV cache
// memory -- blocks shared with copy-on-write are copied when a sharer
// diverges.
//
// Both are HBM-bound streams of 16-byte vectors: one thread moves one 16-byte
// chunk (8 bf16) per step, consecutive threads touch consecutive chunks, so
// every warp access is fully coalesced.
#include "common.cuh"
#include "kernels.h"

namespace pa {

// One thread per (token, kv head, 8-element chunk).  Source k/v are
// [T][Hkv][D] bf16, so the thread index is also the source chunk index.
template <bool FP8>
__global__ void __launch_bounds__(256) write_kv_kernel(const uint4 *__restrict__ k, const uint4 *__restrict__ v,
                                                       const int64_t *__restrict__ slots, int64_t n_chunks,
                                                       int Hkv, int D, int64_t num_blocks, void *__restrict__ kc,
                                                       void *__restrict__ vc, const float *__restrict__ ks,
                                                       const float *__restrict__ vs, unsigned *err) {
    pdl_trigger();
    pdl_wait();
    const int cpr = D / 8;  // chunks per (token, head) row
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n_chunks;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int c = (int)(i % cpr);
        const int64_t th = i / cpr;
        const int h = (int)(th % Hkv);
        const int64_t t = th / Hkv;
        const int64_t s = slots[t];
        if (s < 0) continue;
        const int64_t blk = s >> 4;
        if (blk >= num_blocks) {
            flag_error(err, PA_DEVERR_BAD_SLOT);
            continue;
        }
        const int64_t dst = (((blk * Hkv + h) << 4) + (s & 15)) * D + (int64_t)c * 8;  // element index
        const uint4 kw = k[i], vw = v[i];
        if constexpr (!FP8) {
            reinterpret_cast<uint4 *>(kc)[dst >> 3] = kw;
            reinterpret_cast<uint4 *>(vc)[dst >> 3] = vw;
        } else {
            // code = e4m3_rn_satfinite(x * rn(1/scale)): one fp32 multiply by
            // the correctly rounded reciprocal, then the hardware conversion
            // (nearest even, saturating).
            const float kinv = __frcp_rn(ks[h]), vinv = __frcp_rn(vs[h]);
            const uint32_t kin[4] = {kw.x, kw.y, kw.z, kw.w};
            const uint32_t vin[4] = {vw.x, vw.y, vw.z, vw.w};
            uint32_t kout[2], vout[2];
#pragma unroll
            for (int p = 0; p < 2; ++p) {
                uint32_t kk = 0, vv = 0;
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    float2 kf = bf16x2_to_float2(kin[2 * p + q]);
                    float2 vf = bf16x2_to_float2(vin[2 * p + q]);
                    kf = make_float2(__fmul_rn(kf.x, kinv), __fmul_rn(kf.y, kinv));
                    vf = make_float2(__fmul_rn(vf.x, vinv), __fmul_rn(vf.y, vinv));
                    const uint32_t k2 = __nv_cvt_float2_to_fp8x2(kf, __NV_SATFINITE, __NV_E4M3);
                    const uint32_t v2 = __nv_cvt_float2_to_fp8x2(vf, __NV_SATFINITE, __NV_E4M3);
                    kk |= (k2 & 0xffffu) << (16 * q);
                    vv |= (v2 & 0xffffu) << (16 * q);
                }
                kout[p] = kk;
                vout[p] = vv;
            }
            reinterpret_cast<uint2 *>(kc)[dst >> 3] = make_uint2(kout[0], kout[1]);
            reinterpret_cast<uint2 *>(vc)[dst >> 3] = make_uint2(vout[0], vout[1]);
        }
    }
}

// One CTA per (pair, cache); the block of all kv heads is one contiguous run
// of `vecs` 16-byte vectors.
__global__ void __launch_bounds__(256) copy_blocks_kernel(uint4 *__restrict__ kc, uint4 *__restrict__ vc,
                                                          const int32_t *__restrict__ pairs, int64_t num_blocks,
                                                          int64_t vecs, unsigned *err) {
    pdl_trigger();
    pdl_wait();
    const int64_t s = pairs[2 * blockIdx.x], d = pairs[2 * blockIdx.x + 1];
    if (s < 0 || d < 0 || s >= num_blocks || d >= num_blocks) {
        if (threadIdx.x == 0) flag_error(err, PA_DEVERR_BAD_PAIR);
        return;
    }
    uint4 *base = blockIdx.y == 0 ? kc : vc;
    const uint4 *src = base + s * vecs;
    uint4 *dst = base + d * vecs;
    for (int64_t i = threadIdx.x; i < vecs; i += blockDim.x) dst[i] = src[i];
}

cudaError_t launch_write_kv(const WriteArgs &a, cudaStream_t st) {
    const int64_t n_chunks = a.num_tokens * a.Hkv * (a.D / 8);
    if (n_chunks == 0) return cudaSuccess;
    const int threads = 256;
    int64_t blocks = (n_chunks + threads - 1) / threads;
    const int64_t cap = (int64_t)sm_count() * 8;  // 8 resident CTAs of 256 threads per SM, grid-stride beyond
    if (blocks > cap) blocks = cap;
    return launch_pdl(a.fp8 ? write_kv_kernel<true> : write_kv_kernel<false>, dim3((unsigned)blocks), dim3(threads),
                      0, st, (const uint4 *)a.k, (const uint4 *)a.v, a.slots, n_chunks, a.Hkv, a.D, a.num_blocks,
                      a.k_cache, a.v_cache, a.k_scale, a.v_scale, a.err);
}

cudaError_t launch_copy_blocks(const CopyArgs &a, cudaStream_t st) {
    if (a.num_pairs == 0) return cudaSuccess;
    const int64_t vecs = (int64_t)a.Hkv * 16 * a.D * a.elem_bytes / 16;
    dim3 grid((unsigned)a.num_pairs, 2);
    return launch_pdl(copy_blocks_kernel, grid, dim3(256), 0, st, (uint4 *)a.k_cache, (uint4 *)a.v_cache, a.pairs,
                      a.num_blocks, vecs, a.err);
}

}  // namespace pa
