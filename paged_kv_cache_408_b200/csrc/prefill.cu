// prefill.cu -- causal chunked-prefill attention over a paged prefix, on the
// sm_100a tensor cores (tcgen05, TMEM accumulators, TMA tensor copies).
//
// What is computed ("Continuous batching and PagedAttention", How the
// scheduler works: chunked prefill; "Continuous batching and
// PagedAttention: serving many users from one GPU", Prefill gets in the
// way): row i of chunk c sits at position prefix_lens[c] + i and attends,
// per query head, to keys 0 .. prefix_lens[c] + i of its sequence through
// the block table -- the prefix already in the cache and the chunk's own
// keys, written there first.
//
// Design:
//  * One CTA (4 warps) per (chunk, kv head, tile of 128/G query positions).
//    Its 128 accumulator rows are those positions x the G query heads of
//    the kv head (row = position*G + head), so every K/V tile is fetched
//    once per GQA group.
//  * K and V are streamed in tiles of 128 keys = 8 paged blocks.  Each
//    block of one kv head is a 16-row x D slab of the cache; warp 0 gathers
//    the 8 slabs through the block table with 2-D TMA tensor copies
//    (64-column boxes, 128-byte swizzle, no multicast) straight into the
//    operand layout of the tensor cores.  K and V buffers are double
//    buffered with their own mbarriers.
//  * S = Q K^T (M=128, N=128 keys, K=D) and O += P V (M=128, N=D, K=128
//    keys) are tcgen05.mma kind::f16 (bf16 in, fp32 accumulate) issued by
//    one thread; S and O live in TMEM.  Softmax reads S from TMEM (one
//    thread per row), applies the causal mask, moves the running max only
//    when it grows by more than 8 (log2 units) -- then it rescales its O
//    row in TMEM -- and writes P as bf16 to shared memory for the second
//    MMA.  The P.V MMA of tile j-1 overlaps S and softmax of tile j.
//  * Key rows past the sequence end in the last tile are zeroed in shared
//    memory before P.V, so stale cache contents can never reach the output.
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace pa {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;

template <int D_, int G_>
struct PCfg {
    static constexpr int D = D_, G = G_;
    static constexpr int M = 128;                 // accumulator rows per CTA
    static constexpr int QPOS = M / G;            // query positions per CTA
    static constexpr int KT = 128;                // keys per K/V tile
    static constexpr int NATOM = D / 64;          // 128-byte column atoms along D
    static constexpr int ATOM = 128 * 128;        // bytes of one atom column of a 128-row tile
    static constexpr int TILE = NATOM * ATOM;     // bytes of a Q, K or V tile
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = TILE;            // two K tiles
    static constexpr int OFF_V = 3 * TILE;        // two V tiles
    static constexpr int OFF_P = 5 * TILE;        // P: 128 rows x 128 keys (two atoms)
    static constexpr int OFF_BAR = OFF_P + 2 * ATOM;
    static constexpr int SMEM = OFF_BAR + 128 + 1024;  // barriers + alignment slack
    static constexpr int NT = 128;
    static constexpr uint32_t TMEM_COLS = 256;
    static constexpr uint32_t COL_S = 0, COL_O = 128;
    static constexpr uint32_t TX_BYTES = 8 * NATOM * 16 * 128;  // one K or V tile
    static_assert(M % G == 0, "group must divide 128");
};

template <class C>
__global__ void __launch_bounds__(C::NT, 1)
    prefill_kernel(const PrefillArgs a, const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV) {
    constexpr int D = C::D, G = C::G;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t *sQ = smem + C::OFF_Q;
    uint8_t *sK = smem + C::OFF_K;
    uint8_t *sV = smem + C::OFF_V;
    uint8_t *sP = smem + C::OFF_P;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint64_t *barK = bars, *barV = bars + 2, *barS = bars + 4, *barO = bars + 5;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 6);

    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const int c = blockIdx.z, kvh = blockIdx.y;
    const int i0 = blockIdx.x * C::QPOS;
    pdl_trigger();
    pdl_wait();
    const int q_start = a.cu_q[c];
    const int clen = a.cu_q[c + 1] - q_start;
    const int pfx = a.prefix_lens[c];
    if (i0 >= clen) return;  // this tile lies past the chunk (uniform per CTA)
    const int L = pfx + clen;
    if (clen < 0 || pfx < 0 || L > a.max_blocks * 16 || q_start < 0 || q_start + clen > a.total_q) {
        if (tid == 0) flag_error(a.err, PA_DEVERR_BAD_LEN);
        return;
    }
    const int nvalid = min(C::QPOS, clen - i0);
    const int n_keys = pfx + i0 + nvalid;  // keys the last valid row sees
    const int ntiles = (n_keys + C::KT - 1) / C::KT;
    const int nalloc = (L + 15) >> 4;     // blocks of the sequence
    const int32_t *bt = a.block_tables + (size_t)c * a.max_blocks;

    if (w == 0) tmem_alloc(tmem_slot, C::TMEM_COLS);
    if (tid == 0) {
        for (int i = 0; i < 6; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
    }

    // ---- Q tile: row t = (position t / G, head t % G), 128-byte swizzle
    const int my_i = tid / G, my_h = tid % G;
    const bool row_valid = my_i < nvalid;
    {
        const __nv_bfloat16 *src = static_cast<const __nv_bfloat16 *>(a.q) +
                                   ((size_t)(q_start + i0 + my_i) * a.Hq + (size_t)kvh * G + my_h) * D;
#pragma unroll
        for (int ch = 0; ch < D / 8; ++ch) {
            const uint4 v = row_valid ? *reinterpret_cast<const uint4 *>(src + ch * 8) : make_uint4(0, 0, 0, 0);
            const int at = ch / 8, cc = ch % 8;
            *reinterpret_cast<uint4 *>(sQ + at * C::ATOM + tid * 128 + ((cc ^ (tid & 7)) * 16)) = v;
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // ---- warp 0 gathers the 8 blocks of a K or V tile through the block table
    auto issue = [&](int j, bool is_v) {
        uint64_t *bar = is_v ? &barV[j & 1] : &barK[j & 1];
        uint8_t *dst = (is_v ? sV : sK) + (j & 1) * C::TILE;
        const CUtensorMap *map = is_v ? &tmV : &tmK;
        if (lane == 0) mbar_arrive_expect_tx(bar, C::TX_BYTES);
        __syncwarp();
        if (lane < 8) {
            const int lb = min(j * 8 + lane, nalloc - 1);  // past the end: a valid block, masked later
            int phys = bt[lb];
            if (phys < 0 || phys >= a.num_blocks) {
                flag_error(a.err, PA_DEVERR_BAD_BLOCK);
                phys = 0;
            }
            const int row = (phys * a.Hkv + kvh) * 16;
#pragma unroll
            for (int at = 0; at < C::NATOM; ++at) tma_load_2d(dst + at * C::ATOM + lane * 16 * 128, map, at * 64, row, bar);
        }
    };
    if (w == 0) {
        issue(0, false);
        issue(0, true);
        if (ntiles > 1) {
            issue(1, false);
            issue(1, true);
        }
    }

    const int pos = pfx + i0 + my_i;
    const float sl2 = a.scale * kLog2e;
    const uint32_t lane_base = tmem + ((uint32_t)(w * 32) << 16);
    constexpr uint32_t idS = idesc_bf16_f32(128, C::KT, false);
    constexpr uint32_t idO = idesc_bf16_f32(128, D, true);
    float m = -INFINITY, l = 0.f;
    bool dead = false;

    for (int j = 0; j < ntiles && !dead; ++j) {
        const int b = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        // ---- S = Q K^T
        bool ok = mbar_wait(&barK[b], ph);
        if (tid == 0 && ok) {
            tc_fence_after();
            const uint32_t q0 = smem_addr(sQ), k0 = smem_addr(sK + b * C::TILE);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t off = (kk / 4) * C::ATOM + (kk % 4) * 32;
                tc_mma_bf16(tmem + C::COL_S, smem_desc_sw128(q0 + off, 16, 1024), smem_desc_sw128(k0 + off, 16, 1024),
                            idS, kk > 0);
            }
            tc_commit(barS);
        }
        ok = mbar_wait(barS, j & 1) && ok;
        tc_fence_after();
        if (w == 0 && j + 2 < ntiles) issue(j + 2, false);  // K buffer b is free again

        // ---- softmax of this thread's row
        float s[C::KT];
#pragma unroll
        for (int q = 0; q < C::KT / 32; ++q) {
            float t32[32];
            tmem_ld32(lane_base + C::COL_S + 32 * q, t32);
#pragma unroll
            for (int e = 0; e < 32; ++e) s[32 * q + e] = t32[e];
        }
        tmem_wait_ld();
        const int kv0 = j * C::KT;
        float mt = -INFINITY;
#pragma unroll
        for (int e = 0; e < C::KT; ++e) {
            s[e] = (row_valid && kv0 + e <= pos) ? s[e] * sl2 : -INFINITY;
            mt = fmaxf(mt, s[e]);
        }
        const bool rescale = mt > m + kRescaleThreshold;
        float alpha = 1.f;
        if (rescale) {
            alpha = (m == -INFINITY) ? 0.f : ex2(m - mt);
            m = mt;
            l *= alpha;
        }
        uint32_t pk[C::KT / 2];
        float sum = 0.f;
#pragma unroll
        for (int e = 0; e < C::KT; e += 2) {
            const float p0 = (s[e] == -INFINITY) ? 0.f : ex2(s[e] - m);
            const float p1 = (s[e + 1] == -INFINITY) ? 0.f : ex2(s[e + 1] - m);
            sum += p0 + p1;
            const __nv_bfloat162 bb = __floats2bfloat162_rn(p0, p1);
            pk[e / 2] = *reinterpret_cast<const uint32_t *>(&bb);
        }
        l += sum;

        // ---- P.V of the previous tile must be done before P and O are touched
        if (j > 0) {
            ok = mbar_wait(barO, (j - 1) & 1) && ok;
            tc_fence_after();
            if (w == 0 && j + 1 < ntiles) issue(j + 1, true);  // its V buffer is free again
        }
        // tcgen05.ld/st are warp-collective: rescale if any row of the warp needs it
        // (rows that do not keep alpha == 1)
        if (__any_sync(0xffffffffu, rescale) && j > 0) {
#pragma unroll
            for (int q = 0; q < D / 32; ++q) {
                float o[32];
                tmem_ld32(lane_base + C::COL_O + 32 * q, o);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) o[e] *= alpha;
                tmem_st32(lane_base + C::COL_O + 32 * q, o);
            }
            tmem_wait_st();
        }
#pragma unroll
        for (int ch = 0; ch < C::KT / 8; ++ch) {
            const int at = ch / 8, cc = ch % 8;
            *reinterpret_cast<uint4 *>(sP + at * C::ATOM + tid * 128 + ((cc ^ (tid & 7)) * 16)) =
                make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
        }
        // ---- V tile: zero key rows past the sequence end (stale cache slots)
        ok = mbar_wait(&barV[b], ph) && ok;
        if (kv0 + tid >= L) {
            uint8_t *vrow = sV + b * C::TILE + tid * 128;
#pragma unroll
            for (int at = 0; at < C::NATOM; ++at)
#pragma unroll
                for (int cc = 0; cc < 8; ++cc)
                    *reinterpret_cast<uint4 *>(vrow + at * C::ATOM + cc * 16) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        dead = __syncthreads_or(!ok) != 0;
        if (dead) break;
        // ---- O += P V
        if (tid == 0) {
            tc_fence_after();
            const uint32_t p0 = smem_addr(sP), v0 = smem_addr(sV + b * C::TILE);
#pragma unroll
            for (int kk = 0; kk < C::KT / 16; ++kk) {
                const uint32_t aoff = (kk / 4) * C::ATOM + (kk % 4) * 32;
                tc_mma_bf16(tmem + C::COL_O, smem_desc_sw128(p0 + aoff, 16, 1024),
                            smem_desc_sw128(v0 + kk * 16 * 128, C::ATOM, 1024), idO, j > 0 || kk > 0);
            }
            tc_commit(barO);
        }
    }

    if (!dead) {
        // ---- epilogue: O / l, bf16, one row per thread
        const bool ok = mbar_wait(barO, (ntiles - 1) & 1);
        tc_fence_after();
        if (!ok && tid == 0) flag_error(a.err, PA_DEVERR_TIMEOUT);
        __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(a.out) +
                             ((size_t)(q_start + i0 + my_i) * a.Hq + (size_t)kvh * G + my_h) * D;
        const float inv = (l > 0.f) ? 1.f / l : 0.f;
#pragma unroll
        for (int q = 0; q < D / 32; ++q) {
            float o[32];
            tmem_ld32(lane_base + C::COL_O + 32 * q, o);
            tmem_wait_ld();
            if (row_valid) {
#pragma unroll
                for (int e = 0; e < 32; e += 8) {
                    uint32_t wds[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const __nv_bfloat162 bb = __floats2bfloat162_rn(o[e + 2 * u] * inv, o[e + 2 * u + 1] * inv);
                        wds[u] = *reinterpret_cast<const uint32_t *>(&bb);
                    }
                    *reinterpret_cast<uint4 *>(dst + 32 * q + e) = make_uint4(wds[0], wds[1], wds[2], wds[3]);
                }
            }
        }
    } else if (tid == 0) {
        flag_error(a.err, PA_DEVERR_TIMEOUT);
        // let MMAs already issued finish before their TMEM is released
        mbar_wait(barO, 0, 100000000ull);
        mbar_wait(barO, 1, 100000000ull);
    }
    tc_fence_before();
    __syncthreads();
    if (w == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// ---- host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// The cache seen as a 2-D bf16 tensor [num_blocks*Hkv*16 rows][D]; a box is
// 16 rows (one block of one kv head) x 64 columns, 128-byte swizzled.
bool cache_map(CUtensorMap *map, const void *base, int64_t rows, int D) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
    const cuuint32_t box[2] = {64, 16};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <class C>
cudaError_t run_prefill(const PrefillArgs &a, cudaStream_t st) {
    static std::mutex mu;
    static bool ready[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (!ready[dev]) {
            e = cudaFuncSetAttribute(prefill_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
            if (e != cudaSuccess) return e;
            ready[dev] = true;
        }
    }
    CUtensorMap tk, tv;
    const int64_t rows = a.num_blocks * a.Hkv * 16;
    if (!cache_map(&tk, a.k_cache, rows, C::D) || !cache_map(&tv, a.v_cache, rows, C::D)) return cudaErrorInvalidValue;
    dim3 grid((a.max_q_len + C::QPOS - 1) / C::QPOS, a.Hkv, a.n_chunks);
    return launch_pdl(prefill_kernel<C>, grid, dim3(C::NT), C::SMEM, st, a, tk, tv);
}

template <int D>
cudaError_t prefill_by_group(const PrefillArgs &a, cudaStream_t st) {
    switch (a.Hq / a.Hkv) {
        case 1: return run_prefill<PCfg<D, 1>>(a, st);
        case 2: return run_prefill<PCfg<D, 2>>(a, st);
        case 4: return run_prefill<PCfg<D, 4>>(a, st);
        case 8: return run_prefill<PCfg<D, 8>>(a, st);
        default: return cudaErrorNotSupported;
    }
}

}  // namespace

cudaError_t launch_prefill(const PrefillArgs &a, cudaStream_t st) {
    if (a.D == 128) return prefill_by_group<128>(a, st);
    if (a.D == 64) return prefill_by_group<64>(a, st);
    return cudaErrorNotSupported;
}

}  // namespace pa
