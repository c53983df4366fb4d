// copy_rates.cu -- how fast a K/V tile can be moved into shared memory on this
// GPU: 148 CTAs (one per SM) each fill a ring of 32 KB tiles, a tile being 8
// random 16-row blocks of an L2-resident 64 MB buffer laid out like a bf16
// cache with head_dim 128 (16 rows x 256 bytes per block), by
//   mode 0: 2-D TMA tensor copies of 16 rows x 128 bytes, 128-byte swizzle
//           (the prefill kernel's K/V loads);
//   mode 1: 1-D bulk copies of a block's 4 KB;
//   mode 2: 1-D bulk copies of 2 KB;
//   LSU:    16-byte cp.async from 128 threads;
//   pair:   clusters of 2 CTAs walking the same tiles, each loading the whole
//           tile by TMA (pair mode 0), or loading half by TMA and pushing it
//           into the other CTA's slot with a shared::cta -> shared::cluster
//           bulk copy (pair mode 1).
// Prints bytes per clock per SM.  Every wait is bounded (2 s), every copy
// stays inside its buffer and its ring slot.
// Build and run: nvcc -gencode arch=compute_100a,code=sm_100a -O3 -std=c++17
//   --expt-relaxed-constexpr -I include -o /tmp/copy_rates tests/gpu_checks/copy_rates.cu -lcuda
//   && /tmp/copy_rates
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <cstdio>
#include <cstdint>
#include <vector>
#include "../../paged_kv_cache_408_b200/csrc/common.cuh"
#include "../../paged_kv_cache_408_b200/csrc/tc.cuh"
using namespace pa;

constexpr int TILE = 32768;
__global__ void __launch_bounds__(32, 1) bench(const __grid_constant__ CUtensorMap tm, const uint8_t *base, int nblk, int S,
                                               int mode, int iters, long long *out, unsigned *err) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + S * TILE);
    const int lane = threadIdx.x;
    if (lane == 0) {
        for (int i = 0; i < S; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
    }
    __syncwarp();
    const uint64_t dl = wait_deadline();
    uint32_t seed = blockIdx.x * 7919u + 17u;
    long long t0 = clock64();
    bool ok = true;
    int issued = 0;
    for (int it = 0; it < iters && ok; ++it) {
        const int s = it % S;
        if (it >= S) ok = mbar_wait(&bars[s], ((it / S) - 1) & 1, dl);
        if (!ok) break;
        issued = it + 1;
        if (lane == 0) mbar_arrive_expect_tx(&bars[s], TILE);
        __syncwarp();
        seed = seed * 1664525u + 1013904223u;
        if (lane < 8) {
            const int blk = (int)(((seed >> 8) + (unsigned)lane * 2654435761u) % (unsigned)nblk);  // 16-row block of this lane
            uint8_t *dst = smem + s * TILE + lane * 16 * 128;
            if (mode == 0) {  // two 2-D boxes of 16 rows x 64 bf16 (128B swizzle), like the prefill loader
                tma_load_2d(dst, &tm, 0, blk * 16, &bars[s]);
                tma_load_2d(dst + 16384, &tm, 64, blk * 16, &bars[s]);
            } else if (mode == 1) {  // one 1-D bulk copy of the block's 4 KB
                bulk_g2s(smem + s * TILE + lane * 4096, base + (size_t)blk * 4096, 4096, &bars[s]);
            } else {  // two 1-D bulk copies of 2 KB
                bulk_g2s(smem + s * TILE + lane * 4096, base + (size_t)blk * 4096, 2048, &bars[s]);
                bulk_g2s(smem + s * TILE + lane * 4096 + 2048, base + (size_t)blk * 4096 + 2048, 2048, &bars[s]);
            }
        }
        __syncwarp();
    }
    // drain
    const uint64_t dd = ok ? dl : drain_deadline();
    for (int s = 0; s < S && s < issued; ++s) {
        const int last = s + S * ((issued - 1 - s) / S);
        if (!mbar_wait(&bars[s], (last / S) & 1, dd)) ok = false;
    }
    long long t1 = clock64();
    if (lane == 0) {
        out[blockIdx.x] = t1 - t0;
        if (!ok) atomicOr(err, 1u);
    }
}

// LSU path: 128 threads copy a 32 KB tile of 8 random blocks with cp.async (16 B each), then
// cp.async.wait_all + bar per tile (ring of S tiles, the wait trails by S-1 tiles via wait_group).
__global__ void __launch_bounds__(128, 1) bench_lsu(const uint8_t *base, int nblk, int S, int iters, long long *out) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int tid = threadIdx.x;
    uint32_t seed = blockIdx.x * 7919u + 17u;
    long long t0 = clock64();
    for (int it = 0; it < iters; ++it) {
        const int s = it % S;
        seed = seed * 1664525u + 1013904223u;
        // 2048 chunks of 16 B per tile; thread tid takes chunks tid + 128 k
#pragma unroll 4
        for (int k = 0; k < 16; ++k) {
            const int ch = tid + 128 * k, b = ch >> 8, within = ch & 255;  // block b of the tile, 16-B chunk in its 4 KB
            const int blk = (int)(((seed >> 8) + (unsigned)b * 2654435761u) % (unsigned)nblk);
            const uint8_t *src = base + (size_t)blk * 4096 + within * 16;
            const uint32_t dst = smem_addr(smem + s * TILE + ch * 16);
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
        if (S == 1) asm volatile("cp.async.wait_group 0;" ::: "memory");
        else if (S == 2) asm volatile("cp.async.wait_group 1;" ::: "memory");
        else asm volatile("cp.async.wait_group 3;" ::: "memory");
        __syncthreads();
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncthreads();
    long long t1 = clock64();
    if (tid == 0) out[blockIdx.x] = t1 - t0;
}

constexpr int HALF = 16384;

__device__ __forceinline__ uint32_t cluster_rank() { uint32_t r; asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r)); return r; }
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t map_peer(uint32_t saddr, uint32_t rank) {
    uint32_t r; asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank)); return r;
}
__device__ __forceinline__ void remote_arrive(uint32_t remote_bar) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(remote_bar) : "memory");
}
__device__ __forceinline__ void push_to_peer(uint32_t dst_remote, const void *src, uint32_t bytes, uint32_t remote_bar) {
    asm volatile("cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst_remote),
                 "r"(smem_addr(src)), "r"(bytes), "r"(remote_bar) : "memory");
}

// mode 0: whole tile by TMA (16 boxes) per CTA; mode 1: half by TMA + push of the half to the peer
__global__ void __launch_bounds__(32, 1) bench_pair(const __grid_constant__ CUtensorMap tm, int nblk, int S, int mode, int iters,
                                               long long *out, unsigned *err) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + S * TILE);  // [S]: own half (arrive) + pushed half (tx) / whole tile
    uint64_t *mine = full + S;                                       // [S]: own TMA half landed
    uint64_t *pfree = mine + S;                                      // [S]: the peer's slot is free for my push
    const int lane = threadIdx.x;
    const uint32_t rank = cluster_rank(), peer = rank ^ 1u;
    if (lane == 0) {
        for (int i = 0; i < S; ++i) {
            mbar_init(&full[i], mode ? 2 : 1);
            mbar_init(&mine[i], 1);
            mbar_init(&pfree[i], 1);
        }
        fence_mbar_init();
    }
    __syncwarp();
    cluster_sync();  // barriers of both CTAs initialised before any remote access
    const uint64_t dl = wait_deadline();
    uint32_t seed = (blockIdx.x >> 1) * 7919u + 17u;  // both CTAs of a pair walk the same tiles
    long long t0 = clock64();
    bool ok = true;
    int issued = 0;
    for (int it = 0; it < iters && ok; ++it) {
        const int s = it % S, use = it / S;
        // the slot's previous tile: consumed (here: landed) before it is refilled
        if (use > 0) ok = mbar_wait(&full[s], (use - 1) & 1, dl);
        if (!ok) break;
        if (mode == 1) {
            if (lane == 0) remote_arrive(map_peer(smem_addr(&pfree[s]), peer));  // my slot s is free for the peer
            // the peer's slot s is free for my push; the peer signals use u only once its slot's
            // previous tile (with my previous push) has landed, so my previous push has also
            // finished reading my slot before my TMA below overwrites it
            ok = mbar_wait(&pfree[s], use & 1, dl);
            if (!ok) break;
        }
        issued = it + 1;
        seed = seed * 1664525u + 1013904223u;
        uint8_t *slot = smem + s * TILE;
        if (mode == 0) {
            if (lane == 0) mbar_arrive_expect_tx(&full[s], TILE);
            __syncwarp();
            if (lane < 8) {
                const int blk = (int)(((seed >> 8) + (unsigned)lane * 2654435761u) % (unsigned)nblk);
                tma_load_2d(slot + lane * 2048, &tm, 0, blk * 16, &full[s]);
                tma_load_2d(slot + 16384 + lane * 2048, &tm, 64, blk * 16, &full[s]);
            }
            __syncwarp();
        } else {
            if (lane == 0) {
                mbar_arrive_expect_tx(&full[s], HALF);   // the peer's pushed half
                mbar_arrive_expect_tx(&mine[s], HALF);   // my own half
            }
            __syncwarp();
            if (lane < 4) {  // blocks 4*rank + lane of the tile, both atom columns
                const int b = 4 * (int)rank + lane;
                const int blk = (int)(((seed >> 8) + (unsigned)b * 2654435761u) % (unsigned)nblk);
                tma_load_2d(slot + b * 2048, &tm, 0, blk * 16, &mine[s]);
                tma_load_2d(slot + 16384 + b * 2048, &tm, 64, blk * 16, &mine[s]);
            }
            __syncwarp();
            ok = mbar_wait(&mine[s], use & 1, dl);
            if (!ok) break;
            if (lane == 0) {
                const uint32_t rb = map_peer(smem_addr(&full[s]), peer);
                for (int at = 0; at < 2; ++at) {
                    uint8_t *src = slot + at * 16384 + rank * 8192;  // my 4 blocks of atom column at
                    push_to_peer(map_peer(smem_addr(src), peer), src, 8192, rb);
                }
                asm volatile("cp.async.bulk.commit_group;" ::: "memory");
                mbar_arrive(&full[s]);  // my own half is in place
            }
            __syncwarp();
        }
    }
    // drain: the last fill of every slot, my pushes' reads
    const uint64_t dd = ok ? dl : drain_deadline();
    for (int s = 0; s < S && s < issued; ++s) {
        const int last = s + S * ((issued - 1 - s) / S);
        if (!mbar_wait(&full[s], (last / S) & 1, dd)) ok = false;
    }
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
    long long t1 = clock64();
    __syncwarp();
    cluster_sync();  // no CTA leaves while the peer may still write into it
    if (lane == 0) {
        out[blockIdx.x] = t1 - t0;
        if (!ok) atomicOr(err, 1u);
    }
}

int main() {
    const int nblk = 16384;  // 64 MB of 4 KB blocks (L2-sized working set: 126 MB L2)
    const size_t bytes = (size_t)nblk * 4096;
    uint8_t *buf; cudaMalloc(&buf, bytes); cudaMemset(buf, 1, bytes);
    long long *out; cudaMalloc(&out, 148 * sizeof(long long));
    unsigned *err; cudaMalloc(&err, 4); cudaMemset(err, 0, 4);
    void *fp = nullptr; cudaDriverEntryPointQueryResult q;
    cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fp, cudaEnableDefault, &q);
    auto enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fp);
    CUtensorMap tm;
    const cuuint64_t dims[2] = {128, (cuuint64_t)nblk * 16};
    const cuuint64_t strides[1] = {256};
    const cuuint32_t box[2] = {64, 16};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, buf, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS) {
        printf("encode failed\n"); return 1;
    }
    int sms = 0; cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, 0);
    cudaFuncSetAttribute(bench, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
    cudaFuncSetAttribute(bench_lsu, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
    const int iters = 400;
    for (int mode = 0; mode < 3; ++mode)
        for (int S : {1, 2, 3, 4, 6}) {
            const int sm = S * TILE + 64 + 1024;
            for (int rep = 0; rep < 2; ++rep) {
                bench<<<sms, 32, sm>>>(tm, buf, nblk, S, mode, iters, out, err);
                cudaError_t e = cudaDeviceSynchronize();
                if (e != cudaSuccess) { printf("cuda error %s\n", cudaGetErrorString(e)); return 1; }
            }
            std::vector<long long> h(sms);
            cudaMemcpy(h.data(), out, sms * sizeof(long long), cudaMemcpyDeviceToHost);
            unsigned he = 0; cudaMemcpy(&he, err, 4, cudaMemcpyDeviceToHost);
            double mx = 0, sum = 0;
            for (auto v : h) { mx = v > mx ? v : mx; sum += v; }
            const double bpc = (double)iters * TILE / (sum / sms);
            printf("mode %d (%s) slots %d: %.1f B/clk per SM (mean), %.2f TB/s at 1.965 GHz over %d SMs, err %u\n", mode,
                   mode == 0 ? "2-D 16x128B boxes" : mode == 1 ? "1-D 4 KB bulk" : "1-D 2 KB bulk", S, bpc,
                   bpc * sms * 1.965e9 / 1e12, sms, he);
        }
    for (int S : {1, 2, 4}) {
        const int sm = S * TILE + 1024;
        for (int rep = 0; rep < 2; ++rep) {
            bench_lsu<<<sms, 128, sm>>>(buf, nblk, S, iters, out);
            cudaError_t e = cudaDeviceSynchronize();
            if (e != cudaSuccess) { printf("cuda error %s\n", cudaGetErrorString(e)); return 1; }
        }
        std::vector<long long> h(sms);
        cudaMemcpy(h.data(), out, sms * sizeof(long long), cudaMemcpyDeviceToHost);
        double sum = 0;
        for (auto v : h) sum += v;
        const double bpc = (double)iters * TILE / (sum / sms);
        printf("mode LSU cp.async 16 B, 128 threads, groups in flight %d: %.1f B/clk per SM, %.2f TB/s\n", S == 1 ? 1 : (S == 2 ? 2 : 4), bpc,
               bpc * sms * 1.965e9 / 1e12);
    }
    // pairs of CTAs (clusters of 2) sharing each tile: mode 0 both load it whole by TMA, mode 1 each
    // loads half by TMA and pushes that half into the other's slot (shared::cta -> shared::cluster)
    const int grid = sms & ~1;
    cudaFuncSetAttribute(bench_pair, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
    for (int mode = 0; mode < 2; ++mode)
        for (int S : {2, 4}) {
            const int sm = S * TILE + 3 * S * 8 + 1024 + 64;
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(grid); cfg.blockDim = dim3(32); cfg.dynamicSmemBytes = sm;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = 2; attr[0].val.clusterDim.y = 1; attr[0].val.clusterDim.z = 1;
            cfg.attrs = attr; cfg.numAttrs = 1;
            for (int rep = 0; rep < 2; ++rep) {
                cudaError_t e = cudaLaunchKernelEx(&cfg, bench_pair, tm, nblk, S, mode, iters, out, err);
                if (e != cudaSuccess) { printf("launch error %s\n", cudaGetErrorString(e)); return 1; }
                e = cudaDeviceSynchronize();
                if (e != cudaSuccess) { printf("cuda error %s\n", cudaGetErrorString(e)); return 1; }
            }
            std::vector<long long> h(grid);
            cudaMemcpy(h.data(), out, grid * sizeof(long long), cudaMemcpyDeviceToHost);
            unsigned he = 0; cudaMemcpy(&he, err, 4, cudaMemcpyDeviceToHost);
            double sum = 0;
            for (auto v : h) sum += v;
            const double bpc = (double)iters * TILE / (sum / grid);
            printf("pair mode %d (%s) slots %d: %.1f B/clk per SM of tile data, err %u\n", mode,
                   mode == 0 ? "whole tile by TMA" : "half by TMA + half pushed by the peer", S, bpc, he);
        }
    return 0;
}
