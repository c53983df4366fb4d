// mma_rates.cu -- clocks per tcgen05 MMA (kind::f16, bf16, M=128 N=128 K=16,
// one CTA per SM, operands streamed from 8 distinct 16 KB shared-memory tiles)
// under the side traffic of the prefill kernel:
//   mode 0: B K-major (the score MMAs S = Q K^T) alone;
//   mode 1: B MN-major (the P.V MMAs, V rows = keys) alone;
//   mode 2: mode 0 with 16 other warps loading TMEM (tcgen05.ld, other columns);
//   mode 3: mode 0 with 16 other warps storing 16 B a thread to shared memory.
// The peak is 64 clocks (2.25 PFLOP/s dense bf16 over 148 SMs at 1.965 GHz).
// Every wait is bounded (2 s); every access stays inside its buffer.
// Build and run: nvcc -gencode arch=compute_100a,code=sm_100a -O3 -std=c++17
//   --expt-relaxed-constexpr -I include -o /tmp/mma_rates tests/gpu_checks/mma_rates.cu && /tmp/mma_rates
#include <cuda_runtime.h>
#include <cstdio>
#include <cstdint>
#include <vector>
#include "../../paged_kv_cache_408_b200/csrc/common.cuh"
#include "../../paged_kv_cache_408_b200/csrc/tc.cuh"
using namespace pa;

__global__ void __launch_bounds__(544, 1) rate(int n_mma, int mode, long long *out, unsigned *err, float *sink) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t *ops = smem;                  // 8 x 16 KB operand tiles
    uint8_t *scratch = smem + 131072;     // 64 KB store target
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + 196608);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bars + 2);
    volatile int *stop = reinterpret_cast<volatile int *>(bars + 3);
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    for (int i = tid; i < 131072 / 16; i += blockDim.x) reinterpret_cast<uint4 *>(ops)[i] = make_uint4(0x3f803f80u, 0, 0, 0);
    fence_proxy_async_smem();
    if (tid == 0) { mbar_init(&bars[0], 1); fence_mbar_init(); *stop = 0; }
    if (w == 16) tmem_alloc(tslot, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    const uint64_t dl = wait_deadline();
    bool ok = true;
    long long t0 = clock64(), t1 = t0;
    if (w == 16) {
        if (lane == 0) {
            const bool mn = mode == 1;
            const uint32_t idesc = idesc_f16kind_f32(128, 128, mn, true);
            const uint32_t o0 = smem_addr(ops);
            for (int i = 0; i < n_mma; ++i) {
                const int ta = (i >> 2) & 7, tb = ((i >> 2) + 3) & 7;
                const uint64_t ad = smem_desc_sw128(o0 + ta * 16384 + (i & 3) * 32, 16, 1024);
                // MN-major B: 16 rows (K) x 128 B, next K-step 16 rows down; LBO = distance between N atoms
                const uint64_t bd = mn ? smem_desc_sw128(o0 + tb * 16384 + (i & 7) * 16 * 128 % 16384, 8192, 1024)
                                       : smem_desc_sw128(o0 + tb * 16384 + (i & 3) * 32, 16, 1024);
                tc_mma_bf16(tmem, ad, bd, idesc, i > 0);  // accumulator columns 0..127
            }
            tc_commit(&bars[0]);
        }
        __syncwarp();
        ok = mbar_wait(&bars[0], 0, dl);
        t1 = clock64();
        if (lane == 0) *stop = 1;
    } else if (mode == 2) {
        float acc = 0.f;
        const uint32_t lb = tmem + ((uint32_t)((w & 3) * 32) << 16) + 256 + 64 * ((w >> 2) & 3) % 256;
        while (!*stop) {
            float v[32];
            tmem_ld32(lb, v);
            tmem_wait_ld();
            acc += v[0];
        }
        if (acc == 12345.f) sink[tid] = acc;
    } else if (mode == 3) {
        uint4 *dst = reinterpret_cast<uint4 *>(scratch) + tid;
        int k = 0;
        while (!*stop) {
            dst[(k & 7) * 512] = make_uint4(k, k, k, k);
            ++k;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (w == 16) { tc_fence_after(); tmem_dealloc(tmem, 512); }
    if (w == 16 && lane == 0) { out[blockIdx.x] = t1 - t0; if (!ok) atomicOr(err, 1u); }
}

int main() {
    long long *out; unsigned *err; float *sink;
    cudaMalloc(&out, 256 * 8); cudaMalloc(&err, 4); cudaMemset(err, 0, 4); cudaMalloc(&sink, 1024 * 4);
    int sms = 0; cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, 0);
    const int smem = 196608 + 64 + 1024;
    cudaFuncSetAttribute(rate, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    const int n = 4096;
    const char *names[4] = {"score-type MMAs (K-major B)", "P.V-type MMAs (MN-major B)", "score MMAs + 16 warps loading TMEM",
                            "score MMAs + 16 warps storing to shared memory"};
    for (int mode = 0; mode < 4; ++mode) {
        for (int rep = 0; rep < 2; ++rep) {
            rate<<<sms, 544, smem>>>(n, mode, out, err, sink);
            cudaError_t e = cudaDeviceSynchronize();
            if (e != cudaSuccess) { printf("run %s\n", cudaGetErrorString(e)); return 1; }
        }
        std::vector<long long> h(sms); unsigned he; cudaMemcpy(h.data(), out, sms * 8, cudaMemcpyDeviceToHost);
        cudaMemcpy(&he, err, 4, cudaMemcpyDeviceToHost);
        double sum = 0; for (auto v : h) sum += v;
        printf("%s: %.1f clocks per MMA, err %u\n", names[mode], (sum / sms) / n, he);
    }
    return 0;
}
