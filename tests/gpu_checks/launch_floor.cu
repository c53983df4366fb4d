// launch_floor.cu -- what two CUDA events around one launch read when the
// launch does nothing: an empty kernel of 148 CTAs x 384 threads (the decode
// kernel's grid) recorded between two events right after a 256 MB
// L2-flushing kernel, as the timed calls of the benchmark are.  Variants:
// no dynamic shared memory or 220 KB of it (the decode kernel's carve-out),
// with and without the programmatic-dependent-launch attribute, the flush
// kernel asking for the large carve-out too, two empty launches in a row
// (a decode call's decode + merge), and no flush before (the host then
// submits while the GPU idles).  Prints the median, minimum and 90th
// percentile of 50 launches each, in microseconds.  The kernels write
// nothing; the flush writes only inside its buffer.
// Build and run: nvcc -gencode arch=compute_100a,code=sm_100a -O3
//   -o /tmp/launch_floor tests/gpu_checks/launch_floor.cu && /tmp/launch_floor
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdio>
#include <vector>

__global__ void flush_kernel(int *buf, size_t n, int v) {
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
        buf[i] = v;
}

// the same, launched with a large dynamic shared-memory request (the
// shared-memory carve-out of the kernels that follow it)
__global__ void flush_kernel_big_carveout(int *buf, size_t n, int v) {
    extern __shared__ int s[];
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
        buf[i] = v;
    if (v == -12345 && threadIdx.x == 0) s[0] = v;  // never true: keeps the shared array
}

__global__ void empty_kernel(int *p, int v) {
    extern __shared__ int s[];
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (v == -12345 && threadIdx.x == 0) {  // never true
        s[0] = v;
        p[0] = s[0];
    }
}

static cudaError_t launch_empty(size_t smem, bool pdl, cudaStream_t st, int *p) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(148);
    cfg.blockDim = dim3(384);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, empty_kernel, p, 0);
}

int main() {
    const size_t n = ((size_t)256 << 20) / sizeof(int);  // 256 MB
    int *buf = nullptr;
    if (cudaMalloc(&buf, n * sizeof(int)) != cudaSuccess) return 1;
    cudaFuncSetAttribute(empty_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 220 * 1024);
    cudaFuncSetAttribute(flush_kernel_big_carveout, cudaFuncAttributeMaxDynamicSharedMemorySize, 220 * 1024);
    cudaFuncSetAttribute(flush_kernel_big_carveout, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    cudaStream_t st;
    cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking);
    struct Variant {
        const char *name;
        int flush;  // 0 plain, 1 large carve-out, 2 none
        size_t smem;
        bool pdl;
        int launches;
    };
    const std::vector<Variant> vs = {
        {"flush, empty kernel, no shared memory", 0, 0, false, 1},
        {"flush, empty kernel, 220 KB shared", 0, 220 * 1024, false, 1},
        {"flush, empty kernel, 220 KB shared, PDL", 0, 220 * 1024, true, 1},
        {"large-carve-out flush, 220 KB shared, PDL", 1, 220 * 1024, true, 1},
        {"large-carve-out flush, no shared memory, PDL", 1, 0, true, 1},
        {"flush, two empty kernels (220 KB + 0), PDL", 0, 220 * 1024, true, 2},
        {"no flush, empty kernel, 220 KB shared, PDL", 2, 220 * 1024, true, 1},
    };
    cudaEvent_t e0, e1;
    cudaEventCreate(&e0);
    cudaEventCreate(&e1);
    for (int pass = 0; pass < 2; ++pass)  // the first pass warms up
        for (const auto &v : vs) {
            std::vector<float> t;
            for (int r = 0; r < 60; ++r) {
                if (v.flush == 0) flush_kernel<<<148 * 8, 512, 0, st>>>(buf, n, r);
                if (v.flush == 1) flush_kernel_big_carveout<<<148 * 8, 512, 200 * 1024, st>>>(buf, n, r);
                cudaEventRecord(e0, st);
                launch_empty(v.smem, v.pdl, st, buf);
                if (v.launches == 2) launch_empty(0, true, st, buf);
                cudaEventRecord(e1, st);
                cudaStreamSynchronize(st);
                float ms = 0.f;
                cudaEventElapsedTime(&ms, e0, e1);
                if (r >= 10) t.push_back(ms * 1000.f);
            }
            std::sort(t.begin(), t.end());
            if (pass == 1)
                printf("%-48s median %.2f us  min %.2f  p90 %.2f\n", v.name, t[t.size() / 2], t[0],
                       t[t.size() * 9 / 10]);
        }
    const cudaError_t e = cudaDeviceSynchronize();
    printf("status %s\n", cudaGetErrorString(e));
    cudaFree(buf);
    return e == cudaSuccess ? 0 : 1;
}
