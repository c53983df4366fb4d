// exp2_check.cu -- test program: evaluates the FMA-pipe exponential of
// fastexp.cuh and the hardware approximation (ex2.approx.ftz.f32) on the
// same arguments, read as raw fp32 from stdin, and writes both results as
// raw fp32 pairs to stdout.  Built and run by tests/test_exp2_poly.py.
#include <cstdio>
#include <vector>

#include "fastexp.cuh"

__global__ void both(const float *x, float *out, int n) {
    const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
    if (i >= n) return;
    const float2 a = make_float2(x[i], i + 1 < n ? x[i + 1] : 0.f);
    const float2 p = pa::exp2_fma2(a);
    out[2 * i] = p.x;
    out[2 * i + 1] = pa::ex2(a.x);
    if (i + 1 < n) {
        out[2 * i + 2] = p.y;
        out[2 * i + 3] = pa::ex2(a.y);
    }
}

int main() {
    std::vector<float> x;
    float v;
    while (fread(&v, sizeof v, 1, stdin) == 1) x.push_back(v);
    const int n = (int)x.size();
    if (n == 0) return 1;
    float *dx = nullptr, *dout = nullptr;
    if (cudaMalloc(&dx, n * sizeof(float)) != cudaSuccess) return 2;
    if (cudaMalloc(&dout, 2 * (size_t)n * sizeof(float)) != cudaSuccess) return 2;
    cudaMemcpy(dx, x.data(), n * sizeof(float), cudaMemcpyHostToDevice);
    const int pairs = (n + 1) / 2;
    both<<<(pairs + 255) / 256, 256>>>(dx, dout, n);
    std::vector<float> out(2 * (size_t)n);
    if (cudaMemcpy(out.data(), dout, out.size() * sizeof(float), cudaMemcpyDeviceToHost) != cudaSuccess) return 3;
    fwrite(out.data(), sizeof(float), out.size(), stdout);
    cudaFree(dx);
    cudaFree(dout);
    return 0;
}
