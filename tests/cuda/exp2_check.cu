// Evaluates the library's FMA-pipe exp2 (ptx::exp2_fma_x2) and CUDA's exp2f on a grid of
// inputs and writes x, y_fma, y_cuda as float32 triples to the file named by argv[1].
#include <cstdio>
#include <cstdlib>
#include <vector>

#include "../../entropic_ot_attention_b200/csrc/ptx.cuh"

__global__ void eval(const float* x, float* y_fma, float* y_ref, int n) {
    int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
    if (i + 1 >= n) return;
    float a, b;
    eot::ptx::exp2_fma_x2(x[i], x[i + 1], a, b);
    y_fma[i] = a;
    y_fma[i + 1] = b;
    y_ref[i] = exp2f(x[i]);
    y_ref[i + 1] = exp2f(x[i + 1]);
}

int main(int argc, char** argv) {
    const int n = 1 << 22;
    std::vector<float> x(n);
    for (int i = 0; i < n; ++i) x[i] = -124.0f + 124.5f * float(i) / float(n - 1);   // [-124, 0.5]
    float *dx, *df, *dr;
    if (cudaMalloc(&dx, n * 4) || cudaMalloc(&df, n * 4) || cudaMalloc(&dr, n * 4)) return 2;
    cudaMemcpy(dx, x.data(), n * 4, cudaMemcpyHostToDevice);
    eval<<<(n / 2 + 255) / 256, 256>>>(dx, df, dr, n);
    std::vector<float> yf(n), yr(n);
    if (cudaMemcpy(yf.data(), df, n * 4, cudaMemcpyDeviceToHost) != cudaSuccess) return 3;
    cudaMemcpy(yr.data(), dr, n * 4, cudaMemcpyDeviceToHost);
    FILE* f = fopen(argv[1], "wb");
    if (!f) return 4;
    fwrite(x.data(), 4, n, f);
    fwrite(yf.data(), 4, n, f);
    fwrite(yr.data(), 4, n, f);
    fclose(f);
    return 0;
}
