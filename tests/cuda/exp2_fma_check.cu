// Accuracy of the attention softmax's FMA-pipe 2^x against CUDA's exp2f():
// max relative error over a dense sweep of [-125, 9]; exact 0 below -125 and
// for -inf.  Exits non-zero if the error exceeds the bound given as argv[1].
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <vector>

#include "sm100_ptx.cuh"

__global__ void eval(const float *x, float *y, float *ref, int n)
{
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        y[i] = tsd::ptx::exp2_fma(x[i]);
        ref[i] = exp2f(x[i]);
    }
}

int main(int argc, char **argv)
{
    const double bound = argc > 1 ? atof(argv[1]) : 1e-4;
    const int n = 1 << 22;
    std::vector<float> hx(n);
    for (int i = 0; i < n - 4; ++i)
        hx[i] = -125.0f + 134.0f * (float)i / (float)(n - 5);
    hx[n - 4] = -INFINITY;
    hx[n - 3] = -126.5f;
    hx[n - 2] = -1000.0f;
    hx[n - 1] = 0.0f;
    float *dx, *dy, *dr;
    cudaMalloc(&dx, n * sizeof(float));
    cudaMalloc(&dy, n * sizeof(float));
    cudaMalloc(&dr, n * sizeof(float));
    cudaMemcpy(dx, hx.data(), n * sizeof(float), cudaMemcpyHostToDevice);
    eval<<<592, 256>>>(dx, dy, dr, n);
    std::vector<float> hy(n), hr(n);
    cudaMemcpy(hy.data(), dy, n * sizeof(float), cudaMemcpyDeviceToHost);
    cudaMemcpy(hr.data(), dr, n * sizeof(float), cudaMemcpyDeviceToHost);
    if (cudaGetLastError() != cudaSuccess) {
        printf("cuda error\n");
        return 2;
    }
    double worst = 0.0;
    for (int i = 0; i < n; ++i) {
        if (hx[i] < -125.0f) {
            if (hy[i] != 0.0f) {
                printf("x=%g: expected 0, got %g\n", hx[i], hy[i]);
                return 1;
            }
            continue;
        }
        const double rel = std::fabs((double)hy[i] - (double)hr[i]) / (double)hr[i];
        if (rel > worst)
            worst = rel;
    }
    printf("max relative error %.3e over %d points\n", worst, n);
    return worst <= bound ? 0 : 1;
}
