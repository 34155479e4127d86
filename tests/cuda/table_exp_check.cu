// Accuracy of the verifier's table-driven fp64 exp against CUDA's exp().
// Prints the largest relative error over a dense sweep of [-60, 0] and a
// few special points; exits non-zero if it exceeds the bound given as argv[1].
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <vector>

#include "fp64_exp.cuh"

__global__ void eval(const double *x, double *y, double *ref, int n)
{
    __shared__ double table[tsd::kExpTable];
    tsd::fill_exp_table(table, 1.0);
    __syncthreads();
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        y[i] = tsd::table_exp(x[i], table);
        ref[i] = exp(x[i]);
    }
}

int main(int argc, char **argv)
{
    const double bound = argc > 1 ? atof(argv[1]) : 1e-14;
    const int n = 1 << 22;
    std::vector<double> hx(n);
    for (int i = 0; i < n - 8; ++i)
        hx[i] = -60.0 * (double)i / (double)(n - 9);
    const double special[8] = {0.0, -1e-300, -0.5, -0.6931471805599453, -700.0, -707.9, -709.0, -1e4};
    for (int i = 0; i < 8; ++i)
        hx[n - 8 + i] = special[i];
    double *dx, *dy, *dr;
    cudaMalloc(&dx, n * sizeof(double));
    cudaMalloc(&dy, n * sizeof(double));
    cudaMalloc(&dr, n * sizeof(double));
    cudaMemcpy(dx, hx.data(), n * sizeof(double), cudaMemcpyHostToDevice);
    eval<<<592, 256>>>(dx, dy, dr, n);
    std::vector<double> hy(n), hr(n);
    cudaMemcpy(hy.data(), dy, n * sizeof(double), cudaMemcpyDeviceToHost);
    cudaMemcpy(hr.data(), dr, n * sizeof(double), cudaMemcpyDeviceToHost);
    if (cudaGetLastError() != cudaSuccess) {
        printf("cuda error\n");
        return 2;
    }
    double worst = 0.0;
    for (int i = 0; i < n; ++i) {
        const double x = hx[i];
        if (x < -708.0) {
            if (hy[i] != 0.0) {
                printf("x=%g: expected 0, got %g\n", x, hy[i]);
                return 1;
            }
            continue;
        }
        const double rel = std::fabs(hy[i] - hr[i]) / hr[i];
        if (rel > worst)
            worst = rel;
    }
    printf("max relative error %.3e over %d points\n", worst, n);
    return worst <= bound ? 0 : 1;
}
