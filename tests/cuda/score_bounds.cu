// Test helper (not part of the library): evaluates, on the device, the two
// error bounds the two-phase routing kernel relies on, so that a test can
// check them against double-precision references.
//
//  * tanh.approx.f32(x/2) for inputs x, against tanh(x/2) in double
//    (the approximate phase-1 sigmoid key is 0.5 tanh(x/2) + 0.5 + bias);
//  * the paired-reciprocal sigmoid (1/d0 = d1 rcp(d0 d1)) against the single
//    one (rcp(d0)), d = 1 + 2^(-x log2 e), both as the kernels compute them.
//
// Built by the test with nvcc into a temporary shared library.
#include <cuda_runtime.h>
#include <stdint.h>

__device__ __forceinline__ float tanh_apx(float y) {
    float r;
    asm("tanh.approx.f32 %0, %1;" : "=f"(r) : "f"(y));
    return r;
}
__device__ __forceinline__ float ex2_apx(float y) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(y));
    return r;
}
__device__ __forceinline__ float rcp_apx(float y) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(y));
    return r;
}

// out_tanh[i] = |tanh.approx(x/2) - tanh(x/2)| (double), x = xs[i]
// out_pair[i] = |pair sigmoid of (x, partner) - single sigmoid of x|, partner = xs[i ^ 1]
__global__ void bounds_kernel(const float* xs, int n, double* out_tanh, double* out_pair) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const float x = xs[i];
    const float half = 0.5f * x;
    out_tanh[i] = fabs((double)tanh_apx(half) - tanh((double)half));
    // both sigmoids take inputs clamped at -43.5, as the kernels do
    const float xc = fmaxf(x, -43.5f);
    const float xp = fmaxf(xs[i ^ 1], -43.5f);
    const float d0 = 1.0f + ex2_apx(xc * -1.4426950408889634f);
    const float d1 = 1.0f + ex2_apx(xp * -1.4426950408889634f);
    const float pair = d1 * rcp_apx(d0 * d1);
    const float single = rcp_apx(1.0f + ex2_apx(x * -1.4426950408889634f));
    out_pair[i] = fabs((double)pair - (double)single);
}

extern "C" int score_bounds(const float* host_x, int n, double* host_tanh, double* host_pair) {
    float* dx = nullptr;
    double *dt = nullptr, *dp = nullptr;
    if (cudaMalloc(&dx, sizeof(float) * n) != cudaSuccess) return 1;
    if (cudaMalloc(&dt, sizeof(double) * n) != cudaSuccess) return 1;
    if (cudaMalloc(&dp, sizeof(double) * n) != cudaSuccess) return 1;
    cudaMemcpy(dx, host_x, sizeof(float) * n, cudaMemcpyHostToDevice);
    bounds_kernel<<<(n + 255) / 256, 256>>>(dx, n, dt, dp);
    cudaError_t err = cudaDeviceSynchronize();
    cudaMemcpy(host_tanh, dt, sizeof(double) * n, cudaMemcpyDeviceToHost);
    cudaMemcpy(host_pair, dp, sizeof(double) * n, cudaMemcpyDeviceToHost);
    cudaFree(dx);
    cudaFree(dt);
    cudaFree(dp);
    return err == cudaSuccess ? 0 : 2;
}
