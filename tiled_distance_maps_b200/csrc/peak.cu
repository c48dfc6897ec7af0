// Diagnostics: the device's float32 FMA rate, the measured denominator of the
// ALU rooflines.  Every thread runs 8 independent fmaf chains (x <- x m + c,
// which IEEE arithmetic does not let the compiler fold), so issue, not
// dependency latency, bounds the kernel; 8 CTAs of 256 threads per SM keep
// every scheduler full.
#include "common.cuh"

namespace tdm {
namespace {

constexpr int kFmaChains = 8;
constexpr int kFmaUnroll = 16;

__global__ void __launch_bounds__(256) fma_rate_kernel(float *__restrict__ sink, int iters, float seed) {
    float a[kFmaChains];
#pragma unroll
    for (int k = 0; k < kFmaChains; ++k) a[k] = seed + (float)(threadIdx.x + k) * 1e-3f;
    const float m = 0.9999999f, c = 1e-7f;
    for (int i = 0; i < iters; ++i) {
#pragma unroll
        for (int u = 0; u < kFmaUnroll; ++u)
#pragma unroll
            for (int k = 0; k < kFmaChains; ++k) a[k] = fmaf(a[k], m, c);
    }
    float s = 0.0f;
#pragma unroll
    for (int k = 0; k < kFmaChains; ++k) s += a[k];
    // never true for these inputs; keeps the chains live
    if (s == -1.0f) sink[(int64_t)blockIdx.x * blockDim.x + threadIdx.x] = s;
}

}  // namespace

// FMAs per launch: blocks x 256 threads x iters x 8 chains x 16.
cudaError_t launch_fma_rate(float *sink, int64_t sink_floats, int iters, cudaStream_t st, double *fmas) {
    int dev = 0, sms = 148;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const int blocks = 8 * sms;
    if ((int64_t)blocks * 256 > sink_floats) return cudaErrorInvalidValue;
    fma_rate_kernel<<<blocks, 256, 0, st>>>(sink, iters, 1.0f);
    *fmas = (double)blocks * 256.0 * (double)iters * kFmaChains * kFmaUnroll;
    return cudaGetLastError();
}

}  // namespace tdm
