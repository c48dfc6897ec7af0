// Non-finite scan of a float buffer (a check a caller runs on any output).
//
// Raises TDM_FLAG_NONFINITE in the context's status word when any element is
// NaN or +-inf (all exponent bits set).  The 16-byte-aligned body is read with
// 128-bit streaming loads, the ragged head and tail with scalar loads; a warp
// that finds one sets the flag once.
#include "common.cuh"

namespace tdm {
namespace {

__device__ __forceinline__ bool nonfinite(float x) { return (__float_as_uint(x) & 0x7F800000u) == 0x7F800000u; }

__global__ void __launch_bounds__(256) scan_kernel(const float *__restrict__ head, int n_head,
                                                   const float4 *__restrict__ body, int64_t n_body,
                                                   const float *__restrict__ tail, int n_tail,
                                                   uint32_t *__restrict__ flags) {
    bool bad = false;
    const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t nthreads = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = tid; i < n_body; i += nthreads) {
        const float4 v = __ldcs(body + i);
        bad |= nonfinite(v.x) | nonfinite(v.y) | nonfinite(v.z) | nonfinite(v.w);
    }
    if (tid < n_head) bad |= nonfinite(head[tid]);
    if (tid < n_tail) bad |= nonfinite(tail[tid]);
    if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) atomicOr(flags, (uint32_t)TDM_FLAG_NONFINITE);
}

}  // namespace

cudaError_t launch_scan_nonfinite(const float *buf, int64_t n, uint32_t *flags, cudaStream_t st) {
    if (n <= 0) return cudaSuccess;
    const uintptr_t addr = reinterpret_cast<uintptr_t>(buf);
    int64_t n_head = (int64_t)(((16 - (addr & 15)) & 15) / 4);
    if (n_head > n) n_head = n;
    const int64_t n_body = (n - n_head) / 4;
    const int64_t n_tail = n - n_head - 4 * n_body;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int64_t blocks = (n_body + 255) / 256;
    if (blocks < 1) blocks = 1;
    if (blocks > (int64_t)sms * 8) blocks = (int64_t)sms * 8;
    scan_kernel<<<(unsigned)blocks, 256, 0, st>>>(buf, (int)n_head, reinterpret_cast<const float4 *>(buf + n_head),
                                                   n_body, buf + n_head + 4 * n_body, (int)n_tail, flags);
    return cudaGetLastError();
}

}  // namespace tdm
