// Device helpers shared by the kernels: launch shapes and map geometry.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>
#include <map>
#include <mutex>

#include "internal.h"

namespace tdm {

// Launch shape of a kernel on the current device: resident CTAs per SM at the
// given block size and dynamic shared memory (the shared-memory attribute set
// when above the default 48 KiB) and the SM count, computed once per
// (device, kernel) and cached, so launches repeat no driver queries.
struct LaunchShape {
    int per_sm, sms;
};

inline cudaError_t launch_shape(const void *kernel, int threads, size_t smem, LaunchShape *out) {
    static std::mutex mu;
    static std::map<std::pair<int, const void *>, LaunchShape> cache;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    const auto it = cache.find({dev, kernel});
    if (it != cache.end()) {
        *out = it->second;
        return cudaSuccess;
    }
    if (smem > 48 * 1024) {
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    LaunchShape shape{0, 0};
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&shape.per_sm, kernel, threads, smem);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&shape.sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    if (shape.per_sm < 1) shape.per_sm = 1;
    cache[{dev, kernel}] = shape;
    *out = shape;
    return cudaSuccess;
}


// (r << 4 | q) of upper row quad u in row-major order (u < 544).
struct UpperQuadTable {
    uint16_t v[kUpperQuads];
};
constexpr UpperQuadTable make_upper_quads() {
    UpperQuadTable t{};
    int u = 0;
    for (int r = 0; r < kN; ++r)
        for (int q = 0; q < kQuadsPerRow; ++q)
            if (4 * q + 3 >= r) t.v[u++] = (uint16_t)((r << 4) | q);
    return t;
}

__device__ __forceinline__ float4 ld4(const float *p) { return *reinterpret_cast<const float4 *>(p); }
__device__ __forceinline__ float4 ldg4(const float *p) { return __ldg(reinterpret_cast<const float4 *>(p)); }
__device__ __forceinline__ void st4(float *p, float4 v) { *reinterpret_cast<float4 *>(p) = v; }
__device__ __forceinline__ float comp(const float4 &v, int t) {
    return t == 0 ? v.x : t == 1 ? v.y : t == 2 ? v.z : v.w;
}

// Noise id of map (c, k, b).
__device__ __forceinline__ uint64_t noise_id(int64_t base, int c, int T, int k, int64_t B_total,
                                             int64_t b_off, int b) {
    return (uint64_t)(base + ((int64_t)c * T + k) * B_total + b_off + b);
}

}  // namespace tdm
