// Device helpers shared by the kernels: counter-based normals and map geometry.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

#include "internal.h"

namespace tdm {

// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy
// as 1, 2, 3", SC'11): per round, counter words 0 and 2 are multiplied by the
// two round constants; the high halves are xored with words 1 / 3 and the round
// key, the low halves move to words 1 / 3; the key advances by the Weyl
// constants between rounds.
struct Philox {
    static constexpr uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u;
    static constexpr uint32_t W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;
};

__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        const uint64_t p0 = (uint64_t)Philox::M0 * c.x;
        const uint64_t p1 = (uint64_t)Philox::M1 * c.z;
        c = make_uint4((uint32_t)(p1 >> 32) ^ c.y ^ k0, (uint32_t)p1,
                       (uint32_t)(p0 >> 32) ^ c.w ^ k1, (uint32_t)p0);
        k0 += Philox::W0;
        k1 += Philox::W1;
    }
    return c;
}

// Counter of row quad (r, q) of the map with noise id g, stream tag, step word.
__device__ __forceinline__ uint4 noise_counter(int r, int q, uint32_t step_word, uint64_t g, int tag) {
    return make_uint4(((uint32_t)r << 4) | (uint32_t)q, step_word, (uint32_t)g,
                      ((uint32_t)(g >> 32) & 0xFFFFFFu) | ((uint32_t)tag << 24));
}

// Box-Muller on 24-bit uniforms u1 = (a>>8 + 1) 2^-24 in (0, 1] and
// u2 = (b>>8) 2^-24 in [0, 1): r = sqrt(-2 ln u1), (r cos 2 pi u2, r sin 2 pi u2).
// Both uniforms are exact in float32.
__device__ __forceinline__ float2 box_muller(uint32_t a, uint32_t b) {
    const float u1 = (float)((a >> 8) + 1u) * 0x1p-24f;
    const float u2 = (float)(b >> 8) * 0x1p-24f;
    const float r = sqrtf(-2.0f * logf(u1));
    float s, c;
    sincospif(2.0f * u2, &s, &c);
    return make_float2(r * c, r * s);
}

// The four normals of row quad (r, q): columns 4q .. 4q+3.
__device__ __forceinline__ float4 quad_normals(int r, int q, uint32_t step_word, uint64_t g, int tag,
                                               uint32_t k0, uint32_t k1) {
    const uint4 w = philox4x32_10(noise_counter(r, q, step_word, g, tag), k0, k1);
    const float2 z01 = box_muller(w.x, w.y);
    const float2 z23 = box_muller(w.z, w.w);
    return make_float4(z01.x, z01.y, z23.x, z23.y);
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
