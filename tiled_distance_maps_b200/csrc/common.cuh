// Device helpers shared by the kernels: counter-based normals and map geometry.
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


// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy
// as 1, 2, 3", SC'11): per round, counter words 0 and 2 are multiplied by the
// two round constants; the high halves are xored with words 1 / 3 and the round
// key, the low halves move to words 1 / 3; the key advances by the Weyl
// constants between rounds.  The ten round keys of a seed are computed once on
// the host and passed as a kernel parameter.
struct Philox {
    static constexpr uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u;
    static constexpr uint32_t W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;
};

struct PhiloxKeys {
    uint32_t k0[10], k1[10];
};

inline PhiloxKeys philox_keys(uint64_t seed) {
    PhiloxKeys k;
    uint32_t a = (uint32_t)seed, b = (uint32_t)(seed >> 32);
    for (int r = 0; r < 10; ++r) {
        k.k0[r] = a;
        k.k1[r] = b;
        a += Philox::W0;
        b += Philox::W1;
    }
    return k;
}

__device__ __forceinline__ uint4 philox_round(uint4 c, uint32_t k0, uint32_t k1) {
    const uint64_t p0 = (uint64_t)Philox::M0 * c.x;
    const uint64_t p1 = (uint64_t)Philox::M1 * c.z;
    return make_uint4((uint32_t)(p1 >> 32) ^ c.y ^ k0, (uint32_t)p1, (uint32_t)(p0 >> 32) ^ c.w ^ k1,
                      (uint32_t)p0);
}

// rounds FIRST .. 9 (key index = round index)
template <int FIRST>
__device__ __forceinline__ uint4 philox_rounds(uint4 c, const PhiloxKeys &K) {
#pragma unroll
    for (int r = FIRST; r < 10; ++r) c = philox_round(c, K.k0[r], K.k1[r]);
    return c;
}

__device__ __forceinline__ uint4 philox4x32_10(uint4 c, const PhiloxKeys &K) { return philox_rounds<0>(c, K); }

// Counter of row quad (r, q) of the map with noise id g, stream tag, step word.
__device__ __forceinline__ uint4 noise_counter(int r, int q, uint32_t step_word, uint64_t g, int tag) {
    return make_uint4(((uint32_t)r << 4) | (uint32_t)q, step_word, (uint32_t)g,
                      ((uint32_t)(g >> 32) & 0xFFFFFFu) | ((uint32_t)tag << 24));
}

// Box-Muller on 23-bit uniforms built from float mantissas:
//   u1 = 1 - e, e = (a>>9) 2^-23 in [0, 1),  u2 = (b>>9) 2^-23 in [0, 1),
//   r = sqrt(-2 ln u1),  (z0, z1) = (r cos 2 pi u2, r sin 2 pi u2).
// -2 ln u1 comes from the hardware log2 (lg2.approx, absolute error ~2^-22)
// except for e < 2^-6, where that absolute error would be large relative to
// the result and the series -2 ln(1 - e) = 2e + e^2 + (2/3) e^3 + e^4/2 + ...
// truncated after three terms (relative error < e^3 / 4 < 1e-6) is used.
// The angle is taken as 2 pi (u2 - 1/2) in [-pi, pi), where the hardware sine
// and cosine approximations hold their stated error, and the sign is restored:
// cos(2 pi u2) = -cos(2 pi (u2 - 1/2)), likewise for sin.
__device__ __forceinline__ float2 box_muller(uint32_t a, uint32_t b) {
    const float f = __uint_as_float(0x3F800000u | (a >> 9));     // 1 + e
    const float e = f - 1.0f;
    const float u1 = 2.0f - f;
    const float h = __uint_as_float(0x3F800000u | (b >> 9)) - 1.5f;
    float lg, r, sn, cs;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(lg) : "f"(u1));
    // for e >= 2^-6 the log branch is >= 0.03, well clear of its error
    const float v_log = -1.3862943611198906f * lg;                   // -2 ln2 log2 u1
    const float v_ser = e * fmaf(e, fmaf(e, 0.6666667f, 1.0f), 2.0f);
    const float v = e < 0.015625f ? v_ser : v_log;
    asm("sqrt.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v));
    const float ang = 6.2831853071795865f * h;
    asm("sin.approx.ftz.f32 %0, %1;" : "=f"(sn) : "f"(ang));
    asm("cos.approx.ftz.f32 %0, %1;" : "=f"(cs) : "f"(ang));
    return make_float2(-r * cs, -r * sn);
}

// box_muller on the two word pairs (w.x, w.y) and (w.z, w.w) of one Philox
// call at once, in packed float32 arithmetic (two components per instruction,
// each rounded as the scalar operation): zc = -(z0, z2) and zs = -(z1, z3),
// the NEGATED normals of box_muller(w.x, w.y) = (z0, z1) and
// box_muller(w.z, w.w) = (z2, z3) (negation is exact; the caller folds it
// into its coefficients).
__device__ __forceinline__ void box_muller_packed(uint4 w, float2 &zc, float2 &zs) {
    const float2 f = make_float2(__uint_as_float(0x3F800000u | (w.x >> 9)), __uint_as_float(0x3F800000u | (w.z >> 9)));
    const float2 fb = make_float2(__uint_as_float(0x3F800000u | (w.y >> 9)), __uint_as_float(0x3F800000u | (w.w >> 9)));
    const float2 e = __fadd2_rn(f, make_float2(-1.0f, -1.0f));
    const float2 u1 = __ffma2_rn(f, make_float2(-1.0f, -1.0f), make_float2(2.0f, 2.0f));     // 2 - f, exact product
    const float2 h = __fadd2_rn(fb, make_float2(-1.5f, -1.5f));
    float2 lg, r, sn, cs;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(lg.x) : "f"(u1.x));
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(lg.y) : "f"(u1.y));
    const float2 v_log = __fmul2_rn(make_float2(-1.3862943611198906f, -1.3862943611198906f), lg);
    const float2 v_ser = __fmul2_rn(
        e, __ffma2_rn(e, __ffma2_rn(e, make_float2(0.6666667f, 0.6666667f), make_float2(1.0f, 1.0f)),
                      make_float2(2.0f, 2.0f)));
    const float2 v = make_float2(e.x < 0.015625f ? v_ser.x : v_log.x, e.y < 0.015625f ? v_ser.y : v_log.y);
    asm("sqrt.approx.ftz.f32 %0, %1;" : "=f"(r.x) : "f"(v.x));
    asm("sqrt.approx.ftz.f32 %0, %1;" : "=f"(r.y) : "f"(v.y));
    const float2 ang = __fmul2_rn(make_float2(6.2831853071795865f, 6.2831853071795865f), h);
    asm("sin.approx.ftz.f32 %0, %1;" : "=f"(sn.x) : "f"(ang.x));
    asm("cos.approx.ftz.f32 %0, %1;" : "=f"(cs.x) : "f"(ang.x));
    asm("sin.approx.ftz.f32 %0, %1;" : "=f"(sn.y) : "f"(ang.y));
    asm("cos.approx.ftz.f32 %0, %1;" : "=f"(cs.y) : "f"(ang.y));
    zc = __fmul2_rn(r, cs);
    zs = __fmul2_rn(r, sn);
}

// The four normals of row quad (r, q): columns 4q .. 4q+3.
__device__ __forceinline__ float4 quad_normals(int r, int q, uint32_t step_word, uint64_t g, int tag,
                                               const PhiloxKeys &K) {
    const uint4 w = philox4x32_10(noise_counter(r, q, step_word, g, tag), K);
    const float2 z01 = box_muller(w.x, w.y);
    const float2 z23 = box_muller(w.z, w.w);
    return make_float4(z01.x, z01.y, z23.x, z23.y);
}

__device__ __forceinline__ float4 words_to_normals(uint4 w) {
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
