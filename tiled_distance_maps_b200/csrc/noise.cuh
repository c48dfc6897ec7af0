// Counter-based normals: Philox4x32-10 words and the Box-Muller transform.
#pragma once

#include "common.cuh"

namespace tdm {

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
// The radius is formed as r = kRadScale * rho, rho = sqrt(-log2 u1) and
// kRadScale = sqrt(2 ln 2), so that a caller can fold kRadScale into its own
// coefficients.  -log2 u1 comes from the hardware log2 (lg2.approx, absolute
// error ~2^-22) except for e < 2^-9, where that absolute error would be large
// relative to the result and the series -log2(1 - e) = (e + e^2/2 + e^3/3 +
// ...) / ln 2 truncated after three terms (relative error < e^3 / 4) is used.
// The angle is c (u2 - 1/2) in [-pi, pi), where the hardware sine and cosine
// approximations hold their stated error, with c = kTwoPiF, the float next to
// 2 pi (relative error 1.0e-7) whose product with 3/2 is exact, so that the
// angle is one fused multiply-add of the mantissa float 1 + u2 rounded once.
// The sign is restored by the caller: cos(2 pi u2) = -cos(2 pi (u2 - 1/2)),
// likewise for sin.
constexpr float kRadScale = 0x1.2d6abep+0f;     // sqrt(2 ln 2)
constexpr float kTwoPiF = 0x1.921fb8p+2f;       // 2 pi (1 + 1.0e-7)
constexpr float kAngOff = -0x1.2d97cap+3f;      // -3/2 kTwoPiF, exact
constexpr float kSerEdge = 0x1.008p+0f;         // 1 + 2^-9

// -log2(1 - e) by three terms of its series
__device__ __forceinline__ float neglog2_series(float e) {
    return e * fmaf(e, fmaf(e, 0x1.ec709ep-2f, 0x1.715476p-1f), 0x1.715476p+0f);
}

__device__ __forceinline__ float mufu_lg2(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float mufu_sqrt(float x) {
    float y;
    asm("sqrt.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float mufu_sin(float x) {
    float y;
    asm("sin.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float mufu_cos(float x) {
    float y;
    asm("cos.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// 1 + (w >> 9) 2^-23 in [1, 2): the top 23 bits of w as the mantissa of a
// float with exponent 0 (a funnel shift of 0x7F : w does the same in one
// instruction but measured slower in the fused run)
__device__ __forceinline__ float mantissa_float(uint32_t w) { return __uint_as_float(0x3F800000u | (w >> 9)); }

// rho of word a and the cosine and sine of the reduced angle of word b
__device__ __forceinline__ void box_muller_parts(uint32_t a, uint32_t b, float &rho, float &cs, float &sn) {
    const float f = mantissa_float(a);     // 1 + e
    const float lg = mufu_lg2(fmaf(f, -1.0f, 2.0f));                // log2 u1
    rho = mufu_sqrt(f < kSerEdge ? neglog2_series(f - 1.0f) : -lg);
    const float ang = fmaf(mantissa_float(b), kTwoPiF, kAngOff);
    cs = mufu_cos(ang);
    sn = mufu_sin(ang);
}

__device__ __forceinline__ float2 box_muller(uint32_t a, uint32_t b) {
    float rho, cs, sn;
    box_muller_parts(a, b, rho, cs, sn);
    const float nr = -kRadScale * rho;
    return make_float2(nr * cs, nr * sn);
}

// box_muller_parts on the two word pairs (w.x, w.y) and (w.z, w.w) of one
// Philox call at once, in packed float32 arithmetic (two components per
// instruction, each rounded as the scalar operation, so rho, cs and sn are
// bit-identical to box_muller_parts'):  z0 = -kRadScale rho.x cs.x,
// z1 = -kRadScale rho.x sn.x, z2 = -kRadScale rho.y cs.y,
// z3 = -kRadScale rho.y sn.y.  With VOTE the series branch runs only when a
// lane of the warp needs it (about one call in nine at e < 2^-9), decided by
// a warp vote, and all 32 lanes must call together; without it the series is
// computed for every pair and selected, which keeps the branch off each
// lane's dependency chain (for launches too small to hide latency).
template <bool VOTE>
__device__ __forceinline__ void box_muller_packed(uint4 w, float2 &rho, float2 &cs, float2 &sn) {
    const float2 f = make_float2(mantissa_float(w.x), mantissa_float(w.z));
    const float2 fb = make_float2(mantissa_float(w.y), mantissa_float(w.w));
    const float2 u1 = __ffma2_rn(f, make_float2(-1.0f, -1.0f), make_float2(2.0f, 2.0f));     // 2 - f, exact
    float2 v = make_float2(-mufu_lg2(u1.x), -mufu_lg2(u1.y));
    const bool sx = f.x < kSerEdge, sy = f.y < kSerEdge;
    if (!VOTE || __any_sync(0xffffffffu, sx || sy)) {
        const float2 e = __fadd2_rn(f, make_float2(-1.0f, -1.0f));
        const float2 ser = __fmul2_rn(
            e, __ffma2_rn(e, __ffma2_rn(e, make_float2(0x1.ec709ep-2f, 0x1.ec709ep-2f),
                                        make_float2(0x1.715476p-1f, 0x1.715476p-1f)),
                          make_float2(0x1.715476p+0f, 0x1.715476p+0f)));
        if (sx) v.x = ser.x;
        if (sy) v.y = ser.y;
    }
    rho = make_float2(mufu_sqrt(v.x), mufu_sqrt(v.y));
    const float2 ang = __ffma2_rn(fb, make_float2(kTwoPiF, kTwoPiF), make_float2(kAngOff, kAngOff));
    cs = make_float2(mufu_cos(ang.x), mufu_cos(ang.y));
    sn = make_float2(mufu_sin(ang.x), mufu_sin(ang.y));
}

// The four normals of row quad (r, q): columns 4q .. 4q+3.
__device__ __forceinline__ float4 quad_normals(int r, int q, uint32_t step_word, uint64_t g, int tag,
                                               const PhiloxKeys &K) {
    const uint4 w = philox4x32_10(noise_counter(r, q, step_word, g, tag), K);
    const float2 z01 = box_muller(w.x, w.y);
    const float2 z23 = box_muller(w.z, w.w);
    return make_float4(z01.x, z01.y, z23.x, z23.y);
}

}  // namespace tdm
