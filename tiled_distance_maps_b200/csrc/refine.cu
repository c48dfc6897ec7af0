// Coordinate refinement by SMACOF (stress majorisation), one warp per map.
//
// ParaChromo (mdpi.com/2079-9292/15/13/2750), §3.1: the point cloud comes from
// distance-geometry initialisation followed by coordinate refinement.  The
// refinement minimises the raw stress sum_{i<j} (|x_i - x_j| - D_ij)^2 by the
// Guttman transform (de Leeuw 1977): x_i <- (1/n) sum_{j != i} (D_ij / d_ij)
// (x_i - x_j), with d_ij the current distances and terms with d_ij = 0 left
// out; D is symmetrised first.  A fixed number of iterations is run.
//
// Per map, a warp symmetrises D in shared memory (each unordered pair owned
// by one lane, so no barrier between reads and writes); lane l then updates
// beads l and l+32, reading its two rows of D as conflict-free 128-bit loads
// (row stride 68 floats) and the current coordinates as 128-bit broadcasts
// from structure-of-arrays copies, four beads per load.  The weight of a pair
// whose squared distance is below FLT_MIN is taken as zero, as for d = 0.
#include "common.cuh"

namespace tdm {
namespace {

constexpr int kRefWarps = 4;
constexpr int kLdR = kN + 4;
constexpr int kRefWarpFloats = kN * kLdR + 3 * kN;

__device__ __forceinline__ float rsqrt_approx(float x) {
    float r;
    asm("rsqrt.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

struct Bead {
    float x, y, z;
};

// one pair term: accumulates w (x_i - x_j) with w = D_ij / |x_i - x_j|
__device__ __forceinline__ void guttman_term(const Bead &xi, float xj, float yj, float zj, float dij, float &ax,
                                             float &ay, float &az) {
    const float e0 = xi.x - xj, e1 = xi.y - yj, e2 = xi.z - zj;
    const float q = fmaf(e2, e2, fmaf(e1, e1, e0 * e0));
    const float w = q >= 1.17549435e-38f ? dij * rsqrt_approx(q) : 0.0f;
    ax = fmaf(w, e0, ax);
    ay = fmaf(w, e1, ay);
    az = fmaf(w, e2, az);
}

__device__ __forceinline__ float stress_term(const Bead &xi, float xj, float yj, float zj, float dij) {
    const float e0 = xi.x - xj, e1 = xi.y - yj, e2 = xi.z - zj;
    const float r = sqrtf(fmaf(e2, e2, fmaf(e1, e1, e0 * e0))) - dij;
    return r * r;
}

__device__ __forceinline__ void publish(float *sx, int i0, int i1, const Bead &b0, const Bead &b1) {
    sx[i0] = b0.x;
    sx[kN + i0] = b0.y;
    sx[2 * kN + i0] = b0.z;
    sx[i1] = b1.x;
    sx[kN + i1] = b1.y;
    sx[2 * kN + i1] = b1.z;
}

__global__ void __launch_bounds__(kRefWarps * 32) refine_kernel(const float *__restrict__ maps, int64_t n,
                                                                float *__restrict__ coords, int iterations,
                                                                float *__restrict__ stress_out) {
    extern __shared__ __align__(16) float smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float *sD = smem + warp * kRefWarpFloats;
    float *sx = sD + kN * kLdR;    // x[64], y[64], z[64]
    const int i0 = lane, i1 = lane + 32;
    const float *r0 = sD + i0 * kLdR, *r1 = sD + i1 * kLdR;
    constexpr float kInvN = 1.0f / kN;

    for (int64_t m = (int64_t)blockIdx.x * kRefWarps + warp; m < n; m += (int64_t)gridDim.x * kRefWarps) {
        const float *D = maps + m * kMapFloats;
#pragma unroll 8
        for (int it = 0; it < 32; ++it) {
            const int idx = it * 32 + lane;
            const int row = idx >> 4, c4 = (idx & 15) << 2;
            *reinterpret_cast<float4 *>(sD + row * kLdR + c4) =
                __ldcs(reinterpret_cast<const float4 *>(D + row * kN + c4));
        }
        __syncwarp();
        // symmetrise: virtual lane v in {l, l+32} owns the pairs {v, v+k mod 64},
        // k = 0..32 (k = 32 only for v < 32)
#pragma unroll 3
        for (int k = 0; k <= 32; ++k) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                if (k == 32 && h == 1) continue;
                const int v = lane + 32 * h;
                const int w = (v + k) & (kN - 1);
                const float e = 0.5f * (sD[v * kLdR + w] + sD[w * kLdR + v]);
                sD[v * kLdR + w] = e;
                sD[w * kLdR + v] = e;
            }
        }
        float *X = coords + m * (kN * 3);
        Bead b0{X[3 * i0], X[3 * i0 + 1], X[3 * i0 + 2]};
        Bead b1{X[3 * i1], X[3 * i1 + 1], X[3 * i1 + 2]};
        for (int it = 0; it < iterations; ++it) {
            __syncwarp();
            publish(sx, i0, i1, b0, b1);
            __syncwarp();
            float a0x = 0.f, a0y = 0.f, a0z = 0.f, a1x = 0.f, a1y = 0.f, a1z = 0.f;
#pragma unroll 2
            for (int j4 = 0; j4 < kN / 4; ++j4) {
                const float4 px = *reinterpret_cast<const float4 *>(sx + 4 * j4);
                const float4 py = *reinterpret_cast<const float4 *>(sx + kN + 4 * j4);
                const float4 pz = *reinterpret_cast<const float4 *>(sx + 2 * kN + 4 * j4);
                const float4 d0 = *reinterpret_cast<const float4 *>(r0 + 4 * j4);
                const float4 d1 = *reinterpret_cast<const float4 *>(r1 + 4 * j4);
                guttman_term(b0, px.x, py.x, pz.x, d0.x, a0x, a0y, a0z);
                guttman_term(b1, px.x, py.x, pz.x, d1.x, a1x, a1y, a1z);
                guttman_term(b0, px.y, py.y, pz.y, d0.y, a0x, a0y, a0z);
                guttman_term(b1, px.y, py.y, pz.y, d1.y, a1x, a1y, a1z);
                guttman_term(b0, px.z, py.z, pz.z, d0.z, a0x, a0y, a0z);
                guttman_term(b1, px.z, py.z, pz.z, d1.z, a1x, a1y, a1z);
                guttman_term(b0, px.w, py.w, pz.w, d0.w, a0x, a0y, a0z);
                guttman_term(b1, px.w, py.w, pz.w, d1.w, a1x, a1y, a1z);
            }
            b0 = Bead{a0x * kInvN, a0y * kInvN, a0z * kInvN};
            b1 = Bead{a1x * kInvN, a1y * kInvN, a1z * kInvN};
        }
        X[3 * i0] = b0.x;
        X[3 * i0 + 1] = b0.y;
        X[3 * i0 + 2] = b0.z;
        X[3 * i1] = b1.x;
        X[3 * i1 + 1] = b1.y;
        X[3 * i1 + 2] = b1.z;
        if (stress_out != nullptr) {
            __syncwarp();
            publish(sx, i0, i1, b0, b1);
            __syncwarp();
            float acc = 0.0f;
#pragma unroll 2
            for (int j4 = 0; j4 < kN / 4; ++j4) {
                const float4 px = *reinterpret_cast<const float4 *>(sx + 4 * j4);
                const float4 py = *reinterpret_cast<const float4 *>(sx + kN + 4 * j4);
                const float4 pz = *reinterpret_cast<const float4 *>(sx + 2 * kN + 4 * j4);
                const float4 d0 = *reinterpret_cast<const float4 *>(r0 + 4 * j4);
                const float4 d1 = *reinterpret_cast<const float4 *>(r1 + 4 * j4);
                acc += stress_term(b0, px.x, py.x, pz.x, d0.x) + stress_term(b1, px.x, py.x, pz.x, d1.x);
                acc += stress_term(b0, px.y, py.y, pz.y, d0.y) + stress_term(b1, px.y, py.y, pz.y, d1.y);
                acc += stress_term(b0, px.z, py.z, pz.z, d0.z) + stress_term(b1, px.z, py.z, pz.z, d1.z);
                acc += stress_term(b0, px.w, py.w, pz.w, d0.w) + stress_term(b1, px.w, py.w, pz.w, d1.w);
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
            if (lane == 0) stress_out[m] = 0.5f * acc;    // each unordered pair appears twice
        }
        __syncwarp();
    }
}

}  // namespace

cudaError_t launch_refine(const float *maps, int64_t n, float *coords, int iterations, float *stress,
                          cudaStream_t st) {
    if (n <= 0) return cudaSuccess;
    const size_t smem = sizeof(float) * (size_t)kRefWarps * kRefWarpFloats;
    cudaError_t e = cudaFuncSetAttribute(refine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, refine_kernel, kRefWarps * 32, smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int64_t grid = (n + kRefWarps - 1) / kRefWarps;
    const int64_t cap = (int64_t)sms * (per_sm < 1 ? 1 : per_sm);
    if (grid > cap) grid = cap;
    refine_kernel<<<(int)grid, kRefWarps * 32, smem, st>>>(maps, n, coords, iterations, stress);
    return cudaGetLastError();
}

}  // namespace tdm
