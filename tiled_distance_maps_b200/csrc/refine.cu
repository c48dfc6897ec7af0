// Coordinate refinement by SMACOF (stress majorisation), one warp per map.
//
// ParaChromo (mdpi.com/2079-9292/15/13/2750), §3.1: the point cloud comes from
// distance-geometry initialisation followed by coordinate refinement.  The
// refinement minimises the raw stress sum_{i<j} (|x_i - x_j| - D_ij)^2 by the
// Guttman transform (de Leeuw 1977): x_i <- (1/n) sum_{j != i} (D_ij / d_ij)
// (x_i - x_j), with d_ij the current distances and terms with d_ij = 0 left
// out; D is symmetrised first.  A fixed number of iterations is run.
//
// Per map, a warp stages D in shared memory with asynchronous copies (issued
// for the next map while the current one iterates), symmetrises it in place
// (each unordered pair owned by one lane, so no barrier between reads and
// writes) and moves rows l and l+32 into registers; lane l then updates beads
// l and l+32, reading the current coordinates as 128-bit broadcasts from
// structure-of-arrays copies, four beads per load.  The squared distance of a
// pair is seeded with FLT_MIN, so a pair at distance zero (the diagonal,
// coincident beads) contributes w * 0 = 0 without a branch; pairs closer than
// about 1e-19 are weighted as if that far apart.
#include "common.cuh"

namespace tdm {
namespace {

constexpr int kRefWarps = 4;
constexpr int kLdR = kN + 4;
constexpr int kRefWarpFloats = kN * kLdR + 3 * kN;
constexpr float kQSeed = 1.17549435e-38f;    // FLT_MIN

__device__ __forceinline__ float rsqrt_approx(float x) {
    float r;
    asm("rsqrt.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// asynchronous 16-byte global -> shared copies of one map into the padded tile
__device__ __forceinline__ void stage_map_async(float *sD, const float *D, int lane) {
    const uint32_t base = static_cast<uint32_t>(__cvta_generic_to_shared(sD));
#pragma unroll 8
    for (int it = 0; it < 32; ++it) {
        const int idx = it * 32 + lane;
        const int row = idx >> 4, c4 = (idx & 15) << 2;
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(base + 4u * (row * kLdR + c4)),
                     "l"(D + row * kN + c4)
                     : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
}

__device__ __forceinline__ void wait_staged() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// one pair term: accumulates w (x_i - x_j), w = D_ij / |x_i - x_j|
__device__ __forceinline__ void guttman_term(float xi, float yi, float zi, float xj, float yj, float zj, float dij,
                                             float &ax, float &ay, float &az) {
    const float e0 = xi - xj, e1 = yi - yj, e2 = zi - zj;
    const float q = fmaf(e2, e2, fmaf(e1, e1, fmaf(e0, e0, kQSeed)));
    const float w = dij * rsqrt_approx(q);
    ax = fmaf(w, e0, ax);
    ay = fmaf(w, e1, ay);
    az = fmaf(w, e2, az);
}

__device__ __forceinline__ float sqrt_approx(float x) {
    float r;
    asm("sqrt.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ float stress_term(float xi, float yi, float zi, float xj, float yj, float zj, float dij) {
    const float e0 = xi - xj, e1 = yi - yj, e2 = zi - zj;
    const float r = sqrt_approx(fmaf(e2, e2, fmaf(e1, e1, e0 * e0))) - dij;
    return r * r;
}

struct Beads {    // beads l and l+32 of one lane
    float x0, y0, z0, x1, y1, z1;
};

__device__ __forceinline__ void publish(float *sx, int lane, const Beads &b) {
    __syncwarp();
    sx[lane] = b.x0;
    sx[kN + lane] = b.y0;
    sx[2 * kN + lane] = b.z0;
    sx[lane + 32] = b.x1;
    sx[kN + lane + 32] = b.y1;
    sx[2 * kN + lane + 32] = b.z1;
    __syncwarp();
}

__global__ void __launch_bounds__(kRefWarps * 32) refine_kernel(const float *__restrict__ maps, int64_t n,
                                                                float *__restrict__ coords, int iterations,
                                                                float *__restrict__ stress_out) {
    extern __shared__ __align__(16) float smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float *sD = smem + warp * kRefWarpFloats;
    float *sx = sD + kN * kLdR;    // x[64], y[64], z[64]
    const int64_t stride = (int64_t)gridDim.x * kRefWarps;
    constexpr float kInvN = 1.0f / kN;

    int64_t m = (int64_t)blockIdx.x * kRefWarps + warp;
    if (m < n) stage_map_async(sD, maps + m * kMapFloats, lane);
    for (; m < n; m += stride) {
        wait_staged();
        __syncwarp();
        // symmetrise: virtual lane v in {l, l+32} owns the pairs {v, v+k mod 64},
        // k = 0..32 (k = 32 only for v < 32); every element is read and written
        // by its owner only, so a batch of offsets can be loaded before it is stored
#pragma unroll 1
        for (int k0 = 0; k0 < 32; k0 += 4) {
            float e[2][4];
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int v = lane + 32 * h, w = (v + k0 + u) & (kN - 1);
                    e[h][u] = 0.5f * (sD[v * kLdR + w] + sD[w * kLdR + v]);
                }
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int v = lane + 32 * h, w = (v + k0 + u) & (kN - 1);
                    sD[v * kLdR + w] = e[h][u];
                    sD[w * kLdR + v] = e[h][u];
                }
        }
        {
            const int w = (lane + 32) & (kN - 1);
            const float e = 0.5f * (sD[lane * kLdR + w] + sD[w * kLdR + lane]);
            sD[lane * kLdR + w] = e;
            sD[w * kLdR + lane] = e;
        }
        __syncwarp();
        float d0[kN], d1[kN];
#pragma unroll
        for (int j4 = 0; j4 < kN / 4; ++j4) {
            const float4 a = *reinterpret_cast<const float4 *>(sD + lane * kLdR + 4 * j4);
            const float4 b = *reinterpret_cast<const float4 *>(sD + (lane + 32) * kLdR + 4 * j4);
            d0[4 * j4] = a.x;
            d0[4 * j4 + 1] = a.y;
            d0[4 * j4 + 2] = a.z;
            d0[4 * j4 + 3] = a.w;
            d1[4 * j4] = b.x;
            d1[4 * j4 + 1] = b.y;
            d1[4 * j4 + 2] = b.z;
            d1[4 * j4 + 3] = b.w;
        }
        __syncwarp();
        if (m + stride < n) stage_map_async(sD, maps + (m + stride) * kMapFloats, lane);

        float *X = coords + m * (kN * 3);
        Beads b{X[3 * lane], X[3 * lane + 1], X[3 * lane + 2],
                X[3 * (lane + 32)], X[3 * (lane + 32) + 1], X[3 * (lane + 32) + 2]};
        for (int it = 0; it < iterations; ++it) {
            publish(sx, lane, b);
            float a0x = 0.f, a0y = 0.f, a0z = 0.f, a1x = 0.f, a1y = 0.f, a1z = 0.f;
#pragma unroll
            for (int j4 = 0; j4 < kN / 4; ++j4) {
                const float4 px = *reinterpret_cast<const float4 *>(sx + 4 * j4);
                const float4 py = *reinterpret_cast<const float4 *>(sx + kN + 4 * j4);
                const float4 pz = *reinterpret_cast<const float4 *>(sx + 2 * kN + 4 * j4);
                const float jx[4] = {px.x, px.y, px.z, px.w};
                const float jy[4] = {py.x, py.y, py.z, py.w};
                const float jz[4] = {pz.x, pz.y, pz.z, pz.w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    guttman_term(b.x0, b.y0, b.z0, jx[u], jy[u], jz[u], d0[4 * j4 + u], a0x, a0y, a0z);
                    guttman_term(b.x1, b.y1, b.z1, jx[u], jy[u], jz[u], d1[4 * j4 + u], a1x, a1y, a1z);
                }
            }
            b = Beads{a0x * kInvN, a0y * kInvN, a0z * kInvN, a1x * kInvN, a1y * kInvN, a1z * kInvN};
        }
        X[3 * lane] = b.x0;
        X[3 * lane + 1] = b.y0;
        X[3 * lane + 2] = b.z0;
        X[3 * (lane + 32)] = b.x1;
        X[3 * (lane + 32) + 1] = b.y1;
        X[3 * (lane + 32) + 2] = b.z1;
        if (stress_out != nullptr) {
            publish(sx, lane, b);
            float acc0 = 0.0f, acc1 = 0.0f;
#pragma unroll
            for (int j4 = 0; j4 < kN / 4; ++j4) {
                const float4 px = *reinterpret_cast<const float4 *>(sx + 4 * j4);
                const float4 py = *reinterpret_cast<const float4 *>(sx + kN + 4 * j4);
                const float4 pz = *reinterpret_cast<const float4 *>(sx + 2 * kN + 4 * j4);
                const float jx[4] = {px.x, px.y, px.z, px.w};
                const float jy[4] = {py.x, py.y, py.z, py.w};
                const float jz[4] = {pz.x, pz.y, pz.z, pz.w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    acc0 += stress_term(b.x0, b.y0, b.z0, jx[u], jy[u], jz[u], d0[4 * j4 + u]);
                    acc1 += stress_term(b.x1, b.y1, b.z1, jx[u], jy[u], jz[u], d1[4 * j4 + u]);
                }
            }
            float acc = acc0 + acc1;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
            if (lane == 0) stress_out[m] = 0.5f * acc;    // each unordered pair appears twice
        }
    }
}

}  // namespace

cudaError_t launch_refine(const float *maps, int64_t n, float *coords, int iterations, float *stress,
                          cudaStream_t st) {
    if (n <= 0) return cudaSuccess;
    const size_t smem = sizeof(float) * (size_t)kRefWarps * kRefWarpFloats;
    LaunchShape shape;
    const cudaError_t e = launch_shape(reinterpret_cast<const void *>(refine_kernel), kRefWarps * 32, smem, &shape);
    if (e != cudaSuccess) return e;
    int64_t grid = (n + kRefWarps - 1) / kRefWarps;
    const int64_t cap = (int64_t)shape.sms * shape.per_sm;
    if (grid > cap) grid = cap;
    refine_kernel<<<(int)grid, kRefWarps * 32, smem, st>>>(maps, n, coords, iterations, stress);
    return cudaGetLastError();
}

}  // namespace tdm
