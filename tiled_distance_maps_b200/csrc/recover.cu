// Coordinate recovery: classical MDS (one warp per map) and pairwise distances.
//
// ParaChromo (mdpi.com/2079-9292/15/13/2750) recovers a 64-bead point cloud from
// each final distance map by distance-geometry initialisation (§3.1, §5.5).  The
// reading used is classical MDS: B = -1/2 J (D*D) J, the top three eigenpairs,
// x_k = v_k sqrt(max(l_k, 0)).
//
// Per map, one warp stages D in shared memory, forms B (lane l computes rows l
// and l+32 in registers, then writes them over D) and finds the top eigenpairs by subspace iteration on four vectors with a
// Rayleigh-Ritz step (a 4 x 4 Jacobi eigen-solve) every iteration, stopping when
// the residual of the three leading Ritz pairs is below kTol * |l_1|.
#include "common.cuh"

namespace tdm {
namespace {

constexpr int kMdsWarps = 4;
constexpr int kLd = kN + 1;       // smem row stride: conflict-free row and column reads
constexpr int kMaxIt = 32;
constexpr float kTol = 4e-6f;

// start vectors: column c of V0 has entry (-1)^bit_j(v0_mask(c))
__host__ __device__ constexpr unsigned long long v0_mask(int c) {
    return c == 0 ? 0x9E3779B97F4A7C15ull : c == 1 ? 0xBF58476D1CE4E5B9ull
         : c == 2 ? 0x94D049BB133111EBull : 0xD6E8FEB86659FD93ull;
}

__device__ __forceinline__ float wsum(float v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}
__device__ __forceinline__ float wmax(float v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
    return v;
}

// Gram-Schmidt applied twice per column ("twice is enough") on 64 x 4 columns
// held as rows (l, l+32) per lane.
__device__ __forceinline__ void orthonormalize(float (&a0)[4], float (&a1)[4]) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
#pragma unroll
        for (int pass = 0; pass < 2; ++pass) {
            float d[4];
#pragma unroll
            for (int p = 0; p < c; ++p) d[p] = wsum(fmaf(a0[p], a0[c], a1[p] * a1[c]));
#pragma unroll
            for (int p = 0; p < c; ++p) {
                a0[c] = fmaf(-d[p], a0[p], a0[c]);
                a1[c] = fmaf(-d[p], a1[p], a1[c]);
            }
        }
        const float nn = wsum(fmaf(a0[c], a0[c], a1[c] * a1[c]));
        const float inv = nn > 0.0f ? 1.0f / sqrtf(nn) : 0.0f;
        a0[c] *= inv;
        a1[c] *= inv;
    }
}

template <int P, int Q>
__device__ __forceinline__ void jrot(float (&H)[4][4], float (&Y)[4][4]) {
    const float apq = H[P][Q];
    if (apq == 0.0f) return;
    const float tau = (H[Q][Q] - H[P][P]) / (2.0f * apq);
    const float t = copysignf(1.0f, tau) / (fabsf(tau) + sqrtf(fmaf(tau, tau, 1.0f)));
    const float c = 1.0f / sqrtf(fmaf(t, t, 1.0f));
    const float s = t * c;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float hp = H[k][P], hq = H[k][Q];
        H[k][P] = c * hp - s * hq;
        H[k][Q] = s * hp + c * hq;
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float hp = H[P][k], hq = H[Q][k];
        H[P][k] = c * hp - s * hq;
        H[Q][k] = s * hp + c * hq;
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float yp = Y[k][P], yq = Y[k][Q];
        Y[k][P] = c * yp - s * yq;
        Y[k][Q] = s * yp + c * yq;
    }
}

template <int I, int J>
__device__ __forceinline__ void sort_pair(float (&th)[4], float (&Y)[4][4]) {
    if (th[I] < th[J]) {
        const float tt = th[I];
        th[I] = th[J];
        th[J] = tt;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float y = Y[k][I];
            Y[k][I] = Y[k][J];
            Y[k][J] = y;
        }
    }
}

// Cyclic Jacobi on a symmetric 4 x 4 matrix (Golub & Van Loan §8.5); eigenvalues
// sorted in descending order, eigenvectors in the columns of Y.
__device__ __forceinline__ void eig4(float (&H)[4][4], float (&Y)[4][4], float (&th)[4]) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) Y[i][j] = i == j ? 1.0f : 0.0f;
    for (int sweep = 0; sweep < 10; ++sweep) {
        const float off = H[0][1] * H[0][1] + H[0][2] * H[0][2] + H[0][3] * H[0][3] + H[1][2] * H[1][2] +
                          H[1][3] * H[1][3] + H[2][3] * H[2][3];
        const float dia = H[0][0] * H[0][0] + H[1][1] * H[1][1] + H[2][2] * H[2][2] + H[3][3] * H[3][3];
        if (off <= 1e-14f * dia) break;
        jrot<0, 1>(H, Y);
        jrot<0, 2>(H, Y);
        jrot<0, 3>(H, Y);
        jrot<1, 2>(H, Y);
        jrot<1, 3>(H, Y);
        jrot<2, 3>(H, Y);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) th[i] = H[i][i];
    sort_pair<0, 1>(th, Y);
    sort_pair<2, 3>(th, Y);
    sort_pair<0, 2>(th, Y);
    sort_pair<1, 3>(th, Y);
    sort_pair<1, 2>(th, Y);
}

__global__ void __launch_bounds__(kMdsWarps * 32, 3) mds_kernel(const float *__restrict__ maps, int64_t n,
                                                             float *__restrict__ coords,
                                                             float *__restrict__ eig,
                                                             uint32_t *__restrict__ flags) {
    extern __shared__ float smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float *sD = smem + warp * (kN * kLd);
    float4 *sV = reinterpret_cast<float4 *>(smem + kMdsWarps * kN * kLd) + warp * kN;
    float *sR = smem + kMdsWarps * kN * kLd + kMdsWarps * kN * 4 + warp * kN;

    for (int64_t m = (int64_t)blockIdx.x * kMdsWarps + warp; m < n; m += (int64_t)gridDim.x * kMdsWarps) {
        const float *D = maps + m * kMapFloats;
#pragma unroll 8
        for (int it = 0; it < 32; ++it) {
            const int idx = it * 32 + lane;
            const int row = idx >> 4, c4 = (idx & 15) << 2;
            const float4 v = __ldcs(reinterpret_cast<const float4 *>(D + row * kN + c4));
            float *dst = sD + row * kLd + c4;
            dst[0] = v.x;
            dst[1] = v.y;
            dst[2] = v.z;
            dst[3] = v.w;
        }
        __syncwarp();

        // symmetrise and square; lane holds rows lane and lane+32
        float b0[kN], b1[kN];
        float mx = 0.0f;
#pragma unroll
        for (int j = 0; j < kN; ++j) {
            const float d0 = 0.5f * (sD[lane * kLd + j] + sD[j * kLd + lane]);
            const float d1 = 0.5f * (sD[(lane + 32) * kLd + j] + sD[j * kLd + lane + 32]);
            b0[j] = d0 * d0;
            b1[j] = d1 * d1;
            mx = fmaxf(mx, fmaxf(b0[j], b1[j]));
        }
        // exact power-of-two rescale of D*D to O(1), undone on the eigenvalues
        mx = wmax(mx);
        int ex = 0;
        frexpf(mx, &ex);
        const float scale = mx > 0.0f && isfinite(mx) ? ldexpf(1.0f, -ex) : 1.0f;
        float rs0 = 0.0f, rs1 = 0.0f;
#pragma unroll
        for (int j = 0; j < kN; ++j) {
            b0[j] *= scale;
            b1[j] *= scale;
            rs0 += b0[j];
            rs1 += b1[j];
        }
        const float r0 = rs0 * (1.0f / kN), r1 = rs1 * (1.0f / kN);
        const float gm = wsum(r0 + r1) * (1.0f / kN);
        __syncwarp();
        sR[lane] = r0;
        sR[lane + 32] = r1;
        __syncwarp();
        // double centring: B_ij = -1/2 (D2_ij - r_i - r_j + g)
#pragma unroll
        for (int j = 0; j < kN; ++j) {
            const float rj = sR[j];
            b0[j] = -0.5f * (b0[j] - r0 - rj + gm);
            b1[j] = -0.5f * (b1[j] - r1 - rj + gm);
        }

        // first basis: orth(B V0), from the register copy of B's rows
        float v0[4] = {0.f, 0.f, 0.f, 0.f}, v1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int j = 0; j < kN; ++j)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                if ((v0_mask(c) >> j) & 1ull) {
                    v0[c] -= b0[j];
                    v1[c] -= b1[j];
                } else {
                    v0[c] += b0[j];
                    v1[c] += b1[j];
                }
            }
        // B replaces D in shared memory (every lane has finished reading D)
#pragma unroll
        for (int j = 0; j < kN; ++j) {
            sD[lane * kLd + j] = b0[j];
            sD[(lane + 32) * kLd + j] = b1[j];
        }
        orthonormalize(v0, v1);
        sV[lane] = make_float4(v0[0], v0[1], v0[2], v0[3]);
        sV[lane + 32] = make_float4(v1[0], v1[1], v1[2], v1[3]);

        float th[4] = {0.f, 0.f, 0.f, 0.f};
        float u0[4], u1[4];
        bool conv = false;
        const float *bl = sD + lane * kLd, *bh = sD + (lane + 32) * kLd;
        for (int it = 0; it < kMaxIt; ++it) {
            __syncwarp();
            float w0[4] = {0.f, 0.f, 0.f, 0.f}, w1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 16
            for (int j = 0; j < kN; ++j) {
                const float4 v = sV[j];
                const float x0 = bl[j], x1 = bh[j];
                w0[0] = fmaf(x0, v.x, w0[0]);
                w0[1] = fmaf(x0, v.y, w0[1]);
                w0[2] = fmaf(x0, v.z, w0[2]);
                w0[3] = fmaf(x0, v.w, w0[3]);
                w1[0] = fmaf(x1, v.x, w1[0]);
                w1[1] = fmaf(x1, v.y, w1[1]);
                w1[2] = fmaf(x1, v.z, w1[2]);
                w1[3] = fmaf(x1, v.w, w1[3]);
            }
            // Rayleigh quotient H = V^T B V (symmetrised)
            float H[4][4];
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int b = a; b < 4; ++b) {
                    const float h = 0.5f * wsum(fmaf(v0[a], w0[b], fmaf(v0[b], w0[a],
                                                     fmaf(v1[a], w1[b], v1[b] * w1[a]))));
                    H[a][b] = h;
                    H[b][a] = h;
                }
            float Y[4][4];
            eig4(H, Y, th);
            float bu0[4], bu1[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                u0[c] = u1[c] = bu0[c] = bu1[c] = 0.0f;
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                    u0[c] = fmaf(v0[a], Y[a][c], u0[c]);
                    u1[c] = fmaf(v1[a], Y[a][c], u1[c]);
                    bu0[c] = fmaf(w0[a], Y[a][c], bu0[c]);
                    bu1[c] = fmaf(w1[a], Y[a][c], bu1[c]);
                }
            }
            float rmax = 0.0f;
#pragma unroll
            for (int c = 0; c < 3; ++c) {
                const float e0 = fmaf(-th[c], u0[c], bu0[c]);
                const float e1 = fmaf(-th[c], u1[c], bu1[c]);
                rmax = fmaxf(rmax, wsum(fmaf(e0, e0, e1 * e1)));
            }
            const float lim = kTol * fabsf(th[0]);
            if (rmax <= lim * lim) {
                conv = true;
                break;
            }
            orthonormalize(bu0, bu1);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                v0[c] = bu0[c];
                v1[c] = bu1[c];
            }
            __syncwarp();
            sV[lane] = make_float4(v0[0], v0[1], v0[2], v0[3]);
            sV[lane + 32] = make_float4(v1[0], v1[1], v1[2], v1[3]);
        }
        if (!conv && lane == 0) atomicOr(flags, (uint32_t)TDM_FLAG_MDS_NOT_CONVERGED);

        const float inv_scale = 1.0f / scale;
        float *X = coords + m * (kN * 3);
#pragma unroll
        for (int c = 0; c < 3; ++c) {
            const float sq = sqrtf(fmaxf(th[c], 0.0f) * inv_scale);
            X[lane * 3 + c] = u0[c] * sq;
            X[(lane + 32) * 3 + c] = u1[c] * sq;
        }
        if (eig != nullptr && lane < 3) eig[m * 3 + lane] = (lane == 0 ? th[0] : lane == 1 ? th[1] : th[2]) * inv_scale;
        __syncwarp();
    }
}

__global__ void __launch_bounds__(256) pdist_kernel(const float *__restrict__ coords, int64_t n,
                                                    float *__restrict__ maps) {
    __shared__ __align__(16) float sc[kN * 3];
    for (int64_t m = blockIdx.x; m < n; m += gridDim.x) {
        if (threadIdx.x < kN * 3 / 4)
            reinterpret_cast<float4 *>(sc)[threadIdx.x] = ldg4(coords + m * (kN * 3) + 4 * threadIdx.x);
        __syncthreads();
        float *out = maps + m * kMapFloats;
#pragma unroll 4
        for (int p = threadIdx.x; p < kMapFloats / 4; p += blockDim.x) {
            const int i = p >> 4, q = p & 15;
            const float xi = sc[3 * i], yi = sc[3 * i + 1], zi = sc[3 * i + 2];
            float d[4];
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const int j = 4 * q + t;
                const float dx = xi - sc[3 * j], dy = yi - sc[3 * j + 1], dz = zi - sc[3 * j + 2];
                d[t] = sqrtf(fmaf(dz, dz, fmaf(dy, dy, dx * dx)));
            }
            __stcs(reinterpret_cast<float4 *>(out + 4 * p), make_float4(d[0], d[1], d[2], d[3]));
        }
        __syncthreads();
    }
}

int sms() {
    int dev = 0, n = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}

}  // namespace

cudaError_t launch_mds(const float *maps, int64_t n, float *coords, float *eigvals, uint32_t *flags,
                       cudaStream_t st) {
    if (n <= 0) return cudaSuccess;
    const size_t smem = sizeof(float) * (size_t)kMdsWarps * (kN * kLd + kN * 4 + kN);
    cudaError_t e = cudaFuncSetAttribute(mds_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, mds_kernel, kMdsWarps * 32, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) per_sm = 1;
    int64_t grid = (n + kMdsWarps - 1) / kMdsWarps;
    const int64_t cap = (int64_t)sms() * per_sm;
    if (grid > cap) grid = cap;
    mds_kernel<<<(int)grid, kMdsWarps * 32, smem, st>>>(maps, n, coords, eigvals, flags);
    return cudaGetLastError();
}

cudaError_t launch_pdist(const float *coords, int64_t n, float *maps, cudaStream_t st) {
    if (n <= 0) return cudaSuccess;
    int64_t grid = n;
    const int64_t cap = (int64_t)sms() * 8;
    if (grid > cap) grid = cap;
    pdist_kernel<<<(int)grid, 256, 0, st>>>(coords, n, maps);
    return cudaGetLastError();
}

}  // namespace tdm
