// Coordinate recovery: classical MDS (one warp per map) and pairwise distances.
//
// ParaChromo (mdpi.com/2079-9292/15/13/2750) recovers a 64-bead point cloud from
// each final distance map by distance-geometry initialisation (§3.1, §5.5).  The
// reading used is classical MDS: B = -1/2 J (D*D) J, the top three eigenpairs,
// x_k = v_k sqrt(max(l_k, 0)).
//
// Per map, one warp stages D in shared memory by 16-byte asynchronous copies
// (the warp's next map is brought into L2 by one bulk prefetch issued when the
// current map's eigen-solve is done, so those copies wait on L2 rather than
// DRAM) and forms B.  The top
// eigenpairs come from subspace iteration on three vectors with a
// Rayleigh-Ritz step (a 3 x 3 Jacobi eigen-solve) every iteration, stopping
// when the residual of the three Ritz pairs is below kTol * |l_1|.  The start
// basis is the three columns of B with the largest diagonal entries (the
// points farthest from the centroid): for an exact Euclidean map they already
// span the answer.  Row l of B stays in registers for the products; row l+32
// is read from shared memory.
#include "common.cuh"

namespace tdm {
namespace {

constexpr int kMdsWarps = 4;
constexpr int kLd = kN + 4;       // smem row stride: 16-byte rows; row float4 and column reads conflict-free
constexpr int kK = 3;             // subspace dimension
constexpr int kMaxIt = 48;
constexpr float kTol = 4e-6f;

__device__ __forceinline__ float wsum(float v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

__device__ __forceinline__ float rcp_approx(float x) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}
__device__ __forceinline__ float rsqrt_approx(float x) {
    float r;
    asm("rsqrt.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// Gram-Schmidt applied twice per column ("twice is enough") on 64 x kK
// columns held as rows (l, l+32) per lane.
__device__ __forceinline__ void orthonormalize(float (&a0)[kK], float (&a1)[kK]) {
#pragma unroll
    for (int c = 0; c < kK; ++c) {
#pragma unroll
        for (int pass = 0; pass < 2; ++pass) {
            float d[kK];
#pragma unroll
            for (int p = 0; p < c; ++p) d[p] = wsum(fmaf(a0[p], a0[c], a1[p] * a1[c]));
#pragma unroll
            for (int p = 0; p < c; ++p) {
                a0[c] = fmaf(-d[p], a0[p], a0[c]);
                a1[c] = fmaf(-d[p], a1[p], a1[c]);
            }
        }
        const float nn = wsum(fmaf(a0[c], a0[c], a1[c] * a1[c]));
        const float inv = nn > 1e-37f ? rsqrt_approx(nn) : 0.0f;
        a0[c] *= inv;
        a1[c] *= inv;
    }
}

// One Jacobi rotation zeroing H[P][Q] of the symmetric kK x kK H (both
// halves kept), accumulated into Y (Golub & Van Loan §8.5: the symmetric 2 x 2
// Schur step, with the diagonal updated by t * H[P][Q]).
template <int P, int Q>
__device__ __forceinline__ void jrot(float (&H)[kK][kK], float (&Y)[kK][kK]) {
    const float apq = H[P][Q];
    if (!(fabsf(apq) > 1e-9f * (fabsf(H[P][P]) + fabsf(H[Q][Q])))) return;
    const float theta = (H[Q][Q] - H[P][P]) * 0.5f * rcp_approx(apq);
    const float r2 = fmaf(theta, theta, 1.0f);
    const float t = copysignf(rcp_approx(fabsf(theta) + r2 * rsqrt_approx(r2)), theta);
    const float c = rsqrt_approx(fmaf(t, t, 1.0f));
    const float s = t * c;
    H[P][P] = fmaf(-t, apq, H[P][P]);
    H[Q][Q] = fmaf(t, apq, H[Q][Q]);
    H[P][Q] = H[Q][P] = 0.0f;
#pragma unroll
    for (int k = 0; k < kK; ++k) {
        if (k == P || k == Q) continue;
        const float hp = H[k][P], hq = H[k][Q];
        H[k][P] = H[P][k] = fmaf(c, hp, -s * hq);
        H[k][Q] = H[Q][k] = fmaf(s, hp, c * hq);
    }
#pragma unroll
    for (int k = 0; k < kK; ++k) {
        const float yp = Y[k][P], yq = Y[k][Q];
        Y[k][P] = fmaf(c, yp, -s * yq);
        Y[k][Q] = fmaf(s, yp, c * yq);
    }
}

template <int I, int J>
__device__ __forceinline__ void sort_pair(float (&th)[kK], float (&Y)[kK][kK]) {
    if (th[I] < th[J]) {
        const float tt = th[I];
        th[I] = th[J];
        th[J] = tt;
#pragma unroll
        for (int k = 0; k < kK; ++k) {
            const float y = Y[k][I];
            Y[k][I] = Y[k][J];
            Y[k][J] = y;
        }
    }
}

// Cyclic Jacobi on a symmetric 3 x 3 matrix; eigenvalues sorted in descending
// order, eigenvectors in the columns of Y.
__device__ __forceinline__ void eig3(float (&H)[kK][kK], float (&Y)[kK][kK], float (&th)[kK]) {
#pragma unroll
    for (int i = 0; i < kK; ++i)
#pragma unroll
        for (int j = 0; j < kK; ++j) Y[i][j] = i == j ? 1.0f : 0.0f;
    for (int sweep = 0; sweep < 12; ++sweep) {
        const float off = H[0][1] * H[0][1] + H[0][2] * H[0][2] + H[1][2] * H[1][2];
        const float dia = H[0][0] * H[0][0] + H[1][1] * H[1][1] + H[2][2] * H[2][2];
        if (off <= 1e-14f * dia) break;
        jrot<0, 1>(H, Y);
        jrot<0, 2>(H, Y);
        jrot<1, 2>(H, Y);
    }
#pragma unroll
    for (int i = 0; i < kK; ++i) th[i] = H[i][i];
    sort_pair<0, 1>(th, Y);
    sort_pair<1, 2>(th, Y);
    sort_pair<0, 1>(th, Y);
}

// (value, index) of the warp-wide maximum; ties go to the lower index.
__device__ __forceinline__ void warp_argmax(float &v, int &i) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, v, off);
        const int oi = __shfl_xor_sync(0xffffffffu, i, off);
        if (ov > v || (ov == v && oi < i)) {
            v = ov;
            i = oi;
        }
    }
}

__device__ __forceinline__ float sqrt_approx(float x) {
    float r;
    asm("sqrt.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

template <bool DIST>
__global__ void __launch_bounds__(kMdsWarps * 32, 3) mds_kernel(const float *__restrict__ maps, int64_t n,
                                                                float *__restrict__ coords,
                                                                float *__restrict__ eig,
                                                                uint32_t *__restrict__ flags,
                                                                float *__restrict__ dist) {
    extern __shared__ __align__(16) float smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float *sD = smem + warp * (kN * kLd);
    // V as (c0, c1) pairs and c2 values: a broadcast 64-bit load is served
    // per half warp and a 32-bit one per warp (3 wavefronts per row of V
    // against 4 for a 128-bit broadcast)
    float2 *sV01 = reinterpret_cast<float2 *>(smem + kMdsWarps * kN * kLd) + warp * kN * 2;
    float *sV2 = reinterpret_cast<float *>(sV01 + kN);
    float *sR = smem + kMdsWarps * kN * kLd + kMdsWarps * kN * 4 + warp * kN;
    const int i0 = lane, i1 = lane + 32;

    for (int64_t m = (int64_t)blockIdx.x * kMdsWarps + warp; m < n; m += (int64_t)gridDim.x * kMdsWarps) {
        const float *D = maps + m * kMapFloats;
        {   // the map into shared memory by 16-byte asynchronous copies, all in flight at once
            const uint32_t base = static_cast<uint32_t>(__cvta_generic_to_shared(sD));
#pragma unroll
            for (int it = 0; it < 32; ++it) {
                const int idx = it * 32 + lane;
                const int row = idx >> 4, c4 = (idx & 15) << 2;
                asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(base + 4u * (row * kLd + c4)),
                             "l"(D + row * kN + c4)
                             : "memory");
            }
            asm volatile("cp.async.commit_group;\n\tcp.async.wait_all;" ::: "memory");
        }
        __syncwarp();

        // e_ij = D_ij + D_ji (twice the symmetric part); S = (e/2)^2, so
        // B = -1/2 J S J = -1/8 J (e*e) J.  Lane l forms e*e of rows i0 and
        // i1 in registers from row reads (float4) and column reads (lane l
        // reads column l or l+32 of row j: consecutive words), all before any
        // write, so no element is overwritten while another lane reads it.
        float t0[kN], t1[kN];
        float rs0 = 0.0f, rs1 = 0.0f;
#pragma unroll
        for (int j4 = 0; j4 < kN / 4; ++j4) {
            const float4 a = *reinterpret_cast<const float4 *>(sD + i0 * kLd + 4 * j4);
            const float4 b = *reinterpret_cast<const float4 *>(sD + i1 * kLd + 4 * j4);
            const float ra[4] = {a.x, a.y, a.z, a.w}, rb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int j = 4 * j4 + u;
                const float e0 = ra[u] + sD[j * kLd + i0], e1 = rb[u] + sD[j * kLd + i1];
                t0[j] = e0 * e0;
                t1[j] = e1 * e1;
            }
            // row sums in the order of a float4 pass over the rows
            rs0 += (t0[4 * j4] + t0[4 * j4 + 1]) + (t0[4 * j4 + 2] + t0[4 * j4 + 3]);
            rs1 += (t1[4 * j4] + t1[4 * j4 + 1]) + (t1[4 * j4 + 2] + t1[4 * j4 + 3]);
        }
        const float r0 = rs0 * (1.0f / kN), r1 = rs1 * (1.0f / kN);
        const float gm = wsum(r0 + r1) * (1.0f / kN);
        // exact power-of-two scale bringing the mean of e*e to O(1); undone on
        // the eigenvalues
        int ex = 0;
        frexpf(gm, &ex);
        const float scale = gm > 0.0f && isfinite(gm) ? ldexpf(1.0f, -ex) : 1.0f;
        const float cs = -0.125f * scale;
        sR[i0] = r0;
        sR[i1] = r1;
        __syncwarp();    // every lane's reads of D are done: rows of B may replace it
        // double centring: B_ij = cs (e2_ij - r_i - r_j + g); row i0 of B is
        // also kept in registers for the products
        const float g0 = gm - r0, g1 = gm - r1;
        float *b0 = t0;
#pragma unroll
        for (int j4 = 0; j4 < kN / 4; ++j4) {
            const float4 rj = *reinterpret_cast<const float4 *>(sR + 4 * j4);
            float4 a, b;
            a.x = cs * ((t0[4 * j4] + g0) - rj.x);
            a.y = cs * ((t0[4 * j4 + 1] + g0) - rj.y);
            a.z = cs * ((t0[4 * j4 + 2] + g0) - rj.z);
            a.w = cs * ((t0[4 * j4 + 3] + g0) - rj.w);
            b.x = cs * ((t1[4 * j4] + g1) - rj.x);
            b.y = cs * ((t1[4 * j4 + 1] + g1) - rj.y);
            b.z = cs * ((t1[4 * j4 + 2] + g1) - rj.z);
            b.w = cs * ((t1[4 * j4 + 3] + g1) - rj.w);
            b0[4 * j4] = a.x;
            b0[4 * j4 + 1] = a.y;
            b0[4 * j4 + 2] = a.z;
            b0[4 * j4 + 3] = a.w;
            *reinterpret_cast<float4 *>(sD + i0 * kLd + 4 * j4) = a;
            *reinterpret_cast<float4 *>(sD + i1 * kLd + 4 * j4) = b;
        }
        __syncwarp();

        // start basis: the columns of the kK largest diagonal entries
        float v0[kK], v1[kK];
        {
            float d0 = sD[i0 * kLd + i0], d1 = sD[i1 * kLd + i1];
#pragma unroll
            for (int c = 0; c < kK; ++c) {
                float bv = d0 >= d1 ? d0 : d1;
                int bi = d0 >= d1 ? i0 : i1;
                warp_argmax(bv, bi);
                if (bi == i0) d0 = -INFINITY;
                if (bi == i1) d1 = -INFINITY;
                v0[c] = sD[bi * kLd + i0];     // B[i0][bi] = B[bi][i0]
                v1[c] = sD[bi * kLd + i1];
            }
        }
        orthonormalize(v0, v1);
        sV01[i0] = make_float2(v0[0], v0[1]);
        sV01[i1] = make_float2(v1[0], v1[1]);
        sV2[i0] = v0[2];
        sV2[i1] = v1[2];

        float th[kK] = {0.f, 0.f, 0.f};
        float u0[kK], u1[kK];
        bool conv = false;
        const float *bh = sD + i1 * kLd;
        for (int it = 0; it < kMaxIt; ++it) {
            __syncwarp();
            float w0[kK] = {0.f, 0.f, 0.f}, w1[kK] = {0.f, 0.f, 0.f};
#pragma unroll
            for (int j4 = 0; j4 < kN / 4; ++j4) {
                const float4 x1 = *reinterpret_cast<const float4 *>(bh + 4 * j4);
                const float xb[4] = {x1.x, x1.y, x1.z, x1.w};
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    const float2 v01 = sV01[4 * j4 + t];
                    const float4 v = make_float4(v01.x, v01.y, sV2[4 * j4 + t], 0.0f);
                    const float xa = b0[4 * j4 + t];
                    w0[0] = fmaf(xa, v.x, w0[0]);
                    w0[1] = fmaf(xa, v.y, w0[1]);
                    w0[2] = fmaf(xa, v.z, w0[2]);
                    w1[0] = fmaf(xb[t], v.x, w1[0]);
                    w1[1] = fmaf(xb[t], v.y, w1[1]);
                    w1[2] = fmaf(xb[t], v.z, w1[2]);
                }
            }
            // Rayleigh quotient H = V^T B V (symmetrised)
            float H[kK][kK];
#pragma unroll
            for (int a = 0; a < kK; ++a)
#pragma unroll
                for (int b = a; b < kK; ++b) {
                    const float h = 0.5f * wsum(fmaf(v0[a], w0[b], fmaf(v0[b], w0[a],
                                                     fmaf(v1[a], w1[b], v1[b] * w1[a]))));
                    H[a][b] = h;
                    H[b][a] = h;
                }
            float Y[kK][kK];
            eig3(H, Y, th);
            float bu0[kK], bu1[kK];
#pragma unroll
            for (int c = 0; c < kK; ++c) {
                u0[c] = u1[c] = bu0[c] = bu1[c] = 0.0f;
#pragma unroll
                for (int a = 0; a < kK; ++a) {
                    u0[c] = fmaf(v0[a], Y[a][c], u0[c]);
                    u1[c] = fmaf(v1[a], Y[a][c], u1[c]);
                    bu0[c] = fmaf(w0[a], Y[a][c], bu0[c]);
                    bu1[c] = fmaf(w1[a], Y[a][c], bu1[c]);
                }
            }
            float rmax = 0.0f;
#pragma unroll
            for (int c = 0; c < kK; ++c) {
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
            for (int c = 0; c < kK; ++c) {
                v0[c] = bu0[c];
                v1[c] = bu1[c];
            }
            __syncwarp();
            sV01[i0] = make_float2(v0[0], v0[1]);
            sV01[i1] = make_float2(v1[0], v1[1]);
            sV2[i0] = v0[2];
            sV2[i1] = v1[2];
        }
        {   // the warp's next map into L2 while this one's coordinates and
            // distances are written (issued at the start of the map, or before
            // the eigen-solve, it measured slower)
            const int64_t mn = m + (int64_t)gridDim.x * kMdsWarps;
            if (lane == 0 && mn < n)
                asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(maps + mn * kMapFloats),
                             "r"((unsigned)(kMapFloats * sizeof(float)))
                             : "memory");
        }
        if (!conv && lane == 0) atomicOr(flags, (uint32_t)TDM_FLAG_MDS_NOT_CONVERGED);

        const float inv_scale = 1.0f / scale;
        float *X = coords + m * (kN * 3);
#pragma unroll
        for (int c = 0; c < kK; ++c) {
            const float sq = sqrtf(fmaxf(th[c], 0.0f) * inv_scale);
            X[i0 * 3 + c] = u0[c] * sq;
            X[i1 * 3 + c] = u1[c] * sq;
        }
        if (eig != nullptr && lane < 3) eig[m * 3 + lane] = (lane == 0 ? th[0] : lane == 1 ? th[1] : th[2]) * inv_scale;
        if (DIST) {
            // the distance map of the coordinates, as pdist_kernel computes it:
            // the coordinates go to shared memory (the V arrays are free now),
            // then row r is written by the whole warp, two columns per lane,
            // with coalesced 8-byte streaming stores
            float *sc = reinterpret_cast<float *>(sV01);    // x[64], y[64], z[64]
            __syncwarp();
#pragma unroll
            for (int c = 0; c < kK; ++c) {
                const float sq = sqrtf(fmaxf(th[c], 0.0f) * inv_scale);
                sc[c * kN + i0] = u0[c] * sq;
                sc[c * kN + i1] = u1[c] * sq;
            }
            __syncwarp();
            const float2 cx = reinterpret_cast<const float2 *>(sc)[lane];
            const float2 cy = reinterpret_cast<const float2 *>(sc + kN)[lane];
            const float2 cz = reinterpret_cast<const float2 *>(sc + 2 * kN)[lane];
            float2 *out = reinterpret_cast<float2 *>(dist + m * kMapFloats) + lane;
#pragma unroll 8
            for (int row = 0; row < kN; ++row) {
                const float xi = sc[row], yi = sc[kN + row], zi = sc[2 * kN + row];
                float2 d;
                d.x = sqrt_approx(fmaf(zi - cz.x, zi - cz.x, fmaf(yi - cy.x, yi - cy.x, (xi - cx.x) * (xi - cx.x))));
                d.y = sqrt_approx(fmaf(zi - cz.y, zi - cz.y, fmaf(yi - cy.y, yi - cy.y, (xi - cx.y) * (xi - cx.y))));
                __stcs(out + row * (kN / 2), d);
            }
        }
        __syncwarp();
    }
}

// Distance reconstruction: kPdistMaps maps per CTA iteration, their
// coordinates staged as structure of arrays (x[64], y[64], z[64] per map) so
// that a thread's four columns are one conflict-free 128-bit load per axis;
// each thread writes 4 float4 of every staged map with streaming stores.  The
// square root is sqrt.approx (relative error about 2^-23; exact 0 on the
// diagonal).
constexpr int kPdistMaps = 4;


__global__ void __launch_bounds__(256) pdist_kernel(const float *__restrict__ coords, int64_t n,
                                                    float *__restrict__ maps) {
    __shared__ __align__(16) float sc[kPdistMaps][3][kN];
    for (int64_t m0 = (int64_t)blockIdx.x * kPdistMaps; m0 < n; m0 += (int64_t)gridDim.x * kPdistMaps) {
        const int nm = (int)min((int64_t)kPdistMaps, n - m0);
        for (int t = threadIdx.x; t < nm * kN * 3; t += blockDim.x) {
            const int mm = t / (kN * 3), e = t - mm * (kN * 3);
            sc[mm][e % 3][e / 3] = __ldg(coords + (m0 + mm) * (kN * 3) + e);
        }
        __syncthreads();
        for (int mm = 0; mm < nm; ++mm) {
            float *out = maps + (m0 + mm) * kMapFloats;
#pragma unroll
            for (int it = 0; it < kMapFloats / 4 / 256; ++it) {
                const int p = threadIdx.x + it * 256;
                const int i = p >> 4, q = p & 15;
                const float xi = sc[mm][0][i], yi = sc[mm][1][i], zi = sc[mm][2][i];
                const float4 xj = reinterpret_cast<const float4 *>(sc[mm][0])[q];
                const float4 yj = reinterpret_cast<const float4 *>(sc[mm][1])[q];
                const float4 zj = reinterpret_cast<const float4 *>(sc[mm][2])[q];
                float4 d;
                d.x = sqrt_approx(fmaf(zi - zj.x, zi - zj.x, fmaf(yi - yj.x, yi - yj.x, (xi - xj.x) * (xi - xj.x))));
                d.y = sqrt_approx(fmaf(zi - zj.y, zi - zj.y, fmaf(yi - yj.y, yi - yj.y, (xi - xj.y) * (xi - xj.y))));
                d.z = sqrt_approx(fmaf(zi - zj.z, zi - zj.z, fmaf(yi - yj.z, yi - yj.z, (xi - xj.z) * (xi - xj.z))));
                d.w = sqrt_approx(fmaf(zi - zj.w, zi - zj.w, fmaf(yi - yj.w, yi - yj.w, (xi - xj.w) * (xi - xj.w))));
                __stcs(reinterpret_cast<float4 *>(out + 4 * p), d);
            }
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

cudaError_t launch_mds(const float *maps, int64_t n, float *coords, float *eigvals, uint32_t *flags, float *dist,
                       cudaStream_t st) {
    if (n <= 0) return cudaSuccess;
    const size_t smem = sizeof(float) * (size_t)kMdsWarps * (kN * kLd + kN * 4 + kN);
    static_assert((kMdsWarps * kN * kLd * sizeof(float)) % 16 == 0, "float4 alignment of the V tiles");
    const void *kern = dist != nullptr ? reinterpret_cast<const void *>(mds_kernel<true>)
                                       : reinterpret_cast<const void *>(mds_kernel<false>);
    LaunchShape shape;
    const cudaError_t e = launch_shape(kern, kMdsWarps * 32, smem, &shape);
    if (e != cudaSuccess) return e;
    int64_t grid = (n + kMdsWarps - 1) / kMdsWarps;
    const int64_t cap = (int64_t)shape.sms * shape.per_sm;
    if (grid > cap) grid = cap;
    if (dist != nullptr)
        mds_kernel<true><<<(int)grid, kMdsWarps * 32, smem, st>>>(maps, n, coords, eigvals, flags, dist);
    else
        mds_kernel<false><<<(int)grid, kMdsWarps * 32, smem, st>>>(maps, n, coords, eigvals, flags, nullptr);
    return cudaGetLastError();
}

cudaError_t launch_pdist(const float *coords, int64_t n, float *maps, cudaStream_t st) {
    if (n <= 0) return cudaSuccess;
    int64_t grid = (n + kPdistMaps - 1) / kPdistMaps;
    const int64_t cap = (int64_t)sms() * 8;
    if (grid > cap) grid = cap;
    pdist_kernel<<<(int)grid, 256, 0, st>>>(coords, n, maps);
    return cudaGetLastError();
}

}  // namespace tdm
