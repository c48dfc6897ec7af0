// Coordinate recovery: classical MDS (one warp per map) and pairwise distances.
//
// ParaChromo (mdpi.com/2079-9292/15/13/2750) recovers a 64-bead point cloud from
// each final distance map by distance-geometry initialisation (§3.1, §5.5).  The
// reading used is classical MDS: B = -1/2 J (D*D) J, the top three eigenpairs,
// x_k = v_k sqrt(max(l_k, 0)).
//
// Per map, one warp stages D in shared memory by 16-byte asynchronous copies
// and forms B = -1/8 J E J from E = (D + D^T)^2 entrywise.  The copies of the
// warp's next map go into the same tile as soon as this map's rows are done
// with: rows 0-31 once the start basis is formed (row l of B is in
// registers), rows 32-63 once the eigen-solve has converged.  The top
// eigenpairs come from subspace iteration on three vectors with a
// Rayleigh-Ritz step (a 3 x 3 Jacobi eigen-solve) every iteration, stopping
// when the residual of the three Ritz pairs is below kTol * |l_1|.  The start
// basis is the three columns of B with the largest diagonal entries (the
// points farthest from the centroid): for an exact Euclidean map they already
// span the answer.  Row l of B stays in registers for the products; row l+32
// is read from shared memory.  Forming B and the products run in packed
// float32 (two columns per instruction), which halves their instructions.
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
__device__ __forceinline__ float sqrt_approx(float x) {
    float r;
    asm("sqrt.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// Gram-Schmidt applied twice per column ("twice is enough") on 64 x kK
// columns held as rows (l, l+32) per lane, in the classical form with the
// dot products of a round reduced together: four rounds of warp reductions
// instead of one per dot product.  Round 1 projects a_0 out of a_1 and a_2;
// round 2 projects it out again and a_1 out of a_2; round 3 projects both
// out of a_2 again; round 4 normalises.  A column that vanishes becomes zero.
__device__ __forceinline__ void orthonormalize(float (&a0)[kK], float (&a1)[kK]) {
    const auto dot = [&](int p, int q) { return fmaf(a0[p], a0[q], a1[p] * a1[q]); };
    const auto axpy = [&](float f, int p, int q) {    // a_q -= f a_p
        a0[q] = fmaf(-f, a0[p], a0[q]);
        a1[q] = fmaf(-f, a1[p], a1[q]);
    };
    const float g00 = wsum(dot(0, 0)), g01 = wsum(dot(0, 1)), g02 = wsum(dot(0, 2));
    const float i00 = g00 > 1e-37f ? rcp_approx(g00) : 0.0f;
    axpy(g01 * i00, 0, 1);
    axpy(g02 * i00, 0, 2);
    const float r01 = wsum(dot(0, 1)), r02 = wsum(dot(0, 2)), g11 = wsum(dot(1, 1)), g12 = wsum(dot(1, 2));
    axpy(r01 * i00, 0, 1);
    axpy(r02 * i00, 0, 2);
    const float i11 = g11 > 1e-37f ? rcp_approx(g11) : 0.0f;
    axpy(g12 * i11, 1, 2);
    const float p02 = wsum(dot(0, 2)), p12 = wsum(dot(1, 2));
    axpy(p02 * i00, 0, 2);
    axpy(p12 * i11, 1, 2);
    const float n1 = wsum(dot(1, 1)), n2 = wsum(dot(2, 2));
    const float s0 = g00 > 1e-37f ? rsqrt_approx(g00) : 0.0f;
    const float s1 = n1 > 1e-37f ? rsqrt_approx(n1) : 0.0f;
    const float s2 = n2 > 1e-37f ? rsqrt_approx(n2) : 0.0f;
    a0[0] *= s0;
    a1[0] *= s0;
    a0[1] *= s1;
    a1[1] *= s1;
    a0[2] *= s2;
    a1[2] *= s2;
}

// Orthonormalises the kK columns Y (rows (l, l+32) per lane) whose Gram
// matrix G = Y^T Y is given: Y diag(s) is nearly orthonormal when the columns
// are nearly orthogonal, whatever their scale, and Cholesky QR of the scaled
// Gram matrix (a 3 x 3 factorisation done by every lane) then needs no further
// reduction.  A column whose norm or pivot vanishes becomes zero, as in
// orthonormalize.  Returns the largest off-diagonal of the scaled Gram matrix,
// a measure of how far from orthogonal the columns were.
__device__ __forceinline__ float cholqr(float (&a0)[kK], float (&a1)[kK], const float (&G)[kK][kK]) {
    float sc[kK];
#pragma unroll
    for (int c = 0; c < kK; ++c) sc[c] = G[c][c] > 1e-37f ? rsqrt_approx(G[c][c]) : 0.0f;
    const float g01 = G[0][1] * sc[0] * sc[1], g02 = G[0][2] * sc[0] * sc[2], g12 = G[1][2] * sc[1] * sc[2];
    const float g00 = G[0][0] * sc[0] * sc[0], g11 = G[1][1] * sc[1] * sc[1], g22 = G[2][2] * sc[2] * sc[2];
    // G' = L L^T; the new columns are Y diag(sc) L^-T, by forward substitution
    const float p0 = g00;
    const float i0 = p0 > 1e-12f ? rsqrt_approx(p0) : 0.0f;
    const float l10 = g01 * i0, l20 = g02 * i0;
    const float p1 = fmaf(-l10, l10, g11);
    const float i1 = p1 > 1e-12f ? rsqrt_approx(p1) : 0.0f;
    const float l21 = fmaf(-l20, l10, g12) * i1;
    const float p2 = fmaf(-l21, l21, fmaf(-l20, l20, g22));
    const float i2 = p2 > 1e-12f ? rsqrt_approx(p2) : 0.0f;
    const float y0a = a0[0] * sc[0], y0b = a1[0] * sc[0];
    const float y1a = a0[1] * sc[1], y1b = a1[1] * sc[1];
    const float y2a = a0[2] * sc[2], y2b = a1[2] * sc[2];
    a0[0] = y0a * i0;
    a1[0] = y0b * i0;
    a0[1] = fmaf(-l10, a0[0], y1a) * i1;
    a1[1] = fmaf(-l10, a1[0], y1b) * i1;
    a0[2] = fmaf(-l21, a0[1], fmaf(-l20, a0[0], y2a)) * i2;
    a1[2] = fmaf(-l21, a1[1], fmaf(-l20, a1[0], y2b)) * i2;
    return fmaxf(fabsf(g01), fmaxf(fabsf(g02), fabsf(g12)));
}

// The Gram matrix of the kK columns (rows (l, l+32) per lane), reduced over the warp.
__device__ __forceinline__ void gram(const float (&a0)[kK], const float (&a1)[kK], float (&G)[kK][kK]) {
#pragma unroll
    for (int a = 0; a < kK; ++a)
#pragma unroll
        for (int b = a; b < kK; ++b) {
            const float g = wsum(fmaf(a0[a], a0[b], a1[a] * a1[b]));
            G[a][b] = g;
            G[b][a] = g;
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


// Shared memory of one warp: B (the staged D first) at row stride kLd, V as
// three columns of 64 (structure of arrays), and the row means of E.
constexpr int kWarpFloats = kN * kLd + 3 * kN + kN;

// asynchronous 16-byte copies of rows [32 h, 32 h + 32) of map D into the
// padded tile, committed as one group
__device__ __forceinline__ void stage_half(float *sD, const float *D, int h, int lane) {
    const uint32_t base = static_cast<uint32_t>(__cvta_generic_to_shared(sD));
#pragma unroll
    for (int it = 0; it < 16; ++it) {
        const int idx = it * 32 + lane;
        const int row = 32 * h + (idx >> 4), c4 = (idx & 15) << 2;
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(base + 4u * (row * kLd + c4)),
                     "l"(D + row * kN + c4)
                     : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
}

template <bool DIST>
__global__ void __launch_bounds__(kMdsWarps * 32, 3) mds_kernel(const float *__restrict__ maps, int64_t n,
                                                                float *__restrict__ coords,
                                                                float *__restrict__ eig,
                                                                uint32_t *__restrict__ flags,
                                                                float *__restrict__ dist) {
    extern __shared__ __align__(16) float smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float *sE = smem + warp * kWarpFloats;
    float *sV = sE + kN * kLd;     // v_c[64] for c = 0, 1, 2
    float *sR = sV + 3 * kN;       // row means of E, negated
    const int i0 = lane, i1 = lane + 32;

    const int64_t stride = (int64_t)gridDim.x * kMdsWarps;
    int64_t m = (int64_t)blockIdx.x * kMdsWarps + warp;
    if (m < n) {
        stage_half(sE, maps + m * kMapFloats, 0, lane);
        stage_half(sE, maps + m * kMapFloats, 1, lane);
    }
    for (; m < n; m += stride) {
        const int64_t mn = m + stride;    // the warp's next map
        asm volatile("cp.async.wait_all;" ::: "memory");
        __syncwarp();

        // e_ij = D_ij + D_ji (twice the symmetric part) and E = e*e, so that
        // B = -1/2 J (e/2)^2 J = -1/8 J E J.  Lane l forms rows i0 and i1 of E
        // from row reads (float4) and column reads (lane l reads column l or
        // l+32 of row j: consecutive words), as column pairs (2p, 2p+1) in
        // packed float32, all before any write.  E is symmetric bit for bit,
        // since e_ij and e_ji are the same sum.
        float2 t0[kN / 2], t1[kN / 2];
        float2 rs0 = make_float2(0.f, 0.f), rs1 = make_float2(0.f, 0.f);
#pragma unroll
        for (int j4 = 0; j4 < kN / 4; ++j4) {
            const float4 a = ld4(sE + i0 * kLd + 4 * j4);
            const float4 b = ld4(sE + i1 * kLd + 4 * j4);
            float ca[4], cb[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                ca[u] = sE[(4 * j4 + u) * kLd + i0];
                cb[u] = sE[(4 * j4 + u) * kLd + i1];
            }
            const float2 ea = __fadd2_rn(make_float2(a.x, a.y), make_float2(ca[0], ca[1]));
            const float2 eb = __fadd2_rn(make_float2(a.z, a.w), make_float2(ca[2], ca[3]));
            const float2 fa = __fadd2_rn(make_float2(b.x, b.y), make_float2(cb[0], cb[1]));
            const float2 fb = __fadd2_rn(make_float2(b.z, b.w), make_float2(cb[2], cb[3]));
            t0[2 * j4] = __fmul2_rn(ea, ea);
            t0[2 * j4 + 1] = __fmul2_rn(eb, eb);
            t1[2 * j4] = __fmul2_rn(fa, fa);
            t1[2 * j4 + 1] = __fmul2_rn(fb, fb);
            rs0 = __fadd2_rn(rs0, __fadd2_rn(t0[2 * j4], t0[2 * j4 + 1]));
            rs1 = __fadd2_rn(rs1, __fadd2_rn(t1[2 * j4], t1[2 * j4 + 1]));
        }
        const float r0 = (rs0.x + rs0.y) * (1.0f / kN), r1 = (rs1.x + rs1.y) * (1.0f / kN);
        const float gm = wsum(r0 + r1) * (1.0f / kN);
        // exact power-of-two scale bringing the mean of E to O(1); undone on
        // the eigenvalues
        int ex = 0;
        frexpf(gm, &ex);
        const bool scaled = gm > 0.0f && isfinite(gm);
        const float scale = scaled ? ldexpf(1.0f, -ex) : 1.0f;
        const float inv_scale = scaled ? ldexpf(1.0f, ex) : 1.0f;    // exact: a power of two
        const float cs = -0.125f * scale;
        sR[i0] = -r0;    // negated: a - r is the packed sum a + (-r), rounded as the difference
        sR[i1] = -r1;
        __syncwarp();    // every lane's reads of D are done: rows of B may replace it
        // double centring B_ij = cs ((E_ij + g_i) - r_j), g_i = g - r_i, in
        // packed pairs; row i0 of B stays in registers for the products.  The
        // centring is explicit because B annihilates the ones vector to
        // rounding: a basis vector that is rounding noise (the null direction
        // of a planar or collinear map) then does no harm.
        const float2 cs2 = make_float2(cs, cs);
        const float2 g0 = make_float2(gm - r0, gm - r0), g1 = make_float2(gm - r1, gm - r1);
#pragma unroll
        for (int j4 = 0; j4 < kN / 4; ++j4) {
            const float4 rj = ld4(sR + 4 * j4);
            const float2 ra = make_float2(rj.x, rj.y), rb = make_float2(rj.z, rj.w);
            t0[2 * j4] = __fmul2_rn(cs2, __fadd2_rn(__fadd2_rn(t0[2 * j4], g0), ra));
            t0[2 * j4 + 1] = __fmul2_rn(cs2, __fadd2_rn(__fadd2_rn(t0[2 * j4 + 1], g0), rb));
            const float2 c = __fmul2_rn(cs2, __fadd2_rn(__fadd2_rn(t1[2 * j4], g1), ra));
            const float2 d = __fmul2_rn(cs2, __fadd2_rn(__fadd2_rn(t1[2 * j4 + 1], g1), rb));
            st4(sE + i0 * kLd + 4 * j4, make_float4(t0[2 * j4].x, t0[2 * j4].y, t0[2 * j4 + 1].x, t0[2 * j4 + 1].y));
            st4(sE + i1 * kLd + 4 * j4, make_float4(c.x, c.y, d.x, d.y));
        }
        __syncwarp();

        // start basis: the columns of the kK largest diagonal entries of B
        // (the points farthest from the centroid)
        float v0[kK], v1[kK];
        {
            float d0 = sE[i0 * kLd + i0], d1 = sE[i1 * kLd + i1];
#pragma unroll
            for (int c = 0; c < kK; ++c) {
                float bv = d0 >= d1 ? d0 : d1;
                int bi = d0 >= d1 ? i0 : i1;
                warp_argmax(bv, bi);
                if (bi == i0) d0 = -INFINITY;
                if (bi == i1) d1 = -INFINITY;
                v0[c] = sE[bi * kLd + i0];     // B[i0][bi] = B[bi][i0]
                v1[c] = sE[bi * kLd + i1];
            }
        }
        // rows 0-31 of B are no longer read (row i0 is in registers): the next
        // map's first half goes there while this one's eigen-solve runs
        __syncwarp();
        if (mn < n) {
            stage_half(sE, maps + mn * kMapFloats, 0, lane);
        }
        orthonormalize(v0, v1);
#pragma unroll
        for (int c = 0; c < kK; ++c) {
            sV[c * kN + i0] = v0[c];
            sV[c * kN + i1] = v1[c];
        }

        float th[kK] = {0.f, 0.f, 0.f};
        float u0[kK], u1[kK];
        bool conv = false;
        const float *bh = sE + i1 * kLd;
        for (int it = 0; it < kMaxIt; ++it) {
            __syncwarp();
            // W = B V: row i0 of B from registers, row i1 from shared memory,
            // V broadcast four rows at a time; even and odd columns accumulate
            // in the two halves of a packed pair
            float2 a0[kK], a1[kK];
#pragma unroll
            for (int c = 0; c < kK; ++c) a0[c] = a1[c] = make_float2(0.f, 0.f);
#pragma unroll
            for (int j4 = 0; j4 < kN / 4; ++j4) {
                const float4 e1 = ld4(bh + 4 * j4);
#pragma unroll
                for (int c = 0; c < kK; ++c) {
                    const float4 v = ld4(sV + c * kN + 4 * j4);
                    a0[c] = __ffma2_rn(t0[2 * j4], make_float2(v.x, v.y), a0[c]);
                    a0[c] = __ffma2_rn(t0[2 * j4 + 1], make_float2(v.z, v.w), a0[c]);
                    a1[c] = __ffma2_rn(make_float2(e1.x, e1.y), make_float2(v.x, v.y), a1[c]);
                    a1[c] = __ffma2_rn(make_float2(e1.z, e1.w), make_float2(v.z, v.w), a1[c]);
                }
            }
            float w0[kK], w1[kK];
#pragma unroll
            for (int c = 0; c < kK; ++c) {
                w0[c] = a0[c].x + a0[c].y;
                w1[c] = a1[c].x + a1[c].y;
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
            // Ritz vectors U = V Y and B U = W Y
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
            // the Ritz residuals and the Gram matrix of B U, reduced together:
            // B U = U Theta + R with R orthogonal to U, so its columns are
            // nearly orthogonal whatever their scale, and one Cholesky QR of
            // the scaled Gram matrix orthonormalises them (a second pass runs
            // when they were not)
            float rmax = 0.0f, G[kK][kK];
#pragma unroll
            for (int c = 0; c < kK; ++c) {
                const float e0 = fmaf(-th[c], u0[c], bu0[c]);
                const float e1 = fmaf(-th[c], u1[c], bu1[c]);
                rmax = fmaxf(rmax, wsum(fmaf(e0, e0, e1 * e1)));
            }
            gram(bu0, bu1, G);
            const float lim = kTol * fabsf(th[0]);
            if (rmax <= lim * lim) {
                conv = true;
                break;
            }
            if (cholqr(bu0, bu1, G) > 1e-2f) {
                gram(bu0, bu1, G);
                cholqr(bu0, bu1, G);
            }
#pragma unroll
            for (int c = 0; c < kK; ++c) {
                v0[c] = bu0[c];
                v1[c] = bu1[c];
            }
            __syncwarp();
#pragma unroll
            for (int c = 0; c < kK; ++c) {
                sV[c * kN + i0] = v0[c];
                sV[c * kN + i1] = v1[c];
            }
        }
        // rows 32-63 of B are done with too: the next map's second half
        __syncwarp();
        if (mn < n) stage_half(sE, maps + mn * kMapFloats, 1, lane);
        if (!conv && lane == 0) atomicOr(flags, (uint32_t)TDM_FLAG_MDS_NOT_CONVERGED);

        float x0[kK], x1[kK];
#pragma unroll
        for (int c = 0; c < kK; ++c) {
            const float sq = sqrt_approx(fmaxf(th[c], 0.0f) * inv_scale);
            x0[c] = u0[c] * sq;
            x1[c] = u1[c] * sq;
        }
        float *X = coords + m * (kN * 3);
#pragma unroll
        for (int c = 0; c < kK; ++c) {
            X[i0 * 3 + c] = x0[c];
            X[i1 * 3 + c] = x1[c];
        }
        if (eig != nullptr && lane < 3) eig[m * 3 + lane] = (lane == 0 ? th[0] : lane == 1 ? th[1] : th[2]) * inv_scale;
        if (DIST) {
            // the distance map of the coordinates, as pdist_kernel computes it.
            // The coordinates go to shared memory as x[64], y[64], z[64] (in the
            // V arrays).  Lanes 0-15 write row 2p and lanes 16-31 row 2p+1,
            // four columns per lane, with 16-byte streaming stores.
            __syncwarp();
#pragma unroll
            for (int c = 0; c < kK; ++c) {
                sV[c * kN + i0] = x0[c];
                sV[c * kN + i1] = x1[c];
            }
            __syncwarp();
            const int q = lane & 15, h = lane >> 4;
            const float4 cx = ld4(sV + 4 * q), cy = ld4(sV + kN + 4 * q), cz = ld4(sV + 2 * kN + 4 * q);
            const float2 nx01 = make_float2(-cx.x, -cx.y), nx23 = make_float2(-cx.z, -cx.w);
            const float2 ny01 = make_float2(-cy.x, -cy.y), ny23 = make_float2(-cy.z, -cy.w);
            const float2 nz01 = make_float2(-cz.x, -cz.y), nz23 = make_float2(-cz.z, -cz.w);
            float4 *out = reinterpret_cast<float4 *>(dist + m * kMapFloats) + h * (kN / 4) + q;
#pragma unroll 4
            for (int rp = 0; rp < kN / 2; ++rp) {
                const int row = 2 * rp + h;
                const float bx = sV[row], by = sV[kN + row], bzs = sV[2 * kN + row];
                const float2 xx = make_float2(bx, bx), yy = make_float2(by, by), bz = make_float2(bzs, bzs);
                const float2 dx01 = __fadd2_rn(xx, nx01), dx23 = __fadd2_rn(xx, nx23);
                const float2 dy01 = __fadd2_rn(yy, ny01), dy23 = __fadd2_rn(yy, ny23);
                const float2 dz01 = __fadd2_rn(bz, nz01), dz23 = __fadd2_rn(bz, nz23);
                float2 s01 = __fmul2_rn(dx01, dx01), s23 = __fmul2_rn(dx23, dx23);
                s01 = __ffma2_rn(dy01, dy01, s01);
                s23 = __ffma2_rn(dy23, dy23, s23);
                s01 = __ffma2_rn(dz01, dz01, s01);
                s23 = __ffma2_rn(dz23, dz23, s23);
                __stcs(out + rp * (kN / 2),
                       make_float4(sqrt_approx(s01.x), sqrt_approx(s01.y), sqrt_approx(s23.x), sqrt_approx(s23.y)));
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
    const size_t smem = sizeof(float) * (size_t)kMdsWarps * kWarpFloats;
    static_assert((kWarpFloats * sizeof(float)) % 16 == 0 && (kN * kLd * sizeof(float)) % 16 == 0,
                  "float4 alignment of every warp's E and V tiles");
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
