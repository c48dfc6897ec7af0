// Kabsch stitching of per-tile coordinates into chains.
//
// ParaChromo (mdpi.com/2079-9292/15/13/2750), §4.3.2 (last paragraph) and §5.5
// with Fig. 4: adjacent tiles are rigidly aligned on their shared 12 beads and
// stitched into one chromosome-scale chain; the per-seam residual after the
// alignment is reported.  Tile k+1 is mapped onto tile k by x -> R x + t with
// R the orthogonal polar factor of the overlap cross-covariance (improper
// rotations allowed: recovered coordinates are defined up to reflection); the
// maps compose along the chain into tile 0's frame; overlap beads take the
// mean of their two aligned copies.
//
// One warp per (chain, sample); lane k handles seam k and tile k of a chunk
// of 32 tiles, and a shuffle scan composes the maps.
#include "common.cuh"

namespace tdm {
namespace {

struct Rigid {
    float r[9];   // row-major rotation
    float t[3];
};

__device__ __forceinline__ Rigid compose(const Rigid &a, const Rigid &b) {   // a o b: x -> a(b(x))
    Rigid o;
#pragma unroll
    for (int i = 0; i < 3; ++i) {
#pragma unroll
        for (int j = 0; j < 3; ++j)
            o.r[3 * i + j] = fmaf(a.r[3 * i], b.r[j], fmaf(a.r[3 * i + 1], b.r[3 + j], a.r[3 * i + 2] * b.r[6 + j]));
        o.t[i] = fmaf(a.r[3 * i], b.t[0], fmaf(a.r[3 * i + 1], b.t[1], fmaf(a.r[3 * i + 2], b.t[2], a.t[i])));
    }
    return o;
}

__device__ __forceinline__ Rigid identity() {
    Rigid o;
#pragma unroll
    for (int i = 0; i < 9; ++i) o.r[i] = (i % 4 == 0) ? 1.0f : 0.0f;
    o.t[0] = o.t[1] = o.t[2] = 0.0f;
    return o;
}

__device__ __forceinline__ Rigid shfl_up(const Rigid &a, int d) {
    Rigid o;
#pragma unroll
    for (int i = 0; i < 9; ++i) o.r[i] = __shfl_up_sync(0xffffffffu, a.r[i], d);
#pragma unroll
    for (int i = 0; i < 3; ++i) o.t[i] = __shfl_up_sync(0xffffffffu, a.t[i], d);
    return o;
}

__device__ __forceinline__ Rigid shfl_idx(const Rigid &a, int src) {
    Rigid o;
#pragma unroll
    for (int i = 0; i < 9; ++i) o.r[i] = __shfl_sync(0xffffffffu, a.r[i], src);
#pragma unroll
    for (int i = 0; i < 3; ++i) o.t[i] = __shfl_sync(0xffffffffu, a.t[i], src);
    return o;
}

__device__ __forceinline__ void apply(const Rigid &g, const float *x, float *y) {
#pragma unroll
    for (int i = 0; i < 3; ++i)
        y[i] = fmaf(g.r[3 * i], x[0], fmaf(g.r[3 * i + 1], x[1], fmaf(g.r[3 * i + 2], x[2], g.t[i])));
}

// Eigen-decomposition of a symmetric 3 x 3 matrix by cyclic Jacobi (Golub &
// Van Loan §8.5); descending eigenvalues, eigenvectors in the columns of V.
template <int P, int Q>
__device__ __forceinline__ void jrot3(float (&A)[3][3], float (&V)[3][3]) {
    const float apq = A[P][Q];
    if (!(fabsf(apq) > 1e-12f * (fabsf(A[P][P]) + fabsf(A[Q][Q])))) return;
    const float theta = (A[Q][Q] - A[P][P]) / (2.0f * apq);
    const float t = copysignf(1.0f, theta) / (fabsf(theta) + sqrtf(fmaf(theta, theta, 1.0f)));
    const float c = 1.0f / sqrtf(fmaf(t, t, 1.0f));
    const float s = t * c;
    A[P][P] = fmaf(-t, apq, A[P][P]);
    A[Q][Q] = fmaf(t, apq, A[Q][Q]);
    A[P][Q] = A[Q][P] = 0.0f;
    constexpr int K = 3 - P - Q;
    const float kp = A[K][P], kq = A[K][Q];
    A[K][P] = A[P][K] = fmaf(c, kp, -s * kq);
    A[K][Q] = A[Q][K] = fmaf(s, kp, c * kq);
#pragma unroll
    for (int k = 0; k < 3; ++k) {
        const float vp = V[k][P], vq = V[k][Q];
        V[k][P] = fmaf(c, vp, -s * vq);
        V[k][Q] = fmaf(s, vp, c * vq);
    }
}

__device__ __forceinline__ void sym_eig3(float (&A)[3][3], float (&V)[3][3], float (&lam)[3]) {
#pragma unroll
    for (int i = 0; i < 3; ++i)
#pragma unroll
        for (int j = 0; j < 3; ++j) V[i][j] = i == j ? 1.0f : 0.0f;
    for (int sweep = 0; sweep < 16; ++sweep) {
        const float off = A[0][1] * A[0][1] + A[0][2] * A[0][2] + A[1][2] * A[1][2];
        const float dia = A[0][0] * A[0][0] + A[1][1] * A[1][1] + A[2][2] * A[2][2];
        if (off <= 1e-16f * dia) break;
        jrot3<0, 1>(A, V);
        jrot3<0, 2>(A, V);
        jrot3<1, 2>(A, V);
    }
    lam[0] = A[0][0];
    lam[1] = A[1][1];
    lam[2] = A[2][2];
    // sort descending with the columns of V
#pragma unroll
    for (int pass = 0; pass < 2; ++pass)
#pragma unroll
        for (int i = 0; i < 2 - pass; ++i)
            if (lam[i] < lam[i + 1]) {
                const float tl = lam[i];
                lam[i] = lam[i + 1];
                lam[i + 1] = tl;
#pragma unroll
                for (int k = 0; k < 3; ++k) {
                    const float tv = V[k][i];
                    V[k][i] = V[k][i + 1];
                    V[k][i + 1] = tv;
                }
            }
}

// Rigid map of tile k+1 onto tile k over the o overlap beads and its RMSD.
__device__ Rigid align_seam(const float *P, const float *Q, int o, float *rmsd) {
    float pc[3] = {0.f, 0.f, 0.f}, qc[3] = {0.f, 0.f, 0.f};
    for (int i = 0; i < o; ++i)
#pragma unroll
        for (int d = 0; d < 3; ++d) {
            pc[d] += P[3 * i + d];
            qc[d] += Q[3 * i + d];
        }
    const float inv_o = 1.0f / (float)o;
#pragma unroll
    for (int d = 0; d < 3; ++d) {
        pc[d] *= inv_o;
        qc[d] *= inv_o;
    }
    // M = sum_i (p_i - pc)(q_i - qc)^T
    float M[3][3] = {{0.f, 0.f, 0.f}, {0.f, 0.f, 0.f}, {0.f, 0.f, 0.f}};
    for (int i = 0; i < o; ++i) {
        float p[3], q[3];
#pragma unroll
        for (int d = 0; d < 3; ++d) {
            p[d] = P[3 * i + d] - pc[d];
            q[d] = Q[3 * i + d] - qc[d];
        }
#pragma unroll
        for (int a = 0; a < 3; ++a)
#pragma unroll
            for (int b = 0; b < 3; ++b) M[a][b] = fmaf(p[a], q[b], M[a][b]);
    }
    // polar factor R = U V^T of M = U S V^T: V from the eigenvectors of M^T M,
    // U = M V S^-1 re-orthonormalised (third column completed by the cross
    // product when M is rank deficient)
    float A[3][3], V[3][3], lam[3];
#pragma unroll
    for (int a = 0; a < 3; ++a)
#pragma unroll
        for (int b = 0; b < 3; ++b) A[a][b] = M[0][a] * M[0][b] + M[1][a] * M[1][b] + M[2][a] * M[2][b];
    sym_eig3(A, V, lam);
    float U[3][3];
#pragma unroll
    for (int c = 0; c < 3; ++c)
#pragma unroll
        for (int a = 0; a < 3; ++a) U[a][c] = M[a][0] * V[0][c] + M[a][1] * V[1][c] + M[a][2] * V[2][c];
    // Gram-Schmidt on U's columns (largest singular value first)
    float n0 = sqrtf(U[0][0] * U[0][0] + U[1][0] * U[1][0] + U[2][0] * U[2][0]);
    n0 = n0 > 0.0f ? 1.0f / n0 : 0.0f;
#pragma unroll
    for (int a = 0; a < 3; ++a) U[a][0] *= n0;
    float d01 = U[0][0] * U[0][1] + U[1][0] * U[1][1] + U[2][0] * U[2][1];
#pragma unroll
    for (int a = 0; a < 3; ++a) U[a][1] -= d01 * U[a][0];
    float n1 = sqrtf(U[0][1] * U[0][1] + U[1][1] * U[1][1] + U[2][1] * U[2][1]);
    n1 = n1 > 0.0f ? 1.0f / n1 : 0.0f;
#pragma unroll
    for (int a = 0; a < 3; ++a) U[a][1] *= n1;
    const float sigma_rel = lam[0] > 0.0f ? lam[2] / lam[0] : 0.0f;
    if (sigma_rel > 1e-10f) {
        const float d02 = U[0][0] * U[0][2] + U[1][0] * U[1][2] + U[2][0] * U[2][2];
        const float d12 = U[0][1] * U[0][2] + U[1][1] * U[1][2] + U[2][1] * U[2][2];
#pragma unroll
        for (int a = 0; a < 3; ++a) U[a][2] -= d02 * U[a][0] + d12 * U[a][1];
        float n2 = sqrtf(U[0][2] * U[0][2] + U[1][2] * U[1][2] + U[2][2] * U[2][2]);
        n2 = n2 > 0.0f ? 1.0f / n2 : 0.0f;
#pragma unroll
        for (int a = 0; a < 3; ++a) U[a][2] *= n2;
    } else {
        U[0][2] = U[1][0] * U[2][1] - U[2][0] * U[1][1];
        U[1][2] = U[2][0] * U[0][1] - U[0][0] * U[2][1];
        U[2][2] = U[0][0] * U[1][1] - U[1][0] * U[0][1];
    }
    Rigid g;
#pragma unroll
    for (int a = 0; a < 3; ++a)
#pragma unroll
        for (int b = 0; b < 3; ++b) g.r[3 * a + b] = U[a][0] * V[b][0] + U[a][1] * V[b][1] + U[a][2] * V[b][2];
#pragma unroll
    for (int a = 0; a < 3; ++a)
        g.t[a] = pc[a] - (g.r[3 * a] * qc[0] + g.r[3 * a + 1] * qc[1] + g.r[3 * a + 2] * qc[2]);
    float ss = 0.0f;
    for (int i = 0; i < o; ++i) {
        float y[3];
        apply(g, Q + 3 * i, y);
#pragma unroll
        for (int d = 0; d < 3; ++d) {
            const float e = y[d] - P[3 * i + d];
            ss = fmaf(e, e, ss);
        }
    }
    *rmsd = sqrtf(ss * inv_o);
    return g;
}

__global__ void __launch_bounds__(128) stitch_kernel(const float *__restrict__ coords, int C, int T, int B, int o,
                                                     float *__restrict__ chain, float *__restrict__ resid) {
    const int lane = threadIdx.x & 31;
    const int64_t nw = (int64_t)C * B;
    const int s = kN - o;
    const int64_t L = kN + (int64_t)(T - 1) * s;
    for (int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; w < nw;
         w += ((int64_t)gridDim.x * blockDim.x) >> 5) {
        const int c = (int)(w / B), b = (int)(w - (int64_t)c * B);
        float *out = chain + w * L * 3;
        Rigid carry = identity();        // G_k0: tile k0 into tile 0's frame
        Rigid carry_prev = identity();   // G_{k0-1}
        for (int k0 = 0; k0 < T; k0 += 32) {
            const int k = k0 + lane;
            // seam k: tile k+1 onto tile k
            Rigid tk = identity();
            if (k < T - 1) {
                const float *Pk = coords + (((int64_t)c * T + k) * B + b) * (kN * 3) + s * 3;
                const float *Qk = coords + (((int64_t)c * T + k + 1) * B + b) * (kN * 3);
                float r;
                tk = align_seam(Pk, Qk, o, &r);
                if (resid != nullptr) resid[w * (T - 1) + k] = r;
            }
            // inclusive scan within the chunk: S_k = t_k0 o ... o t_k
            Rigid sk = tk;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const Rigid prev = shfl_up(sk, d);
                if (lane >= d) sk = compose(prev, sk);
            }
            const Rigid gnext = compose(carry, sk);          // G_{k+1}
            Rigid gk = shfl_up(gnext, 1);                     // G_k
            if (lane == 0) gk = carry;
            Rigid gkm1 = shfl_up(gk, 1);                      // G_{k-1}
            if (lane == 0) gkm1 = carry_prev;
            if (k < T) {
                const float *Xk = coords + (((int64_t)c * T + k) * B + b) * (kN * 3);
                float *dst = out + (int64_t)k * s * 3;
                // own beads: not the left overlap (written below, averaged) and
                // not the right overlap (the next tile's lane averages it)
                const int j0 = k == 0 ? 0 : o;
                const int j1 = k == T - 1 ? kN : s;
                for (int j = j0; j < j1; ++j) apply(gk, Xk + 3 * j, dst + 3 * j);
                if (k > 0) {
                    const float *Xp = coords + (((int64_t)c * T + k - 1) * B + b) * (kN * 3) + s * 3;
                    for (int j = 0; j < o; ++j) {
                        float y1[3], y2[3];
                        apply(gkm1, Xp + 3 * j, y1);
                        apply(gk, Xk + 3 * j, y2);
#pragma unroll
                        for (int d = 0; d < 3; ++d) dst[3 * j + d] = 0.5f * (y1[d] + y2[d]);
                    }
                }
            }
            carry_prev = shfl_idx(gk, 31);
            carry = shfl_idx(gnext, 31);
        }
    }
}

}  // namespace
}  // namespace tdm

namespace tdm {

cudaError_t launch_stitch(const float *coords, const Tiling &t, float *chain, float *resid, cudaStream_t st) {
    const int64_t warps = (int64_t)t.C * t.B;
    if (warps <= 0) return cudaSuccess;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int64_t grid = (warps + 3) / 4;
    if (grid > (int64_t)sms * 16) grid = (int64_t)sms * 16;
    stitch_kernel<<<(int)grid, 128, 0, st>>>(coords, t.C, t.T, t.B, t.T > 1 ? t.overlap : 0, chain, resid);
    return cudaGetLastError();
}

}  // namespace tdm
