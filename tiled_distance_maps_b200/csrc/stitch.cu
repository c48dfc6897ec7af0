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
// One CTA per (chain, sample) pair walks the chain in chunks of 32 tiles.  It
// stages the chunk's tiles (and the next one) in shared memory, once; its first
// warp aligns the chunk's seams, a lane per seam, and composes the maps by a
// shuffle scan, carried from chunk to chunk; then all its threads place the
// chunk's beads from the staged tiles.  Each tile is read from memory once,
// and chains of any length take this one pass.
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

// Eigen-decomposition of a symmetric positive semidefinite 3 x 3 matrix by
// cyclic Jacobi (Golub & Van Loan §8.5); descending eigenvalues, eigenvectors
// in the columns of V.  An off-diagonal entry counts as zero when
// a_pq^2 <= 1e-14 a_pp a_qq, relative to its own two diagonal entries: a
// test relative to the whole diagonal would leave the eigenvectors of the
// small eigenvalues of an elongated overlap (M^T M squares its condition)
// rotated by about 1e-6 l_1 / gap.  The matrix is scaled by its trace first,
// so no product overflows.  The rotation's reciprocals and square roots are
// the hardware approximations (a few ulp): the rotation stays orthogonal to
// float32 rounding.
template <int P, int Q>
__device__ __forceinline__ void jrot3(float (&A)[3][3], float (&V)[3][3]) {
    const float apq = A[P][Q];
    if (!(apq * apq > 1e-14f * (A[P][P] * A[Q][Q]))) return;
    const float theta = (A[Q][Q] - A[P][P]) * 0.5f * rcp_approx(apq);
    const float at = fabsf(theta);
    // t = sign(theta) / (|theta| + sqrt(theta^2 + 1)), 1 / (2 theta) where theta^2 would overflow
    const float r2 = fmaf(theta, theta, 1.0f);
    const float t = copysignf(at > 1e18f ? 0.5f * rcp_approx(at) : rcp_approx(at + r2 * rsqrt_approx(r2)), theta);
    const float c = rsqrt_approx(fmaf(t, t, 1.0f));
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
    const float tr = A[0][0] + A[1][1] + A[2][2];
    const float sc = tr > 1e-37f ? rcp_approx(tr) : 1.0f;
#pragma unroll
    for (int i = 0; i < 3; ++i)
#pragma unroll
        for (int j = 0; j < 3; ++j) A[i][j] *= sc;
    for (int sweep = 0; sweep < 16; ++sweep) {
        if (!(A[0][1] * A[0][1] > 1e-14f * (A[0][0] * A[1][1])) &&
            !(A[0][2] * A[0][2] > 1e-14f * (A[0][0] * A[2][2])) &&
            !(A[1][2] * A[1][2] > 1e-14f * (A[1][1] * A[2][2])))
            break;
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

// Polar factor R = U V^T of M = U S V^T through the eigenvectors V of M^T M:
// U = M V S^-1 re-orthonormalised, its third column completed by the cross
// product when M is rank deficient (an overlap of 3 beads, or coplanar ones).
// The fallback of newton_polar.
__device__ __noinline__ void polar_by_eig(const float (&M)[3][3], float (&R)[9]) {
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
    float n0 = U[0][0] * U[0][0] + U[1][0] * U[1][0] + U[2][0] * U[2][0];
    n0 = n0 > 1e-37f ? rsqrt_approx(n0) : 0.0f;
#pragma unroll
    for (int a = 0; a < 3; ++a) U[a][0] *= n0;
    float d01 = U[0][0] * U[0][1] + U[1][0] * U[1][1] + U[2][0] * U[2][1];
#pragma unroll
    for (int a = 0; a < 3; ++a) U[a][1] -= d01 * U[a][0];
    float n1 = U[0][1] * U[0][1] + U[1][1] * U[1][1] + U[2][1] * U[2][1];
    n1 = n1 > 1e-37f ? rsqrt_approx(n1) : 0.0f;
#pragma unroll
    for (int a = 0; a < 3; ++a) U[a][1] *= n1;
    if (lam[0] > 0.0f && lam[2] > 1e-10f * lam[0]) {
        const float d02 = U[0][0] * U[0][2] + U[1][0] * U[1][2] + U[2][0] * U[2][2];
        const float d12 = U[0][1] * U[0][2] + U[1][1] * U[1][2] + U[2][1] * U[2][2];
#pragma unroll
        for (int a = 0; a < 3; ++a) U[a][2] -= d02 * U[a][0] + d12 * U[a][1];
        float n2 = U[0][2] * U[0][2] + U[1][2] * U[1][2] + U[2][2] * U[2][2];
        n2 = n2 > 1e-37f ? rsqrt_approx(n2) : 0.0f;
#pragma unroll
        for (int a = 0; a < 3; ++a) U[a][2] *= n2;
    } else {
        U[0][2] = U[1][0] * U[2][1] - U[2][0] * U[1][1];
        U[1][2] = U[2][0] * U[0][1] - U[0][0] * U[2][1];
        U[2][2] = U[0][0] * U[1][1] - U[1][0] * U[0][1];
    }
#pragma unroll
    for (int a = 0; a < 3; ++a)
#pragma unroll
        for (int b = 0; b < 3; ++b) R[3 * a + b] = U[a][0] * V[b][0] + U[a][1] * V[b][1] + U[a][2] * V[b][2];
}

// Polar factor of M by the scaled Newton iteration X <- (g X + X^-T / g) / 2,
// g = (|X^-1|_F / |X|_F)^(1/2) (Higham, "Computing the polar decomposition --
// with applications", 1986), from X = M / |M|_F.  It works on M itself, so
// the condition of M is not squared as in M^T M, and it converges to the
// orthogonal factor whatever the sign of det M (an improper R is wanted:
// recovered coordinates are defined up to reflection).  X^-T is the cofactor
// matrix over the determinant.  Returns false, leaving R alone, when M is
// nearly singular (|det X| < 1e-6) or the iteration has not settled after 12
// steps; the caller then takes polar_by_eig.
__device__ __forceinline__ bool newton_polar(const float (&M)[3][3], float (&R)[9]) {
    float X[9], nx = 0.0f;
#pragma unroll
    for (int a = 0; a < 9; ++a) {
        X[a] = M[a / 3][a % 3];
        nx = fmaf(X[a], X[a], nx);
    }
    if (!(nx > 1e-37f)) return false;
    const float inx = rsqrt_approx(nx);
#pragma unroll
    for (int a = 0; a < 9; ++a) X[a] *= inx;
    nx = 1.0f;
    for (int it = 0; it < 12; ++it) {
        float Cf[9];
        Cf[0] = fmaf(X[4], X[8], -X[5] * X[7]);
        Cf[1] = fmaf(X[5], X[6], -X[3] * X[8]);
        Cf[2] = fmaf(X[3], X[7], -X[4] * X[6]);
        Cf[3] = fmaf(X[2], X[7], -X[1] * X[8]);
        Cf[4] = fmaf(X[0], X[8], -X[2] * X[6]);
        Cf[5] = fmaf(X[1], X[6], -X[0] * X[7]);
        Cf[6] = fmaf(X[1], X[5], -X[2] * X[4]);
        Cf[7] = fmaf(X[2], X[3], -X[0] * X[5]);
        Cf[8] = fmaf(X[0], X[4], -X[1] * X[3]);
        const float det = fmaf(X[0], Cf[0], fmaf(X[1], Cf[1], X[2] * Cf[2]));
        if (it == 0 && !(fabsf(det) > 1e-6f)) return false;
        const float rd = rcp_approx(det);
        float ny = 0.0f;
#pragma unroll
        for (int a = 0; a < 9; ++a) {
            Cf[a] *= rd;                       // X^-T
            ny = fmaf(Cf[a], Cf[a], ny);
        }
        // g = (ny / nx)^(1/4); X <- (g/2) X + (1/(2g)) X^-T
        const float g = rsqrt_approx(rsqrt_approx(ny * rcp_approx(nx)));
        const float ha = 0.5f * g, hb = 0.5f * rcp_approx(g);
        float dmax = 0.0f, nn = 0.0f;
#pragma unroll
        for (int a = 0; a < 9; ++a) {
            const float xn = fmaf(ha, X[a], hb * Cf[a]);
            dmax = fmaxf(dmax, fabsf(xn - X[a]));
            X[a] = xn;
            nn = fmaf(xn, xn, nn);
        }
        nx = nn;
        if (dmax <= 1e-6f) {
#pragma unroll
            for (int a = 0; a < 9; ++a) R[a] = X[a];
            return true;
        }
    }
    return false;
}

// Rigid map of tile k+1 onto tile k over the o overlap beads and its RMSD.
// The beads are visited from bead `rot` on (cyclically), so that lanes which
// read their own seams at a common stride spread over the banks.  The cross-
// covariance is formed in one pass from offsets to the first bead visited:
// M = sum (dp_i)(dq_i)^T - o m_p m_q^T, with m the mean offsets, which keeps
// its terms near the overlap's own extent however far the tiles sit from the
// origin.
__device__ Rigid align_seam(const float *P, const float *Q, int o, int rot, float *rmsd) {
    float pr[3], qr[3];
    const int i0 = rot % o;
#pragma unroll
    for (int d = 0; d < 3; ++d) {
        pr[d] = P[3 * i0 + d];
        qr[d] = Q[3 * i0 + d];
    }
    float sp[3] = {0.f, 0.f, 0.f}, sq[3] = {0.f, 0.f, 0.f};
    float M[3][3] = {{0.f, 0.f, 0.f}, {0.f, 0.f, 0.f}, {0.f, 0.f, 0.f}};
    int i = i0;
    for (int n = 0; n < o; ++n) {
        float dp[3], dq[3];
#pragma unroll
        for (int d = 0; d < 3; ++d) {
            dp[d] = P[3 * i + d] - pr[d];
            dq[d] = Q[3 * i + d] - qr[d];
            sp[d] += dp[d];
            sq[d] += dq[d];
        }
#pragma unroll
        for (int a = 0; a < 3; ++a)
#pragma unroll
            for (int b = 0; b < 3; ++b) M[a][b] = fmaf(dp[a], dq[b], M[a][b]);
        if (++i == o) i = 0;
    }
    const float inv_o = 1.0f / (float)o;
    float pc[3], qc[3];
#pragma unroll
    for (int d = 0; d < 3; ++d) {
        sp[d] *= inv_o;
        sq[d] *= inv_o;
        pc[d] = pr[d] + sp[d];
        qc[d] = qr[d] + sq[d];
    }
#pragma unroll
    for (int a = 0; a < 3; ++a)
#pragma unroll
        for (int b = 0; b < 3; ++b) M[a][b] = fmaf(-(float)o * sp[a], sq[b], M[a][b]);
    Rigid g;
    if (!newton_polar(M, g.r)) polar_by_eig(M, g.r);
#pragma unroll
    for (int a = 0; a < 3; ++a)
        g.t[a] = pc[a] - (g.r[3 * a] * qc[0] + g.r[3 * a + 1] * qc[1] + g.r[3 * a + 2] * qc[2]);
    float ss = 0.0f;
    i = i0;
    for (int n = 0; n < o; ++n) {
        float y[3];
        apply(g, Q + 3 * i, y);
#pragma unroll
        for (int d = 0; d < 3; ++d) {
            const float e = y[d] - P[3 * i + d];
            ss = fmaf(e, e, ss);
        }
        if (++i == o) i = 0;
    }
    *rmsd = sqrtf(ss * inv_o);
    return g;
}


// Seam maps of one chunk of 32 tiles, composed into tile 0's frame (warp-wide;
// lane l ends with G_{k0+l}); P / Q: lane l's seam k0+l beads (tile k0+l's
// last o, tile k0+l+1's first o), read only when that seam exists.  carry /
// carry_prev hold G_{k0} / G_{k0-1} on entry and G_{k0+32} / G_{k0+31} on
// return.  Residuals of the chunk's seams are written when resid is not NULL.
__device__ __forceinline__ Rigid chunk_maps(const float *P, const float *Q, int T, int o, int k0, int64_t pair,
                                            float *__restrict__ resid, Rigid &carry, Rigid &carry_prev) {
    const int lane = threadIdx.x & 31;
    const int k = k0 + lane;
    Rigid tk = identity();    // seam k: tile k+1 onto tile k
    if (k < T - 1) {
        float r;
        tk = align_seam(P, Q, o, lane, &r);
        if (resid != nullptr) resid[pair * (T - 1) + k] = r;
    }
    Rigid sk = tk;    // inclusive scan: t_{k0} o ... o t_k
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const Rigid prev = shfl_up(sk, d);
        if (lane >= d) sk = compose(prev, sk);
    }
    const Rigid gnext = compose(carry, sk);    // G_{k+1}
    Rigid gk = shfl_up(gnext, 1);               // G_k
    if (lane == 0) gk = carry;
    carry_prev = shfl_idx(gk, 31);
    carry = shfl_idx(gnext, 31);
    return gk;
}

__device__ __forceinline__ Rigid smem_map(const Rigid *g) {
    const float4 *v = reinterpret_cast<const float4 *>(g);
    const float4 a = v[0], b = v[1], c = v[2];
    Rigid o;
    o.r[0] = a.x, o.r[1] = a.y, o.r[2] = a.z, o.r[3] = a.w;
    o.r[4] = b.x, o.r[5] = b.y, o.r[6] = b.z, o.r[7] = b.w;
    o.r[8] = c.x, o.t[0] = c.y, o.t[1] = c.z, o.t[2] = c.w;
    return o;
}

__device__ __forceinline__ void smem_store_map(Rigid *g, const Rigid &m) {
    float4 *v = reinterpret_cast<float4 *>(g);
    v[0] = make_float4(m.r[0], m.r[1], m.r[2], m.r[3]);
    v[1] = make_float4(m.r[4], m.r[5], m.r[6], m.r[7]);
    v[2] = make_float4(m.r[8], m.t[0], m.t[1], m.t[2]);
}

constexpr int kStitchThreads = 128;
constexpr int kChunk = 32;                 // seams aligned per chunk, a lane each
constexpr int kSlots = kChunk + 1;         // tiles staged per chunk: its 32 and the next
constexpr int kTileLd = kN * 3 + 4;        // 196 floats: 16-byte rows; lane k's seam reads rotate by k beads
// shared memory: the maps of the chunk's tiles and of the tile before it, the
// staged tiles, and the last o beads of the tile before the chunk
constexpr int kMapsFloats = (kSlots + 1) * 12;
constexpr int kStitchSmemFloats = kMapsFloats + kSlots * kTileLd + 96;

// x / d for 0 <= x < 2^31 and 0 < d < 2^16 by the multiply-shift of m = ceil(2^32 / d)
__device__ __forceinline__ int div_by(int x, int d, uint32_t m) {
    int k = (int)(((uint64_t)(uint32_t)x * m) >> 32);
    if (k * d > x) --k;
    return k;
}

// G chain beads of tile k from bead j on (G = 4: 12 floats, 16-byte aligned in
// the staged tile, the previous tile's copy and the chain; G = 1 otherwise):
// the tile's aligned copy, averaged with tile k-1's over the overlap.
template <int G>
__device__ __forceinline__ void place_beads(const float *tile, const float *prev, const Rigid *gk, const Rigid *gp,
                                            bool ov, float *dst) {
    float x[3 * G], y[3 * G];
    if constexpr (G == 4) {
#pragma unroll
        for (int v = 0; v < 3; ++v) *reinterpret_cast<float4 *>(x + 4 * v) = reinterpret_cast<const float4 *>(tile)[v];
    } else {
#pragma unroll
        for (int v = 0; v < 3; ++v) x[v] = tile[v];
    }
    const Rigid g = smem_map(gk);
#pragma unroll
    for (int u = 0; u < G; ++u) apply(g, x + 3 * u, y + 3 * u);
    if (ov) {
        float xp[3 * G];
        if constexpr (G == 4) {
#pragma unroll
            for (int v = 0; v < 3; ++v)
                *reinterpret_cast<float4 *>(xp + 4 * v) = reinterpret_cast<const float4 *>(prev)[v];
        } else {
#pragma unroll
            for (int v = 0; v < 3; ++v) xp[v] = prev[v];
        }
        const Rigid h = smem_map(gp);
#pragma unroll
        for (int u = 0; u < G; ++u) {
            float y1[3];
            apply(h, xp + 3 * u, y1);
#pragma unroll
            for (int d = 0; d < 3; ++d) y[3 * u + d] = 0.5f * (y1[d] + y[3 * u + d]);
        }
    }
    if constexpr (G == 4) {
#pragma unroll
        for (int v = 0; v < 3; ++v) reinterpret_cast<float4 *>(dst)[v] = *reinterpret_cast<const float4 *>(y + 4 * v);
    } else {
#pragma unroll
        for (int v = 0; v < 3; ++v) dst[v] = y[v];
    }
}

// One CTA per (chain, sample) pair.  Tile k owns chain positions [k s, k s + s),
// the last tile [k s, k s + 64); the first o beads of tile k > 0 are the mean of
// tile k-1's and tile k's aligned copies.  The arithmetic does not depend on
// the chunking.  G = 4 beads per thread needs o % 4 == 0 (four beads then stay
// in one tile and on one side of the overlap boundary, 16-byte aligned).
template <int G>
__global__ void __launch_bounds__(kStitchThreads, 7) stitch_kernel(const float *__restrict__ coords, int T, int B,
                                                                   int o, float *__restrict__ chain,
                                                                   float *__restrict__ resid) {
    extern __shared__ __align__(16) float sm[];
    Rigid *smaps = reinterpret_cast<Rigid *>(sm);           // [0, 32): tiles k0 .. k0+31; [32]: tile k0-1
    float *stile = sm + kMapsFloats;                         // [33][196]: tiles k0 .. k0+32
    float *sprev = stile + kSlots * kTileLd;                 // tile k0-1's beads s .. 63
    const int64_t pair = blockIdx.x;
    const int c = (int)(pair / B), b = (int)(pair - (int64_t)(pair / B) * B);
    const int s = kN - o;
    const int L = kN + (T - 1) * s;
    const int tid = threadIdx.x;
    const int gpt = s / G;                                   // bead groups per tile stride
    const uint32_t mg = (uint32_t)((0x100000000ULL + (uint64_t)gpt - 1) / (uint64_t)gpt);
    float *dst = chain + pair * (int64_t)L * 3;
    Rigid carry = identity(), carry_prev = identity();       // warp 0: G_{k0}, G_{k0-1}
    for (int k0 = 0; k0 < T; k0 += kChunk) {
        const int nt = min(kSlots, T - k0);                  // tiles staged
        const int nc = min(kChunk, T - k0);                  // tiles placed
        // 16-byte copies: 48 per tile
        for (int idx = tid; idx < nt * 48; idx += kStitchThreads) {
            const int i = idx / 48, e = idx - i * 48;
            const float *src = coords + (((int64_t)c * T + k0 + i) * B + b) * (kN * 3) + 4 * e;
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(
                             __cvta_generic_to_shared(stile + i * kTileLd + 4 * e))),
                         "l"(src)
                         : "memory");
        }
        asm volatile("cp.async.commit_group;\n\tcp.async.wait_all;" ::: "memory");
        __syncthreads();
        if (tid < 32) {
            const int lane = tid;
            if (lane == 0) smem_store_map(smaps + kChunk, carry_prev);
            const Rigid gk = chunk_maps(stile + lane * kTileLd + 3 * s, stile + (lane + 1) * kTileLd, T, o, k0, pair,
                                        resid, carry, carry_prev);
            if (lane < nc) smem_store_map(smaps + lane, gk);
        }
        __syncthreads();
        // the chunk's bead groups: nc tiles of s beads, plus the last tile's o
        const int ng = nc * gpt + (k0 + nc == T ? o / G : 0);
        for (int g = tid; g < ng; g += kStitchThreads) {
            int kl = div_by(g, gpt, mg);
            if (kl > nc - 1) kl = nc - 1;
            const int j = (g - kl * gpt) * G;
            const int k = k0 + kl;
            const bool ov = k > 0 && j < o;
            place_beads<G>(stile + kl * kTileLd + 3 * j,
                           kl > 0 ? stile + (kl - 1) * kTileLd + 3 * (s + j) : sprev + 3 * j, smaps + kl,
                           smaps + (kl > 0 ? kl - 1 : kChunk), ov, dst + ((int64_t)k * s + j) * 3);
        }
        __syncthreads();
        // the chunk's last tile is the next chunk's tile before it
        if (k0 + kChunk < T)
            for (int e = tid; e < 3 * o; e += kStitchThreads) sprev[e] = stile[(kChunk - 1) * kTileLd + 3 * s + e];
        __syncthreads();
    }
}

}  // namespace
}  // namespace tdm

namespace tdm {

cudaError_t launch_stitch(const float *coords, const Tiling &t, float *chain, float *resid, cudaStream_t st) {
    const int64_t pairs = (int64_t)t.C * t.B;
    if (pairs <= 0) return cudaSuccess;
    if (pairs > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    const int o = t.T > 1 ? t.overlap : 0;
    const size_t smem = sizeof(float) * kStitchSmemFloats;
    static_assert(kMapsFloats % 4 == 0 && kTileLd % 4 == 0, "16-byte alignment of the staged maps and tiles");
    if (o % 4 == 0)
        stitch_kernel<4><<<(unsigned)pairs, kStitchThreads, smem, st>>>(coords, t.T, t.B, o, chain, resid);
    else
        stitch_kernel<1><<<(unsigned)pairs, kStitchThreads, smem, st>>>(coords, t.T, t.B, o, chain, resid);
    return cudaGetLastError();
}

}  // namespace tdm
