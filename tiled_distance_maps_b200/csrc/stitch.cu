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
// Chains of up to kFusedMaxT tiles take one pass: a CTA per (chain, sample)
// pair, whose first warp aligns the seams and composes the maps by a shuffle
// scan, 32 tiles at a time, into shared memory, after which all its threads
// place the pair's beads.  Longer chains take two passes over chunks of pairs
// whose maps fit the context scratch: the same alignment into global memory,
// then one thread per group of chain beads.
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

// Eigen-decomposition of a symmetric 3 x 3 matrix by cyclic Jacobi (Golub &
// Van Loan §8.5); descending eigenvalues, eigenvectors in the columns of V.
// The rotation's reciprocals and square roots are the hardware approximations
// (a few ulp): the rotation stays orthogonal to float32 rounding, and the skip
// test below keeps theta^2 finite (|theta| < 5e11).
template <int P, int Q>
__device__ __forceinline__ void jrot3(float (&A)[3][3], float (&V)[3][3]) {
    const float apq = A[P][Q];
    if (!(fabsf(apq) > 1e-12f * (fabsf(A[P][P]) + fabsf(A[Q][Q])))) return;
    const float theta = (A[Q][Q] - A[P][P]) * 0.5f * rcp_approx(apq);
    const float r2 = fmaf(theta, theta, 1.0f);
    const float t = copysignf(rcp_approx(fabsf(theta) + r2 * rsqrt_approx(r2)), theta);
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
    for (int sweep = 0; sweep < 16; ++sweep) {
        const float off = A[0][1] * A[0][1] + A[0][2] * A[0][2] + A[1][2] * A[1][2];
        const float dia = A[0][0] * A[0][0] + A[1][1] * A[1][1] + A[2][2] * A[2][2];
        if (off <= 1e-12f * dia) break;    // off-diagonal within 1e-6 of the diagonal (float32 reaches no further)
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
        tk = align_seam(P, Q, o, &r);
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

// 4-byte asynchronous global -> shared copy (the copies of a chunk are all in
// flight before the warp waits for them)
__device__ __forceinline__ void async_copy4(float *dst, const float *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
                 "l"(src)
                 : "memory");
}

// The maps of every tile of pair (c, b) into out[0 .. T) and its residuals
// into resid (warp-wide): the seam beads of 32 tiles at a time are staged in
// shared memory (sbeads: [2][32][3o+1], P then Q per lane) by coalesced
// warp-wide asynchronous copies (per-lane stride 3o+1 floats, odd, so the
// lanes' reads do not conflict); out may be global or shared memory.
__device__ __forceinline__ void pair_maps(const float *__restrict__ coords, int T, int B, int o, int c, int b,
                                          int64_t pair, float *sbeads, float *__restrict__ resid, Rigid *out) {
    const int lane = threadIdx.x & 31;
    const int s = kN - o;
    const int n3 = 3 * o, ld = 3 * o + 1;
    float *sP = sbeads, *sQ = sbeads + 32 * ld;
    Rigid carry = identity(), carry_prev = identity();
    for (int k0 = 0; k0 < T; k0 += 32) {
        const int nseam = min(32, T - 1 - k0);    // seams k0 .. k0+nseam-1
        __syncwarp();
        for (int r = 0; r < nseam; ++r) {
            const float *Pg = coords + (((int64_t)c * T + k0 + r) * B + b) * (kN * 3) + s * 3;
            const float *Qg = coords + (((int64_t)c * T + k0 + r + 1) * B + b) * (kN * 3);
            for (int i = lane; i < n3; i += 32) {
                async_copy4(sP + r * ld + i, Pg + i);
                async_copy4(sQ + r * ld + i, Qg + i);
            }
        }
        asm volatile("cp.async.commit_group;\n\tcp.async.wait_all;" ::: "memory");
        __syncwarp();
        const Rigid gk = chunk_maps(sP + lane * ld, sQ + lane * ld, T, o, k0, pair, resid, carry, carry_prev);
        if (k0 + lane < T) out[k0 + lane] = gk;
    }
}

// Pass 1 of the two-pass form: one warp (one CTA) per (chain, sample) of
// pairs [pair0, pair0 + n): every tile's map into gmaps[(pair - pair0) * T + k]
// and the residuals into resid.
__global__ void __launch_bounds__(32) stitch_align_kernel(const float *__restrict__ coords, int T, int B, int o,
                                                          int64_t pair0, Rigid *__restrict__ gmaps,
                                                          float *__restrict__ resid) {
    extern __shared__ float sbeads[];    // [2][32][3o+1]
    const int64_t q = blockIdx.x;
    const int64_t pair = pair0 + q;
    const int c = (int)(pair / B), b = (int)(pair - (int64_t)(pair / B) * B);
    pair_maps(coords, T, B, o, c, b, pair, sbeads, resid, gmaps + q * T);
}

__device__ __forceinline__ Rigid load_map(const Rigid *g) {
    const float4 *v = reinterpret_cast<const float4 *>(g);
    const float4 a = __ldg(v), b = __ldg(v + 1), c = __ldg(v + 2);
    Rigid o;
    o.r[0] = a.x, o.r[1] = a.y, o.r[2] = a.z, o.r[3] = a.w;
    o.r[4] = b.x, o.r[5] = b.y, o.r[6] = b.z, o.r[7] = b.w;
    o.r[8] = c.x, o.t[0] = c.y, o.t[1] = c.z, o.t[2] = c.w;
    return o;
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

// Chain beads [p, p + G) of pair (c, b) from its tiles' coordinates and maps
// (maps: the pair's T maps, global when GLOBAL_MAPS, else shared).  Tile k owns
// chain positions [k s, k s + s), the last tile [k s, k s + 64); the first o
// beads of tile k > 0 are the mean of tile k-1's and tile k's aligned copies.
// G = 4 needs o % 4 == 0: four beads then stay in one tile and on one side of
// the overlap boundary, and their 12 coordinates are 16-byte aligned in the
// tile and in the chain.
template <int G, bool GLOBAL_MAPS>
__device__ __forceinline__ void place_group(const float *__restrict__ coords, int T, int B, int o, int c, int b,
                                            int p, const Rigid *maps, float *dst) {
    const int s = kN - o;
    int k = p / s;
    if (k > T - 1) k = T - 1;
    const int j = p - k * s;
    // both rounds of loads (the tile's beads and map; for overlap beads also
    // the previous tile's) are issued before any arithmetic
    const bool ov = k > 0 && j < o;
    float x[3 * G], xp[3 * G], y[3 * G];
    const float *xk = coords + (((int64_t)c * T + k) * B + b) * (kN * 3) + 3 * j;
    const float *xq = coords + (((int64_t)c * T + (ov ? k - 1 : k)) * B + b) * (kN * 3) + 3 * (s + j);
    const Rigid gk = GLOBAL_MAPS ? load_map(maps + k) : smem_map(maps + k);
    Rigid gp = gk;
    if constexpr (G == 4) {
#pragma unroll
        for (int v = 0; v < 3; ++v) *reinterpret_cast<float4 *>(x + 4 * v) = __ldg(reinterpret_cast<const float4 *>(xk) + v);
        if (ov) {
#pragma unroll
            for (int v = 0; v < 3; ++v)
                *reinterpret_cast<float4 *>(xp + 4 * v) = __ldg(reinterpret_cast<const float4 *>(xq) + v);
            gp = GLOBAL_MAPS ? load_map(maps + k - 1) : smem_map(maps + k - 1);
        }
    } else {
#pragma unroll
        for (int v = 0; v < 3 * G; ++v) x[v] = __ldg(xk + v);
        if (ov) {
#pragma unroll
            for (int v = 0; v < 3 * G; ++v) xp[v] = __ldg(xq + v);
            gp = GLOBAL_MAPS ? load_map(maps + k - 1) : smem_map(maps + k - 1);
        }
    }
#pragma unroll
    for (int u = 0; u < G; ++u) apply(gk, x + 3 * u, y + 3 * u);
    if (ov) {
#pragma unroll
        for (int u = 0; u < G; ++u) {
            float y1[3];
            apply(gp, xp + 3 * u, y1);
#pragma unroll
            for (int d = 0; d < 3; ++d) y[3 * u + d] = 0.5f * (y1[d] + y[3 * u + d]);
        }
    }
    if constexpr (G == 4) {
#pragma unroll
        for (int v = 0; v < 3; ++v) reinterpret_cast<float4 *>(dst)[v] = *reinterpret_cast<const float4 *>(y + 4 * v);
    } else {
#pragma unroll
        for (int v = 0; v < 3 * G; ++v) dst[v] = y[v];
    }
}

// Pass 2 of the two-pass form: one thread per G beads of the chains of pairs
// [pair0, pair0 + n).  32-bit indices: a chunk holds n L <= (scratch / 12T) *
// 64T beads, and pairs < 2^31 is checked by the caller.
template <int G>
__global__ void __launch_bounds__(256) stitch_place_kernel(const float *__restrict__ coords, int T, int B, int o,
                                                           int pair0, int n, const Rigid *__restrict__ gmaps,
                                                           float *__restrict__ chain) {
    const int s = kN - o;
    const int L = kN + (T - 1) * s;
    const int LG = L / G;
    const int total = n * LG;
    for (int idx = blockIdx.x * blockDim.x + threadIdx.x; idx < total; idx += gridDim.x * blockDim.x) {
        const int q = idx / LG;
        const int p = (idx - q * LG) * G;
        const int pair = pair0 + q;
        const int c = pair / B, b = pair - (pair / B) * B;
        place_group<G, true>(coords, T, B, o, c, b, p, gmaps + (int64_t)q * T, chain + ((int64_t)pair * L + p) * 3);
    }
}

// The one-pass form for chains of at most kFusedMaxT tiles: one CTA of 128
// threads per (chain, sample) pair, 7 CTAs per SM (72 registers, no spills),
// so that 1036 pairs are resident at once.  Warp 0 computes the pair's maps into
// shared memory (pair_maps), then all threads place its beads.
constexpr int kFusedMaxT = 512;
constexpr int kFusedThreads = 128;

template <int G>
__global__ void __launch_bounds__(kFusedThreads, 7) stitch_kernel(const float *__restrict__ coords, int T, int B, int o,
                                                     float *__restrict__ chain, float *__restrict__ resid) {
    extern __shared__ __align__(16) float sm[];    // [2][32][3o+1] bead staging, then [T] maps
    Rigid *smaps = reinterpret_cast<Rigid *>(sm + 2 * 32 * (3 * o + 1));
    const int64_t pair = blockIdx.x;
    const int c = (int)(pair / B), b = (int)(pair - (int64_t)(pair / B) * B);
    if (threadIdx.x < 32) pair_maps(coords, T, B, o, c, b, pair, sm, resid, smaps);
    __syncthreads();
    const int L = kN + (T - 1) * (kN - o);
    float *dst = chain + pair * (int64_t)L * 3;
    for (int g = threadIdx.x; g < L / G; g += blockDim.x)
        place_group<G, false>(coords, T, B, o, c, b, g * G, smaps, dst + (int64_t)g * G * 3);
}

}  // namespace
}  // namespace tdm

namespace tdm {

cudaError_t launch_stitch(const float *coords, const Tiling &t, float *chain, float *resid, float *scratch,
                          size_t scratch_floats, cudaStream_t st) {
    const int64_t pairs = (int64_t)t.C * t.B;
    if (pairs <= 0) return cudaSuccess;
    if (pairs > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    const int o = t.T > 1 ? t.overlap : 0;
    const int64_t per_pair = (int64_t)t.T * (int64_t)(sizeof(Rigid) / sizeof(float));
    // T <= 65535 (checked with the tiling) keeps one pair's maps within the scratch
    const int64_t chunk = scratch == nullptr ? 0 : (int64_t)scratch_floats / per_pair;
    if (chunk < 1) return cudaErrorInvalidValue;
    const bool vec = o % 4 == 0;
    if (t.T <= kFusedMaxT) {
        // 2 * 32 * (3o + 1) floats: a multiple of 16 bytes, so the maps that follow are aligned
        const size_t smem = sizeof(float) * 2 * 32 * (3 * o + 1) + sizeof(Rigid) * (size_t)t.T;
        if (vec)
            stitch_kernel<4><<<(unsigned)pairs, kFusedThreads, smem, st>>>(coords, t.T, t.B, o, chain, resid);
        else
            stitch_kernel<1><<<(unsigned)pairs, kFusedThreads, smem, st>>>(coords, t.T, t.B, o, chain, resid);
        return cudaGetLastError();
    }
    Rigid *gmaps = reinterpret_cast<Rigid *>(scratch);
    for (int64_t p0 = 0; p0 < pairs; p0 += chunk) {
        const int64_t n = pairs - p0 < chunk ? pairs - p0 : chunk;
        const size_t smem = sizeof(float) * 2 * 32 * (3 * o + 1);
        stitch_align_kernel<<<(unsigned)n, 32, smem, st>>>(coords, t.T, t.B, o, p0, gmaps, resid);
        const int64_t beads = n * (kN + (int64_t)(t.T - 1) * (kN - o));
        int64_t blocks = ((vec ? beads / 4 : beads) + 255) / 256;
        if (blocks > 148LL * 64) blocks = 148LL * 64;
        if (vec)
            stitch_place_kernel<4><<<(unsigned)blocks, 256, 0, st>>>(coords, t.T, t.B, o, (int)p0, (int)n, gmaps, chain);
        else
            stitch_place_kernel<1><<<(unsigned)blocks, 256, 0, st>>>(coords, t.T, t.B, o, (int)p0, (int)n, gmaps, chain);
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace tdm
