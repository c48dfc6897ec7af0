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

// 4-byte asynchronous global -> shared copy (a chunk's copies are all in
// flight before the CTA waits for them)
__device__ __forceinline__ void async_copy4(float *dst, const float *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
                 "l"(src)
                 : "memory");
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
constexpr int kTileLd = kN * 3 + 1;        // 193 floats: odd, so the lanes' reads of their seams do not conflict
// shared memory: the maps of the chunk's tiles and of the tile before it, the
// staged tiles, and the last o beads of the tile before the chunk
constexpr int kMapsFloats = (kSlots + 1) * 12;
constexpr int kStitchSmemFloats = kMapsFloats + kSlots * kTileLd + 96;

// One CTA per (chain, sample) pair.  Tile k owns chain positions [k s, k s + s),
// the last tile [k s, k s + 64); the first o beads of tile k > 0 are the mean of
// tile k-1's and tile k's aligned copies.  Bit for bit the arithmetic of the
// alignment (align_seam), the scan (chunk_maps) and the placement (apply, then
// the mean) does not depend on the chunking.
__global__ void __launch_bounds__(kStitchThreads, 7) stitch_kernel(const float *__restrict__ coords, int T, int B,
                                                                   int o, float *__restrict__ chain,
                                                                   float *__restrict__ resid) {
    extern __shared__ __align__(16) float sm[];
    Rigid *smaps = reinterpret_cast<Rigid *>(sm);           // [0, 32]: tiles k0 .. k0+31; [32]: tile k0-1
    float *stile = sm + kMapsFloats;                         // [33][193]: tiles k0 .. k0+32
    float *sprev = stile + kSlots * kTileLd;                 // tile k0-1's beads s .. 63
    const int64_t pair = blockIdx.x;
    const int c = (int)(pair / B), b = (int)(pair - (int64_t)(pair / B) * B);
    const int s = kN - o;
    const int L = kN + (T - 1) * s;
    const int tid = threadIdx.x;
    float *dst = chain + pair * (int64_t)L * 3;
    Rigid carry = identity(), carry_prev = identity();       // warp 0: G_{k0}, G_{k0-1}
    for (int k0 = 0; k0 < T; k0 += kChunk) {
        const int nt = min(kSlots, T - k0);                  // tiles staged
        const int nc = min(kChunk, T - k0);                  // tiles placed
        for (int i = 0; i < nt; ++i) {
            const float *src = coords + (((int64_t)c * T + k0 + i) * B + b) * (kN * 3);
            for (int e = tid; e < kN * 3; e += kStitchThreads) async_copy4(stile + i * kTileLd + e, src + e);
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
        // the chunk's beads: nc * s of them, plus the last tile's o beyond its stride
        const int nb = nc * s + (k0 + nc == T ? o : 0);
        for (int idx = tid; idx < nb; idx += kStitchThreads) {
            int kl = idx / s;
            if (kl > nc - 1) kl = nc - 1;
            const int j = idx - kl * s;
            const int k = k0 + kl;
            float x[3], y[3];
#pragma unroll
            for (int d = 0; d < 3; ++d) x[d] = stile[kl * kTileLd + 3 * j + d];
            apply(smem_map(smaps + kl), x, y);
            if (k > 0 && j < o) {
                float xp[3], y1[3];
                const float *bp = kl > 0 ? stile + (kl - 1) * kTileLd + 3 * (s + j) : sprev + 3 * j;
#pragma unroll
                for (int d = 0; d < 3; ++d) xp[d] = bp[d];
                apply(smem_map(smaps + (kl > 0 ? kl - 1 : kChunk)), xp, y1);
#pragma unroll
                for (int d = 0; d < 3; ++d) y[d] = 0.5f * (y1[d] + y[d]);
            }
            float *out = dst + ((int64_t)k * s + j) * 3;
#pragma unroll
            for (int d = 0; d < 3; ++d) out[d] = y[d];
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
    static_assert(kMapsFloats % 4 == 0, "16-byte alignment of the staged maps");
    stitch_kernel<<<(unsigned)pairs, kStitchThreads, smem, st>>>(coords, t.T, t.B, o, chain, resid);
    return cudaGetLastError();
}

}  // namespace tdm
