// Coordinate refinement by SMACOF (stress majorisation), one warp per map.
//
// ParaChromo (mdpi.com/2079-9292/15/13/2750), §3.1: the point cloud comes from
// distance-geometry initialisation followed by coordinate refinement.  The
// refinement minimises the raw stress sum_{i<j} (|x_i - x_j| - D_ij)^2 by the
// Guttman transform (de Leeuw 1977): x_i <- (1/n) sum_{j != i} (D_ij / d_ij)
// (x_i - x_j), with d_ij the current distances and terms with d_ij = 0 left
// out; D is symmetrised first.  A fixed number of iterations is run.
//
// The pair term w_ij (x_i - x_j), w_ij = D_ij / d_ij, is antisymmetric, so each
// unordered pair is evaluated once and credited to both beads.  The 64 beads
// form 16 groups of four (group g = beads 4g..4g+3); lane l of each half-warp
// owns group l.  Group pairs {g, g+k mod 16} are taken round a ring: the lower
// half-warp takes offsets k = 1..4, the upper k = 5..8.  At offset k lane l
// reads group l+k's coordinates (three 128-bit loads from a structure-of-arrays
// copy), evaluates the 16 bead pairs, adds its own beads' shares to registers
// and the partner's shares to a travelling accumulator, which moves one lane
// down the ring before the next offset, so that after the last offset it holds
// the shares of one group and reaches the owner in one shuffle.  Offset 8 meets
// each group pair from both ends, so its weights are halved.  Of the six pairs
// inside a group each half-warp takes three: the upper half holds its beads in
// a rotated register order, so the same register pairs name other bead pairs.
// The halves' sums are added by one exchange.  Per map-iteration that is 2,144
// pair terms (2,016 distinct) against 4,096 when every ordered pair is
// evaluated.
//
// The arithmetic is packed float32: one instruction serves the lane's bead
// against two partner beads (e = x_partner - x_own, formed as an FMA with -1,
// so the own sums are kept negated and the partners' shares need no sign
// change).  D stays in shared memory only to be read into registers: each lane
// keeps the 67 symmetrised weights of its pairs, and the copy for the next map
// is issued while the current one iterates.  The squared distance of a pair is
// seeded with FLT_MIN, so a pair at distance zero (coincident beads)
// contributes w * 0 = 0 without a branch; pairs closer than about 1e-19 are
// weighted as if that far apart.
#include "common.cuh"

namespace tdm {
namespace {

constexpr int kRefWarps = 4;
constexpr int kLdR = kN + 4;
constexpr int kRefWarpFloats = kN * kLdR + 3 * kN;
constexpr int kRing = 4;    // ring offsets per half-warp
constexpr float kQSeed = 1.17549435e-38f;    // FLT_MIN

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

struct Group {    // coordinates of the four beads of one group
    float x[4], y[4], z[4];
};

struct Pairs {    // coordinates of a group as float2 pairs: beads (0, 1) and (2, 3)
    float2 x[2], y[2], z[2];
};

__device__ __forceinline__ void shuffle_pairs(Pairs &t, int src) {
#pragma unroll
    for (int c = 0; c < 2; ++c) {
        t.x[c].x = __shfl_sync(0xffffffffu, t.x[c].x, src);
        t.x[c].y = __shfl_sync(0xffffffffu, t.x[c].y, src);
        t.y[c].x = __shfl_sync(0xffffffffu, t.y[c].x, src);
        t.y[c].y = __shfl_sync(0xffffffffu, t.y[c].y, src);
        t.z[c].x = __shfl_sync(0xffffffffu, t.z[c].x, src);
        t.z[c].y = __shfl_sync(0xffffffffu, t.z[c].y, src);
    }
}

__device__ __forceinline__ Pairs load_pairs(const float *sx, int g) {
    const float4 px = ld4(sx + 4 * g), py = ld4(sx + kN + 4 * g), pz = ld4(sx + 2 * kN + 4 * g);
    return Pairs{{make_float2(px.x, px.y), make_float2(px.z, px.w)},
                 {make_float2(py.x, py.y), make_float2(py.z, py.w)},
                 {make_float2(pz.x, pz.y), make_float2(pz.z, pz.w)}};
}

// own bead (bx, by, bz), broadcast, against partner beads (2cp, 2cp+1) in
// packed float32: with e = x_partner - x_own, w e is added to the own bead's
// negated sum and to the partners' shares
__device__ __forceinline__ void pair_term2(const float2 &bx, const float2 &by, const float2 &bz, const Pairs &p,
                                           int cp, float2 dij, float2 &ax, float2 &ay, float2 &az, Pairs &t) {
    const float2 m1 = make_float2(-1.0f, -1.0f);
    const float2 e0 = __ffma2_rn(bx, m1, p.x[cp]), e1 = __ffma2_rn(by, m1, p.y[cp]),
                 e2 = __ffma2_rn(bz, m1, p.z[cp]);
    float2 q = __ffma2_rn(e0, e0, make_float2(kQSeed, kQSeed));
    q = __ffma2_rn(e1, e1, q);
    q = __ffma2_rn(e2, e2, q);
    const float2 w = __fmul2_rn(dij, make_float2(rsqrt_approx(q.x), rsqrt_approx(q.y)));
    ax = __ffma2_rn(w, e0, ax);
    ay = __ffma2_rn(w, e1, ay);
    az = __ffma2_rn(w, e2, az);
    t.x[cp] = __ffma2_rn(w, e0, t.x[cp]);
    t.y[cp] = __ffma2_rn(w, e1, t.y[cp]);
    t.z[cp] = __ffma2_rn(w, e2, t.z[cp]);
}

// Register order of the own beads: the lower half-warp keeps beads 0..3 in
// registers 0..3, the upper half-warp bead (a + 3) mod 4 in register a.  Then
// the same three register pairs (0, 1), (2, 3), (0, 2) are the bead pairs
// (0,1), (2,3), (0,2) in one half and (3,0), (1,2), (3,1) in the other: the
// six pairs inside a group, each once.
__device__ __forceinline__ int bead_of(int h, int a) { return h ? (a + 3) & 3 : a; }
// hi where sel = 0x7654, lo where sel = 0x3210: a byte permute, so that the
// choice between two registers is never turned into an indexed access
__device__ __forceinline__ float pick(unsigned sel, float hi, float lo) {
    return __int_as_float((int)__byte_perm((unsigned)__float_as_int(lo), (unsigned)__float_as_int(hi), sel));
}
__device__ __forceinline__ float rot(unsigned sel, const float (&v)[4], int a) { return pick(sel, v[(a + 3) & 3], v[a]); }
__device__ __forceinline__ float unrot(unsigned sel, const float (&v)[4], int a) { return pick(sel, v[(a + 1) & 3], v[a]); }
__host__ __device__ constexpr int inner_u(int j) { return j == 1 ? 2 : 0; }
__host__ __device__ constexpr int inner_v(int j) { return j == 0 ? 1 : j == 1 ? 3 : 2; }

__device__ __forceinline__ float stress_term(const Group &b, int a, const Group &p, int c, float dij) {
    const float e0 = b.x[a] - p.x[c], e1 = b.y[a] - p.y[c], e2 = b.z[a] - p.z[c];
    const float r = sqrt_approx(fmaf(e2, e2, fmaf(e1, e1, e0 * e0))) - dij;
    return r * r;
}

__global__ void __launch_bounds__(kRefWarps * 32, 2) refine_kernel(const float *__restrict__ maps, int64_t n,
                                                                   float *__restrict__ coords, int iterations,
                                                                   float *__restrict__ stress_out) {
    extern __shared__ __align__(16) float smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = lane >> 4, l = lane & 15;
    float *sD = smem + warp * kRefWarpFloats;
    float *sx = sD + kN * kLdR;    // x[64], y[64], z[64]
    const int64_t stride = (int64_t)gridDim.x * kRefWarps;
    constexpr float kInvN = 1.0f / kN;
    const int k0 = 1 + kRing * h;                       // first ring offset of this half
    const int next = (h << 4) | ((l + 1) & 15);          // ring neighbour the accumulator comes from
    const int owner_src = (h << 4) | ((l - kRing + 1 - k0 + 32) & 15);    // lane holding this group's shares

    const bool up = h == 1;
    const unsigned sel = up ? 0x7654u : 0x3210u;    // byte-permute selector of the upper half

    int64_t m = (int64_t)blockIdx.x * kRefWarps + warp;
    if (m < n) stage_map_async(sD, maps + m * kMapFloats, lane);
    for (; m < n; m += stride) {
        wait_staged();
        __syncwarp();
        // symmetrised weights of this lane's pairs, own beads in register
        // order; offset 8 (upper half, last offset) meets each group pair from
        // both ends, so its weights are halved
        float2 d[kRing][4][2];
        float dw[3];
#pragma unroll
        for (int s = 0; s < kRing; ++s) {
            const int g = (l + k0 + s) & 15;
            const float sc = (up && s == kRing - 1) ? 0.25f : 0.5f;
            float4 r[4], t[4];
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                r[a] = ld4(sD + (4 * l + bead_of(h, a)) * kLdR + 4 * g);
                t[a] = ld4(sD + (4 * g + a) * kLdR + 4 * l);
            }
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float v[4] = {t[c].x, t[c].y, t[c].z, t[c].w};
                t[c] = make_float4(rot(sel, v, 0), rot(sel, v, 1), rot(sel, v, 2), rot(sel, v, 3));
            }
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int cp = 0; cp < 2; ++cp)
                    d[s][a][cp] = make_float2(sc * (comp(r[a], 2 * cp) + comp(t[2 * cp], a)),
                                              sc * (comp(r[a], 2 * cp + 1) + comp(t[2 * cp + 1], a)));
        }
        {
            float4 r[4];
#pragma unroll
            for (int a = 0; a < 4; ++a) r[a] = ld4(sD + (4 * l + a) * kLdR + 4 * l);
            // register pairs (0,1), (2,3), (0,2): bead pairs (0,1), (2,3), (0,2)
            // in the lower half, (3,0), (1,2), (3,1) in the upper
            auto ds = [&](int a, int c) { return 0.5f * (comp(r[a], c) + comp(r[c], a)); };
            dw[0] = pick(sel, ds(3, 0), ds(0, 1));
            dw[1] = pick(sel, ds(1, 2), ds(2, 3));
            dw[2] = pick(sel, ds(3, 1), ds(0, 2));
        }
        __syncwarp();
        if (m + stride < n) stage_map_async(sD, maps + (m + stride) * kMapFloats, lane);

        float *X = coords + m * (kN * 3) + 12 * l;
        Group b;    // bead order
#pragma unroll
        for (int a = 0; a < 4; ++a) {
            b.x[a] = X[3 * a];
            b.y[a] = X[3 * a + 1];
            b.z[a] = X[3 * a + 2];
        }
        for (int it = 0; it < iterations; ++it) {
            __syncwarp();
            if (h == 0) {
                st4(sx + 4 * l, make_float4(b.x[0], b.x[1], b.x[2], b.x[3]));
                st4(sx + kN + 4 * l, make_float4(b.y[0], b.y[1], b.y[2], b.y[3]));
                st4(sx + 2 * kN + 4 * l, make_float4(b.z[0], b.z[1], b.z[2], b.z[3]));
            }
            __syncwarp();
            Group r;    // register order
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                r.x[a] = rot(sel, b.x, a);
                r.y[a] = rot(sel, b.y, a);
                r.z[a] = rot(sel, b.z, a);
            }
            float2 ax[4], ay[4], az[4];
            Pairs t;
#pragma unroll
            for (int a = 0; a < 4; ++a) ax[a] = ay[a] = az[a] = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int c = 0; c < 2; ++c) t.x[c] = t.y[c] = t.z[c] = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int s = 0; s < kRing; ++s) {
                const Pairs p = load_pairs(sx, (l + k0 + s) & 15);
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int cp = 0; cp < 2; ++cp)
                        pair_term2(make_float2(r.x[a], r.x[a]), make_float2(r.y[a], r.y[a]),
                                   make_float2(r.z[a], r.z[a]), p, cp, d[s][a][cp], ax[a], ay[a], az[a], t);
                if (s + 1 < kRing) shuffle_pairs(t, next);
            }
            // own sums (negated, register order) and this half's three pairs
            // inside the group
            float sx_[4], sy_[4], sz_[4];
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                sx_[a] = ax[a].x + ax[a].y;
                sy_[a] = ay[a].x + ay[a].y;
                sz_[a] = az[a].x + az[a].y;
            }
#pragma unroll
            for (int j = 0; j < 3; ++j) {
                const int u = inner_u(j), v = inner_v(j);
                const float e0 = r.x[v] - r.x[u], e1 = r.y[v] - r.y[u], e2 = r.z[v] - r.z[u];
                const float q = fmaf(e2, e2, fmaf(e1, e1, fmaf(e0, e0, kQSeed)));
                const float w = dw[j] * rsqrt_approx(q);
                sx_[u] = fmaf(w, e0, sx_[u]);
                sy_[u] = fmaf(w, e1, sy_[u]);
                sz_[u] = fmaf(w, e2, sz_[u]);
                sx_[v] = fmaf(-w, e0, sx_[v]);
                sy_[v] = fmaf(-w, e1, sy_[v]);
                sz_[v] = fmaf(-w, e2, sz_[v]);
            }
            shuffle_pairs(t, owner_src);
            float tx[4] = {t.x[0].x, t.x[0].y, t.x[1].x, t.x[1].y};
            float ty[4] = {t.y[0].x, t.y[0].y, t.y[1].x, t.y[1].y};
            float tz[4] = {t.z[0].x, t.z[0].y, t.z[1].x, t.z[1].y};
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                tx[a] -= unrot(sel, sx_, a);
                ty[a] -= unrot(sel, sy_, a);
                tz[a] -= unrot(sel, sz_, a);
            }
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                tx[a] += __shfl_xor_sync(0xffffffffu, tx[a], 16);
                ty[a] += __shfl_xor_sync(0xffffffffu, ty[a], 16);
                tz[a] += __shfl_xor_sync(0xffffffffu, tz[a], 16);
            }
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                b.x[a] = tx[a] * kInvN;
                b.y[a] = ty[a] * kInvN;
                b.z[a] = tz[a] * kInvN;
            }
        }
        if (h == 0) {
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                X[3 * a] = b.x[a];
                X[3 * a + 1] = b.y[a];
                X[3 * a + 2] = b.z[a];
            }
        }
        if (stress_out != nullptr) {
            __syncwarp();
            if (h == 0) {
                st4(sx + 4 * l, make_float4(b.x[0], b.x[1], b.x[2], b.x[3]));
                st4(sx + kN + 4 * l, make_float4(b.y[0], b.y[1], b.y[2], b.y[3]));
                st4(sx + 2 * kN + 4 * l, make_float4(b.z[0], b.z[1], b.z[2], b.z[3]));
            }
            __syncwarp();
            // every unordered pair once: offset 8's halved weights are doubled
            // back and its terms counted at half weight
            Group r;
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                r.x[a] = rot(sel, b.x, a);
                r.y[a] = rot(sel, b.y, a);
                r.z[a] = rot(sel, b.z, a);
            }
            float2 acc2 = make_float2(0.0f, 0.0f), last2 = make_float2(0.0f, 0.0f);
            const float2 m1 = make_float2(-1.0f, -1.0f);
            const float2 dbl = up ? make_float2(2.0f, 2.0f) : make_float2(1.0f, 1.0f);
#pragma unroll
            for (int s = 0; s < kRing; ++s) {
                const Pairs p = load_pairs(sx, (l + k0 + s) & 15);
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int cp = 0; cp < 2; ++cp) {
                        const float2 e0 = __ffma2_rn(make_float2(r.x[a], r.x[a]), m1, p.x[cp]);
                        const float2 e1 = __ffma2_rn(make_float2(r.y[a], r.y[a]), m1, p.y[cp]);
                        const float2 e2 = __ffma2_rn(make_float2(r.z[a], r.z[a]), m1, p.z[cp]);
                        float2 q = __fmul2_rn(e0, e0);
                        q = __ffma2_rn(e1, e1, q);
                        q = __ffma2_rn(e2, e2, q);
                        const float2 dd = s == kRing - 1 ? __fmul2_rn(d[s][a][cp], dbl) : d[s][a][cp];
                        const float2 rr = __ffma2_rn(dd, m1, make_float2(sqrt_approx(q.x), sqrt_approx(q.y)));
                        if (s == kRing - 1) last2 = __ffma2_rn(rr, rr, last2);
                        else acc2 = __ffma2_rn(rr, rr, acc2);
                    }
            }
            float acc = fmaf(up ? 0.5f : 1.0f, last2.x + last2.y, acc2.x + acc2.y);
#pragma unroll
            for (int j = 0; j < 3; ++j) acc += stress_term(r, inner_u(j), r, inner_v(j), dw[j]);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
            if (lane == 0) stress_out[m] = acc;
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
