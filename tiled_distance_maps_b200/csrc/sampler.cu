// Sampler kernels: initial noise, stand-in eps, one DDIM step, and the fused
// whole-trajectory run.
//
// ParaChromo (mdpi.com/2079-9292/15/13/2750): the reverse chain runs DDIM at a
// reduced step count (§4.1, §5.1.1) with classifier-free guidance (§3.1, ref.
// [15]); tiled regions are coupled only through the overlap projection of
// §4.3.2.  The stand-in eps is the ideal denoiser toward x0 plus Philox noise.
#include "noise.cuh"

namespace tdm {
namespace {

__device__ const UpperQuadTable kUpperQuadTable = make_upper_quads();

constexpr int kMapThreads = 256;   // CTA size of the one-map-per-iteration kernels
constexpr int kZLd = kN + 1;       // row stride of the symmetric noise tile in smem


// Fills zs[64][65] with the symmetric normal field of map noise id g.
__device__ __forceinline__ void fill_symmetric_noise(float *zs, uint64_t g, int tag, uint32_t step_word,
                                                     const PhiloxKeys &K) {
    for (int u = threadIdx.x; u < kUpperQuads; u += blockDim.x) {
        const int rq = kUpperQuadTable.v[u];
        const int r = rq >> 4, q = rq & 15;
        const float4 z = quad_normals(r, q, step_word, g, tag, K);
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const int j = 4 * q + t;
            if (j >= r) {
                zs[r * kZLd + j] = comp(z, t);
                zs[j * kZLd + r] = comp(z, t);
            }
        }
    }
}

// ---- initial state ---------------------------------------------------------

__global__ void __launch_bounds__(256) init_noise_kernel(float *__restrict__ maps, int64_t n_maps, int T,
                                                         int B, int64_t B_total, int64_t b_off,
                                                         int64_t base, const PhiloxKeys K) {
    const int64_t total = n_maps * kUpperQuads;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t m = idx / kUpperQuads;
        const int u = (int)(idx - m * kUpperQuads);
        const int rq = kUpperQuadTable.v[u];
        const int r = rq >> 4, q = rq & 15;
        const int64_t tile = m / B;
        const int b = (int)(m - tile * B);
        const int c = (int)(tile / T), k = (int)(tile - (int64_t)c * T);
        const uint64_t g = noise_id(base, c, T, k, B_total, b_off, b);
        const float4 z = quad_normals(r, q, 0u, g, TDM_STREAM_INIT, K);
        float *mp = maps + m * kMapFloats;
        if (4 * q > r) {
            st4(mp + r * kN + 4 * q, z);
#pragma unroll
            for (int t = 0; t < 4; ++t) mp[(4 * q + t) * kN + r] = comp(z, t);
        } else {
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const int j = 4 * q + t;
                if (j >= r) mp[r * kN + j] = comp(z, t);
                if (j > r) mp[j * kN + r] = comp(z, t);
            }
        }
    }
}

// ---- stand-in eps of one stream ---------------------------------------------

__global__ void __launch_bounds__(kMapThreads) eps_standin_kernel(
    const StepCoef *__restrict__ coef, int step, const float *__restrict__ maps, const float *__restrict__ x0,
    float s, int tag, const PhiloxKeys K, Tiling t, float *__restrict__ eps) {
    __shared__ float zs[kN * kZLd];
    const StepCoef cf = coef[step];
    const int64_t n = t.n_maps();
    for (int64_t m = blockIdx.x; m < n; m += gridDim.x) {
        const int64_t tile = m / t.B;
        const int b = (int)(m - tile * t.B);
        const int c = (int)(tile / t.T), k = (int)(tile - (int64_t)c * t.T);
        const uint64_t g = noise_id(t.sample_id_base, c, t.T, k, t.B_total, t.b_offset, b);
        fill_symmetric_noise(zs, g, tag, (uint32_t)step, K);
        __syncthreads();
        const float *xm = maps + m * kMapFloats;
        const float *x0m = x0 + tile * kMapFloats;
        float *em = eps + m * kMapFloats;
#pragma unroll 4
        for (int p = threadIdx.x; p < kMapFloats / 4; p += kMapThreads) {
            const int r = p >> 4, q = p & 15;
            const float4 x = ld4(xm + 4 * p);
            const float4 xr = ldg4(x0m + 4 * p);
            const float *z = zs + r * kZLd + 4 * q;
            float4 e;
            e.x = fmaf(s, z[0], (x.x - cf.sa * xr.x) * cf.isa1);
            e.y = fmaf(s, z[1], (x.y - cf.sa * xr.y) * cf.isa1);
            e.z = fmaf(s, z[2], (x.z - cf.sa * xr.z) * cf.isa1);
            e.w = fmaf(s, z[3], (x.w - cf.sa * xr.w) * cf.isa1);
            st4(em + 4 * p, e);
        }
        __syncthreads();
    }
}

// ---- one DDIM step ------------------------------------------------------------

// The guided eps and the DDIM update of one entry, in one order for every
// entry (its own map's, or its partner's across a seam).
template <bool HAS_U, bool HAS_ETA>
__device__ __forceinline__ float step_entry(const StepCoef &cf, float wc, float w, float x, float ec, float eu,
                                            float z) {
    const float e = HAS_U ? fmaf(wc, ec, -w * eu) : ec;
    const float y = fmaf(cf.a, x, cf.kb * e);
    return HAS_ETA ? fmaf(cf.ks, z, y) : y;
}

// One CTA per map.  With PROJ (the step after which the overlap projection of
// §4.3.2 is due), the CTA of tile k < T-1 also updates the partner entries of
// tile k+1 over their shared o x o block and writes the mean of the two
// updated values to both maps; the CTA of tile k > 0 leaves its own block
// with tile k-1 to that tile's CTA.  So every entry is read and written by one
// CTA, and the projection costs no pass of its own.
template <bool HAS_U, bool HAS_ETA, bool PROJ>
__global__ void __launch_bounds__(kMapThreads) ddim_step_kernel(
    const StepCoef *__restrict__ coef, int step, float *__restrict__ maps, const float *__restrict__ eps_c,
    const float *__restrict__ eps_u, float w, const PhiloxKeys K, Tiling t) {
    constexpr int kBlockLd = 33;
    __shared__ float zs[HAS_ETA ? kN * kZLd : 1];
    __shared__ float zn[HAS_ETA && PROJ ? 32 * kBlockLd : 1];    // the partner's ETA field over the block
    const StepCoef cf = coef[step];
    const float wc = 1.0f + w;
    const int64_t n = t.n_maps();
    const int o = t.overlap, s = kN - o;
    for (int64_t m = blockIdx.x; m < n; m += gridDim.x) {
        const int64_t tile = m / t.B;
        const int b = (int)(m - tile * t.B);
        const int c = (int)(tile / t.T), k = (int)(tile - (int64_t)c * t.T);
        const bool right = PROJ && k < t.T - 1, left = PROJ && k > 0;
        if (HAS_ETA) {
            const uint64_t g = noise_id(t.sample_id_base, c, t.T, k, t.B_total, t.b_offset, b);
            fill_symmetric_noise(zs, g, TDM_STREAM_ETA, (uint32_t)step, K);
            if (PROJ && right) {
                // upper quads of the partner's o x o block (map id g + B_total), mirrored
                const uint64_t gn = g + (uint64_t)t.B_total;
                const int oq4 = (o + 3) >> 2;
                for (int u = threadIdx.x; u < o * oq4; u += blockDim.x) {
                    const int r = u / oq4, q = u - r * oq4;
                    if (4 * q + 3 < r) continue;
                    const float4 z = quad_normals(r, q, (uint32_t)step, gn, TDM_STREAM_ETA, K);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int j = 4 * q + e;
                        if (j >= r && j < o) {
                            zn[r * kBlockLd + j] = comp(z, e);
                            zn[j * kBlockLd + r] = comp(z, e);
                        }
                    }
                }
            }
            __syncthreads();
        }
        float *xm = maps + m * kMapFloats;
        const float *ec = eps_c + m * kMapFloats;
        const float *eu = HAS_U ? eps_u + m * kMapFloats : nullptr;
        float *xn = xm + (int64_t)t.B * kMapFloats;    // the same sample of tile k+1
        const float *ecn = ec + (int64_t)t.B * kMapFloats;
        const float *eun = HAS_U ? eu + (int64_t)t.B * kMapFloats : nullptr;
#pragma unroll 4
        for (int p = threadIdx.x; p < kMapFloats / 4; p += kMapThreads) {
            const int r = p >> 4, c0 = 4 * (p & 15);
            const float4 x = ld4(xm + 4 * p);
            const float4 e = ldg4(ec + 4 * p);
            const float4 v = HAS_U ? ldg4(eu + 4 * p) : make_float4(0.f, 0.f, 0.f, 0.f);
            const float *z = HAS_ETA ? zs + r * kZLd + c0 : nullptr;
            float4 y;
            y.x = step_entry<HAS_U, HAS_ETA>(cf, wc, w, x.x, e.x, v.x, HAS_ETA ? z[0] : 0.f);
            y.y = step_entry<HAS_U, HAS_ETA>(cf, wc, w, x.y, e.y, v.y, HAS_ETA ? z[1] : 0.f);
            y.z = step_entry<HAS_U, HAS_ETA>(cf, wc, w, x.z, e.z, v.z, HAS_ETA ? z[2] : 0.f);
            y.w = step_entry<HAS_U, HAS_ETA>(cf, wc, w, x.w, e.w, v.w, HAS_ETA ? z[3] : 0.f);
            const bool in_left = left && r < o && c0 < o;
            const bool in_right = right && r >= s && c0 + 3 >= s;
            if (!(PROJ && (in_left || in_right))) {
                st4(xm + 4 * p, y);
            } else {
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int col = c0 + u;
                    if (in_left && col < o) continue;              // written by tile k-1's CTA
                    float val = comp(y, u);
                    if (in_right && col >= s) {
                        const int off = (r - s) * kN + (col - s);
                        const float yn = step_entry<HAS_U, HAS_ETA>(
                            cf, wc, w, xn[off], __ldg(ecn + off), HAS_U ? __ldg(eun + off) : 0.f,
                            HAS_ETA ? zn[(r - s) * kBlockLd + (col - s)] : 0.f);
                        val = 0.5f * (val + yn);
                        xn[off] = val;
                    }
                    xm[4 * p + u] = val;
                }
            }
        }
        if (HAS_ETA) __syncthreads();
    }
}

// ---- the fused whole-trajectory run -------------------------------------------
//
// One lane owns one row quad (r, 4q..4q+3) of the folded (upper-triangle)
// state of one map and keeps it in registers for all S steps.  With the
// stand-in denoiser every update is elementwise, so the only coupling between
// lanes is the overlap projection, which pairs entry (s+i, s+j) of tile k with
// entry (i, j) of tile k+1 of the same sample.  The lane plan puts both quads
// of such a pair in lanes l and l^16 of one warp, so the projection is one
// register exchange; no CTA ever waits on another.

// The lanes of one chain-sample (17 T warps) cover the 544 T upper row
// quads of its T tiles.  With overlap o = 4 oq and stride s = 64 - o, the
// upper quads of the o x o overlap block of a seam are indexed u in row-major
// order (row i < o, column quad jq < oq, 4 jq + 3 >= i: Q = 2 oq (oq + 1) of
// them), and pair p = k Q + u joins quad (s + i, sq + jq) of tile k with quad
// (i, jq) of tile k + 1 (sq = s / 4).  Warp w < P / 16 holds pairs 16 w ..
// 16 w + 15, first quads in lanes 0-15 and second quads in lanes l + 16; the
// next warp holds the last P % 16 pairs in the same way and fills its other
// lanes two at a time (l, l + 16) with the first singles; the remaining warps
// hold 32 singles each.  The singles are every other upper quad in the order
// tile, row, column quad.
//
// Two constant tables, built at compile time, hold what depends only on oq:
// the (i, jq) of each block quad u, and for each kind of tile (with or without
// a left block, with or without a right block) the (r, q) of its singles in
// order.  A lane's descriptor is then two divisions and one table read.
struct LaneTables {
    uint16_t single[9][4][kUpperQuads];    // [oq][left | right << 1][index] -> r << 4 | q
    uint8_t pair[9][144];                  // [oq][u] -> i | jq << 5
};

constexpr LaneTables make_lane_tables() {
    LaneTables t{};
    for (int oq = 0; oq <= 8; ++oq) {
        const int ov = 4 * oq, s = kN - ov, sq = kQuadsPerRow - oq;
        int u = 0;
        for (int i = 0; i < ov; ++i)
            for (int jq = 0; jq < oq; ++jq)
                if (4 * jq + 3 >= i) t.pair[oq][u++] = (uint8_t)(i | jq << 5);
        for (int kind = 0; kind < 4; ++kind) {
            const bool L = (kind & 1) != 0, R = (kind & 2) != 0;
            int n = 0;
            for (int r = 0; r < kN; ++r)
                for (int q = 0; q < kQuadsPerRow; ++q) {
                    if (4 * q + 3 < r) continue;
                    const bool left = L && r < ov && q < oq, right = R && r >= s && q >= sq;
                    if (!left && !right) t.single[oq][kind][n++] = (uint16_t)(r << 4 | q);
                }
        }
    }
    return t;
}

__device__ const LaneTables kLaneTablesDev = make_lane_tables();

// x / d for 0 <= x < 2^31 and 0 < d < 2^16, with m = ceil(2^32 / d): the
// product's top word is x / d or one more, and one comparison corrects it.
__host__ __device__ inline int div_magic(int x, int d, uint32_t m) {
    int k = (int)(((uint64_t)(uint32_t)x * m) >> 32);
    if (k * d > x) --k;
    return k;
}

__host__ __device__ inline uint32_t div_magic_of(int d) {
    return d > 1 ? (uint32_t)((0x100000000ULL + (uint64_t)d - 1) / (uint64_t)d) : 0xFFFFFFFFu;
}

// q | r << 4 | k << 10 | paired << 31 of lane `lane` of warp `wi`; mq and
// mmid are div_magic_of(Q) and div_magic_of(544 - 2 Q).
__host__ __device__ inline uint32_t run_lane_desc(const LaneTables &tab, int T, int overlap, int wi, int lane,
                                                  uint32_t mq, uint32_t mmid) {
    const int oq = overlap >> 2, sq = kQuadsPerRow - oq;
    const int Q = 2 * oq * (oq + 1);
    const int P = (T - 1) * Q, Pw = P >> 4, Pr = P & 15;
    const int pl = lane & 15;
    const bool hi = lane >= 16;
    if (wi < Pw || (wi == Pw && pl < Pr)) {
        const int p = 16 * wi + pl;
        const int k = div_magic(p, Q, mq);
        const int e = tab.pair[oq][p - k * Q];
        const int i = e & 31, jq = e >> 5;
        return hi ? ((uint32_t)jq | (uint32_t)i << 4 | (uint32_t)(k + 1) << 10 | 0x80000000u)
                  : ((uint32_t)(sq + jq) | (uint32_t)(4 * sq + i) << 4 | (uint32_t)k << 10 | 0x80000000u);
    }
    int si;
    if (wi == Pw && Pr > 0)
        si = 2 * (pl - Pr) + (hi ? 1 : 0);
    else
        si = (Pr > 0 ? 2 * (16 - Pr) : 0) + 32 * (wi - Pw - (Pr > 0 ? 1 : 0)) + lane;
    // the tile: tile 0 and tile T-1 lose one block each, the others two
    const int n_first = kUpperQuads - (T > 1 ? Q : 0), n_mid = kUpperQuads - 2 * Q;
    int k = 0, sl = si;
    if (si >= n_first) {
        const int rem = si - n_first;
        k = 1 + div_magic(rem, n_mid, mmid);
        sl = rem - (k - 1) * n_mid;
        if (k >= T - 1) {
            k = T - 1;
            sl = rem - (T - 2) * n_mid;
        }
    }
    const int kind = (k > 0 ? 1 : 0) | (k < T - 1 ? 2 : 0);
    const uint32_t rq = tab.single[oq][kind][sl];
    return (rq & 15u) | (rq >> 4) << 4 | (uint32_t)k << 10;
}

struct RunArgs {
    const StepCoef *coef;
    float *maps;
    const float *x0;
    int64_t total_warps;       // C * B * 17 T
    int64_t B_total, b_off, base;
    int S, T, B, overlap, sync_every, warps_per_chain;
    uint32_t mq, mmid;         // division constants of the lane descriptors
    int first, last;           // steps first, first-1, .., last (first = S-1, last = 0 for a whole run)
    float cc, cu;              // (1 + w) s_c and w s_u
    PhiloxKeys K;
};

// Round 1 of Philox for a lane whose counter words 0 (position) and 2 (noise
// id, low half) never change: its products are computed once, and the round-1
// output for step word i and stream tag t is (A ^ i, L1, B ^ t << 24, L0).
struct LaneCounter {
    uint32_t A, L1, B, L0;
};

__device__ __forceinline__ LaneCounter lane_counter(int r, int q, uint64_t g, const PhiloxKeys &K) {
    const uint64_t p0 = (uint64_t)Philox::M0 * (((uint32_t)r << 4) | (uint32_t)q);
    const uint64_t p1 = (uint64_t)Philox::M1 * (uint32_t)g;
    LaneCounter L;
    L.A = (uint32_t)(p1 >> 32) ^ K.k0[0];
    L.L1 = (uint32_t)p1;
    L.B = (uint32_t)(p0 >> 32) ^ ((uint32_t)(g >> 32) & 0xFFFFFFu) ^ K.k1[0];
    L.L0 = (uint32_t)p0;
    return L;
}

// Round-2 output words 0 and 1 of stream tag t: the product of round-1 word 2
// (B ^ t << 24) carries the tag but not the step word, so it is computed once
// per lane and stream.
__device__ __forceinline__ uint2 round2_xy(const LaneCounter &L, int tag, const PhiloxKeys &K) {
    const uint64_t p1 = (uint64_t)Philox::M1 * (L.B ^ ((uint32_t)tag << 24));
    return make_uint2((uint32_t)(p1 >> 32) ^ L.L1 ^ K.k0[1], (uint32_t)p1);
}

// The draws of NS streams of one step for one lane (xy: round2_xy of each
// stream), as the radius and angle parts of box_muller_packed, each stream's
// term nk[s] rho (cos | sin) added to (a02, a13) as soon as it is drawn.
// Round 2's product of word 0 (A ^ step word) is shared by the streams.
template <int NS, bool VOTE>
__device__ __forceinline__ void lane_noise_packed(const LaneCounter &L, uint32_t step_word, const uint2 (&xy)[NS],
                                                  const PhiloxKeys &K, const float2 (&nk)[NS], float2 &a02,
                                                  float2 &a13) {
    const uint64_t p0 = (uint64_t)Philox::M0 * (L.A ^ step_word);
    const uint32_t w2 = (uint32_t)(p0 >> 32) ^ L.L0 ^ K.k1[1];
    const uint32_t w3 = (uint32_t)p0;
#pragma unroll
    for (int s = 0; s < NS; ++s) {
        const uint4 c = philox_rounds<2>(make_uint4(xy[s].x, xy[s].y, w2, w3), K);
        float2 rho, cs, sn;
        box_muller_packed<VOTE>(c, rho, cs, sn);
        const float2 t = __fmul2_rn(nk[s], rho);
        a02 = __ffma2_rn(t, cs, a02);
        a13 = __ffma2_rn(t, sn, a13);
    }
}

// WIDE: 8-warp CTAs of a launch large enough to be throughput-bound (the
// series behind a warp vote, the partner's x0 exchanged at each projection
// to save registers); otherwise 2-warp CTAs of a latency-bound launch (the
// series selected per pair, the x0 term of the projection formed once).
template <bool HAS_U, bool HAS_ETA, bool INIT, bool WIDE>
__global__ void __launch_bounds__(256) ddim_run_kernel(const RunArgs a) {
    // per step, packed (both halves equal): (ka, kx0) then (-kc, -ku) kRadScale,
    // the noise coefficients times the factor z = -kRadScale rho cos (sin) of
    // box_muller_packed's parts; then [S] -ks kRadScale
    extern __shared__ float4 sco[];
    float2 *sks = reinterpret_cast<float2 *>(sco + 2 * a.S);
    for (int i = threadIdx.x; i < a.S; i += blockDim.x) {
        const StepCoef c = a.coef[i];
        const float nkc = -(c.kb * a.cc) * kRadScale, nku = (c.kb * a.cu) * kRadScale;
        sco[2 * i] = make_float4(c.ka, c.ka, c.kx0, c.kx0);
        sco[2 * i + 1] = make_float4(nkc, nkc, nku, nku);
        if (HAS_ETA) sks[i] = make_float2(-c.ks * kRadScale, -c.ks * kRadScale);
    }
    __syncthreads();

    const int lane = threadIdx.x & 31;
    const int64_t gw = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (gw >= a.total_warps) return;
    const int64_t cs = gw / a.warps_per_chain;               // chain-sample c * B + b
    const int wi = (int)(gw - cs * a.warps_per_chain);
    const uint32_t d = run_lane_desc(kLaneTablesDev, a.T, a.overlap, wi, lane, a.mq, a.mmid);
    const int q = d & 15, r = (d >> 4) & 63, k = (d >> 10) & 0xFFFF;
    const bool paired = (d >> 31) != 0;
    const int c = (int)(cs / a.B), b = (int)(cs - (int64_t)c * a.B);
    const int64_t tile = (int64_t)c * a.T + k;
    float *mp = a.maps + (tile * a.B + b) * kMapFloats;
    const uint64_t g = (uint64_t)(a.base + tile * a.B_total + a.b_off + b);
    const float4 xr = ldg4(a.x0 + tile * kMapFloats + r * kN + 4 * q);
    const float2 r02 = make_float2(xr.x, xr.z), r13 = make_float2(xr.y, xr.w);
    const LaneCounter L = lane_counter(r, q, g, a.K);

    // the state as packed column pairs (x0, x2) and (x1, x3) of the quad
    float2 x02, x13;
    if (INIT) {
        const uint2 xy[1] = {round2_xy(L, TDM_STREAM_INIT, a.K)};
        const float2 nk[1] = {make_float2(-kRadScale, -kRadScale)};
        x02 = x13 = make_float2(0.0f, 0.0f);
        lane_noise_packed<1, WIDE>(L, 0u, xy, a.K, nk, x02, x13);
    } else {
        const float4 x = ld4(mp + r * kN + 4 * q);
        x02 = make_float2(x.x, x.z);
        x13 = make_float2(x.y, x.w);
    }
    const bool warp_pairs = __shfl_sync(0xffffffffu, paired ? 1 : 0, 0) != 0;
    const bool sync_warp = a.T > 1 && a.sync_every > 0 && warp_pairs;
    // the projection follows the steps counted from the start of the whole
    // run, so a run resumed at step `first` projects where the whole run would
    int until_sync = a.sync_every > 0 ? a.sync_every - (a.S - 1 - a.first) % a.sync_every : 0;
    // the state is stepped as y = x - gam x0 (the loop's x02, x13), so the x0
    // term of every step is one scalar update of gam: x' = ka x + kx0 x0 + n
    // gives y' = ka y + n and gam' = ka gam + kx0; x = y + gam x0 at the end.
    // The projection averages x over a pair: y' = (y + y_o) / 2 + gam d with
    // d = (x0_o - x0) / 2 (zero where the two tiles' x0 agree).
    float gam = 0.0f;
    float2 d02 = make_float2(0.f, 0.f), d13 = make_float2(0.f, 0.f);
    const auto half_x0_gap = [&]() {    // (x0 of the partner - x0) / 2
        d02.x = __shfl_xor_sync(0xffffffffu, r02.x, 16);
        d02.y = __shfl_xor_sync(0xffffffffu, r02.y, 16);
        d13.x = __shfl_xor_sync(0xffffffffu, r13.x, 16);
        d13.y = __shfl_xor_sync(0xffffffffu, r13.y, 16);
        d02 = __fmul2_rn(make_float2(0.5f, 0.5f), __fadd2_rn(d02, make_float2(-r02.x, -r02.y)));
        d13 = __fmul2_rn(make_float2(0.5f, 0.5f), __fadd2_rn(d13, make_float2(-r13.x, -r13.y)));
    };
    if (!WIDE && sync_warp) half_x0_gap();

    constexpr int NS = 1 + (HAS_U ? 1 : 0) + (HAS_ETA ? 1 : 0);
    constexpr int kTags[3] = {TDM_STREAM_EPS_C, HAS_U ? TDM_STREAM_EPS_U : TDM_STREAM_ETA, TDM_STREAM_ETA};
    uint2 xy[NS];
#pragma unroll
    for (int s = 0; s < NS; ++s) xy[s] = round2_xy(L, kTags[s], a.K);

    for (int i = a.first; i >= a.last; --i) {
        const float4 c0 = sco[2 * i], c1 = sco[2 * i + 1];
        const float2 ka = make_float2(c0.x, c0.y);
        const float2 nkc = make_float2(c1.x, c1.y), nku = make_float2(c1.z, c1.w);
        float2 nk[NS];
        nk[0] = nkc;
        if (HAS_U) nk[1] = nku;
        if (HAS_ETA) nk[NS - 1] = sks[i];
        float2 a02 = make_float2(0.f, 0.f), a13 = make_float2(0.f, 0.f);
        lane_noise_packed<NS, WIDE>(L, (uint32_t)i, xy, a.K, nk, a02, a13);
        x02 = __ffma2_rn(ka, x02, a02);
        x13 = __ffma2_rn(ka, x13, a13);
        gam = fmaf(c0.x, gam, c0.z);
        if (sync_warp && --until_sync == 0) {
            until_sync = a.sync_every;
            float2 o02, o13;
            o02.x = __shfl_xor_sync(0xffffffffu, x02.x, 16);
            o02.y = __shfl_xor_sync(0xffffffffu, x02.y, 16);
            o13.x = __shfl_xor_sync(0xffffffffu, x13.x, 16);
            o13.y = __shfl_xor_sync(0xffffffffu, x13.y, 16);
            if (WIDE) half_x0_gap();
            if (paired) {
                const float2 g2 = make_float2(gam, gam);
                x02 = __ffma2_rn(g2, d02, __fmul2_rn(make_float2(0.5f, 0.5f), __fadd2_rn(x02, o02)));
                x13 = __ffma2_rn(g2, d13, __fmul2_rn(make_float2(0.5f, 0.5f), __fadd2_rn(x13, o13)));
            }
        }
    }
    x02 = __ffma2_rn(make_float2(gam, gam), r02, x02);
    x13 = __ffma2_rn(make_float2(gam, gam), r13, x13);
    const float4 x = make_float4(x02.x, x13.x, x02.y, x13.y);

    // unfold: the quad's upper entries go to (r, j) and their mirrors to (j, r)
    if (4 * q > r) {
        st4(mp + r * kN + 4 * q, x);
#pragma unroll
        for (int t = 0; t < 4; ++t) mp[(4 * q + t) * kN + r] = comp(x, t);
    } else {
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const int j = 4 * q + t;
            if (j >= r) mp[r * kN + j] = comp(x, t);
            if (j > r) mp[j * kN + r] = comp(x, t);
        }
    }
}

// ---- the noise primitives on caller words (for exhaustive checks) -------------

__global__ void __launch_bounds__(256) philox_kernel(const uint4 *__restrict__ ctr, int64_t n, const PhiloxKeys K,
                                                     uint4 *__restrict__ out) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        out[i] = philox4x32_10(ctr[i], K);
}

__global__ void __launch_bounds__(256) box_muller_kernel(const uint2 *__restrict__ words, int64_t n,
                                                         float2 *__restrict__ z) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const uint2 w = words[i];
        z[i] = box_muller(w.x, w.y);
    }
}

int grid_for(int64_t work_items, int per_sm) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t cap = (int64_t)sms * per_sm;
    return (int)(work_items < cap ? (work_items > 0 ? work_items : 1) : cap);
}

}  // namespace

// ---- host side -------------------------------------------------------------------

}  // namespace tdm

extern "C" tdm_status tdm_fused_lane_map(int32_t T, int32_t overlap, uint32_t *out, int64_t n) {
    if (T < 1 || T > 0xFFFF || out == nullptr) return TDM_EINVAL;
    const int ov = T > 1 ? overlap : 0;
    if (ov < 0 || ov > 32 || ov % 4 != 0 || (T > 1 && ov < 4)) return TDM_EINVAL;
    if (n < (int64_t)tdm::kUpperQuads * T) return TDM_EINVAL;
    static const tdm::LaneTables tab = tdm::make_lane_tables();
    const int oq = ov >> 2, Q = 2 * oq * (oq + 1);
    const uint32_t mq = tdm::div_magic_of(Q), mmid = tdm::div_magic_of(tdm::kUpperQuads - 2 * Q);
    for (int wi = 0; wi < 17 * T; ++wi)
        for (int l = 0; l < 32; ++l) out[(int64_t)wi * 32 + l] = tdm::run_lane_desc(tab, T, ov, wi, l, mq, mmid);
    return TDM_OK;
}

namespace tdm {

cudaError_t launch_init_noise(float *maps, const Tiling &t, uint64_t seed, cudaStream_t st) {
    const int64_t items = t.n_maps() * kUpperQuads;
    const int grid = grid_for((items + 255) / 256, 16);
    init_noise_kernel<<<grid, 256, 0, st>>>(maps, t.n_maps(), t.T, t.B, t.B_total, t.b_offset,
                                            t.sample_id_base, philox_keys(seed));
    return cudaGetLastError();
}

cudaError_t launch_eps_standin(const StepCoef *coef, int step, const float *maps, const float *x0, float s,
                               int tag, uint64_t seed, const Tiling &t, float *eps, cudaStream_t st) {
    const int grid = grid_for(t.n_maps(), 8);
    eps_standin_kernel<<<grid, kMapThreads, 0, st>>>(coef, step, maps, x0, s, tag, philox_keys(seed), t, eps);
    return cudaGetLastError();
}

cudaError_t launch_ddim_step(const StepCoef *coef, int step, float *maps, const float *eps_c,
                             const float *eps_u, float w, bool has_eta, bool project, uint64_t seed,
                             const Tiling &t, cudaStream_t st) {
    const int grid = grid_for(t.n_maps(), 8);
    const PhiloxKeys K = philox_keys(seed);
    const bool has_u = eps_u != nullptr && w != 0.0f;
    const int v = (has_u ? 4 : 0) | (has_eta ? 2 : 0) | (project && t.T > 1 ? 1 : 0);
#define TDM_STEP(U, E, P)                                                                                    \
    ddim_step_kernel<U, E, P><<<grid, kMapThreads, 0, st>>>(coef, step, maps, eps_c, U ? eps_u : nullptr, w, K, t)
    switch (v) {
        case 7: TDM_STEP(true, true, true); break;
        case 6: TDM_STEP(true, true, false); break;
        case 5: TDM_STEP(true, false, true); break;
        case 4: TDM_STEP(true, false, false); break;
        case 3: TDM_STEP(false, true, true); break;
        case 2: TDM_STEP(false, true, false); break;
        case 1: TDM_STEP(false, false, true); break;
        default: TDM_STEP(false, false, false); break;
    }
#undef TDM_STEP
    return cudaGetLastError();
}

template <bool U, bool E, bool I, bool V>
static cudaError_t run_variant4(const RunArgs &a, int grid, int threads, size_t smem, cudaStream_t st) {
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(ddim_run_kernel<U, E, I, V>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    ddim_run_kernel<U, E, I, V><<<grid, threads, smem, st>>>(a);
    return cudaGetLastError();
}

// 8-warp CTAs: the WIDE kernel; 2-warp CTAs (small launches): the other
template <bool U, bool E, bool I>
static cudaError_t run_variant(const RunArgs &a, int grid, int threads, size_t smem, cudaStream_t st) {
    return threads == 256 ? run_variant4<U, E, I, true>(a, grid, threads, smem, st)
                          : run_variant4<U, E, I, false>(a, grid, threads, smem, st);
}

cudaError_t launch_ddim_run(const StepCoef *coef, int S, int first, int n_steps, float *maps, const float *x0,
                            float w, float s_c, float s_u, bool has_eta, uint64_t seed, bool init_noise,
                            const Tiling &t, cudaStream_t st) {
    RunArgs a;
    a.first = first;
    a.last = first - n_steps + 1;
    a.coef = coef;
    a.maps = maps;
    a.x0 = x0;
    a.overlap = t.T > 1 ? t.overlap : 0;
    {
        const int oq = a.overlap >> 2, Q = 2 * oq * (oq + 1);
        a.mq = div_magic_of(Q);
        a.mmid = div_magic_of(kUpperQuads - 2 * Q);
    }
    a.warps_per_chain = 17 * t.T;
    a.total_warps = (int64_t)t.C * t.B * a.warps_per_chain;
    a.B_total = t.B_total;
    a.b_off = t.b_offset;
    a.base = t.sample_id_base;
    a.S = S;
    a.T = t.T;
    a.B = t.B;
    a.sync_every = t.sync_every;
    a.cc = (1.0f + w) * s_c;
    a.cu = w * s_u;
    a.K = philox_keys(seed);
    // a launch too small to give every SM several 8-warp CTAs runs 2-warp CTAs
    // instead, spreading its warps over more SMs (fewer warps per scheduler:
    // the run is then latency-bound, not issue-bound)
    int sms = 148, dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int wpc = a.total_warps >= 4LL * 8 * sms ? 8 : 2;
    const int64_t grid64 = (a.total_warps + wpc - 1) / wpc;
    if (grid64 > 0x7FFFFFFF) return cudaErrorInvalidConfiguration;
    const int grid = (int)grid64;
    const size_t smem = (size_t)S * (2 * sizeof(float4) + (has_eta ? sizeof(float2) : 0));
    const bool has_u = w != 0.0f;
    if (has_u) {
        if (has_eta) return init_noise ? run_variant<true, true, true>(a, grid, 32 * wpc, smem, st)
                                       : run_variant<true, true, false>(a, grid, 32 * wpc, smem, st);
        return init_noise ? run_variant<true, false, true>(a, grid, 32 * wpc, smem, st)
                          : run_variant<true, false, false>(a, grid, 32 * wpc, smem, st);
    }
    if (has_eta) return init_noise ? run_variant<false, true, true>(a, grid, 32 * wpc, smem, st)
                                   : run_variant<false, true, false>(a, grid, 32 * wpc, smem, st);
    return init_noise ? run_variant<false, false, true>(a, grid, 32 * wpc, smem, st)
                      : run_variant<false, false, false>(a, grid, 32 * wpc, smem, st);
}

}  // namespace tdm

namespace tdm {

cudaError_t launch_philox(const uint32_t *ctr, int64_t n, uint64_t seed, uint32_t *out, cudaStream_t st) {
    if (n <= 0) return cudaSuccess;
    const int grid = grid_for((n + 255) / 256, 16);
    philox_kernel<<<grid, 256, 0, st>>>(reinterpret_cast<const uint4 *>(ctr), n, philox_keys(seed),
                                        reinterpret_cast<uint4 *>(out));
    return cudaGetLastError();
}

cudaError_t launch_box_muller(const uint32_t *words, int64_t n_pairs, float *z, cudaStream_t st) {
    if (n_pairs <= 0) return cudaSuccess;
    const int grid = grid_for((n_pairs + 255) / 256, 16);
    box_muller_kernel<<<grid, 256, 0, st>>>(reinterpret_cast<const uint2 *>(words), n_pairs,
                                            reinterpret_cast<float2 *>(z));
    return cudaGetLastError();
}

}  // namespace tdm
