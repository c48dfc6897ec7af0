// Non-overlap drift of synchronised maps from an independent run.
//
// ParaChromo (mdpi.com/2079-9292/15/13/2750), §5.7, Table 8: beside the
// overlap discrepancy, the synchronisation-frequency sweep reports how far the
// distance values outside the overlapping subblocks move away from the matched
// unsynchronised run.  Per tile (c, k), over its samples and its non-overlap
// entries (all but the upper-left o x o block when k > 0 and the lower-right
// o x o block when k < T-1): num = sum |S - V|, den = sum |V|; the relative
// drift of a chain is sum_k num / sum_k den.
//
// One CTA per (tile, chunk of samples): thread t owns float4 columns t, t+256,
// t+512, t+768 of every map (coalesced), with the non-overlap mask of its 16
// entries fixed once; the CTA reduces in a fixed order, so results do not
// depend on scheduling.  A finalize pass, one warp per chain, adds the chunks
// and forms the ratio.
#include "common.cuh"

namespace tdm {
namespace {

constexpr int kDriftThreads = 256;
constexpr int kF4PerThread = kMapFloats / 4 / kDriftThreads;    // 4

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

__device__ __forceinline__ bool counts(int row, int col, int k, int T, int o) {
    const bool left = k > 0 && row < o && col < o;
    const bool right = k < T - 1 && row >= kN - o && col >= kN - o;
    return !(left || right);
}

// partial[(tile * chunks + chunk) * 2 + {0, 1}] = (sum |S - V|, sum |V|)
__global__ void __launch_bounds__(kDriftThreads) drift_sums_kernel(const float *__restrict__ S,
                                                                   const float *__restrict__ V, int T, int B,
                                                                   int o, int chunks, float *__restrict__ partial) {
    __shared__ float red[2][kDriftThreads / 32];
    const int64_t tile = blockIdx.x;
    const int chunk = blockIdx.y;
    const int k = (int)(tile % T);
    const int per = (B + chunks - 1) / chunks;
    const int b0 = chunk * per, b1 = min(B, b0 + per);
    float4 mask[kF4PerThread];
#pragma unroll
    for (int r = 0; r < kF4PerThread; ++r) {
        const int q = threadIdx.x + r * kDriftThreads;
        const int row = q >> 4, col = (q & 15) << 2;
        mask[r] = make_float4(counts(row, col, k, T, o) ? 1.f : 0.f, counts(row, col + 1, k, T, o) ? 1.f : 0.f,
                              counts(row, col + 2, k, T, o) ? 1.f : 0.f, counts(row, col + 3, k, T, o) ? 1.f : 0.f);
    }
    float num = 0.0f, den = 0.0f;
    const float4 *s4 = reinterpret_cast<const float4 *>(S + tile * B * kMapFloats);
    const float4 *v4 = reinterpret_cast<const float4 *>(V + tile * B * kMapFloats);
    for (int b = b0; b < b1; ++b) {
        const int64_t base = (int64_t)b * (kMapFloats / 4);
#pragma unroll
        for (int r = 0; r < kF4PerThread; ++r) {
            const int q = threadIdx.x + r * kDriftThreads;
            const float4 s = __ldcs(s4 + base + q), v = __ldcs(v4 + base + q);
            const float4 m = mask[r];
            num = fmaf(m.x, fabsf(s.x - v.x), num);
            num = fmaf(m.y, fabsf(s.y - v.y), num);
            num = fmaf(m.z, fabsf(s.z - v.z), num);
            num = fmaf(m.w, fabsf(s.w - v.w), num);
            den = fmaf(m.x, fabsf(v.x), den);
            den = fmaf(m.y, fabsf(v.y), den);
            den = fmaf(m.z, fabsf(v.z), den);
            den = fmaf(m.w, fabsf(v.w), den);
        }
    }
    num = warp_sum(num);
    den = warp_sum(den);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) {
        red[0][warp] = num;
        red[1][warp] = den;
    }
    __syncthreads();
    if (warp == 0) {
        float a = lane < kDriftThreads / 32 ? red[0][lane] : 0.0f;
        float d = lane < kDriftThreads / 32 ? red[1][lane] : 0.0f;
        a = warp_sum(a);
        d = warp_sum(d);
        if (lane == 0) {
            partial[(tile * chunks + chunk) * 2] = a;
            partial[(tile * chunks + chunk) * 2 + 1] = d;
        }
    }
}

// One warp per chain: tile sums over the chunks (written when chunks > 1) and
// the chain's ratio (written when drift is not NULL).
__global__ void __launch_bounds__(256) drift_finalize_kernel(const float *__restrict__ partial, int64_t C, int T,
                                                             int chunks, float *__restrict__ tile_sums,
                                                             float *__restrict__ drift) {
    const int lane = threadIdx.x & 31;
    const int64_t c = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (c >= C) return;
    float num = 0.0f, den = 0.0f;
    for (int k = lane; k < T; k += 32) {
        const int64_t tile = c * T + k;
        float a = 0.0f, d = 0.0f;
        for (int ch = 0; ch < chunks; ++ch) {
            a += partial[(tile * chunks + ch) * 2];
            d += partial[(tile * chunks + ch) * 2 + 1];
        }
        if (chunks > 1) {
            tile_sums[tile * 2] = a;
            tile_sums[tile * 2 + 1] = d;
        }
        num += a;
        den += d;
    }
    num = warp_sum(num);
    den = warp_sum(den);
    if (drift != nullptr && lane == 0) drift[c] = num / den;
}

}  // namespace

int drift_chunks(int64_t tiles, int B) {
    // split a tile's samples over CTAs only when there are too few tiles to
    // fill the GPU: about four CTAs per SM
    const int64_t target = 4LL * 148;
    if (tiles >= target) return 1;
    int64_t ch = (target + tiles - 1) / tiles;
    return (int)(ch < B ? ch : B);
}

cudaError_t launch_drift(const float *S, const float *V, const Tiling &t, float *scratch, int chunks,
                         float *tile_sums, float *drift, cudaStream_t st) {
    const int64_t tiles = (int64_t)t.C * t.T;
    float *partial = chunks > 1 ? scratch : tile_sums;
    drift_sums_kernel<<<dim3((unsigned)tiles, (unsigned)chunks), kDriftThreads, 0, st>>>(S, V, t.T, t.B, t.overlap,
                                                                                         chunks, partial);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || (chunks == 1 && drift == nullptr)) return e;
    const int64_t blocks = ((int64_t)t.C * 32 + 255) / 256;
    drift_finalize_kernel<<<(unsigned)blocks, 256, 0, st>>>(partial, t.C, t.T, chunks, tile_sums, drift);
    return cudaGetLastError();
}

}  // namespace tdm
