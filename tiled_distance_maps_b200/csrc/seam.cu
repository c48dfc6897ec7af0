// Overlap projection and seam discrepancy.
//
// ParaChromo (mdpi.com/2079-9292/15/13/2750) §4.3.2, Algorithm 1: for adjacent
// regions k, k+1 and the same sample b, the lower-right o x o block of region k
// and the upper-left o x o block of region k+1 hold the same bead pairs; both
// become their elementwise mean.  §5.5 Eq. (6): the seam discrepancy is the mean
// over that block of |mean_b (block of k) - mean_b (block of k+1)|.
#include "common.cuh"

namespace tdm {
namespace {

__global__ void __launch_bounds__(256) seam_project_kernel(float *__restrict__ maps, int C, int T, int B,
                                                           int o) {
    const int s = kN - o;
    const int64_t per_sample = (int64_t)o * o;
    const int64_t total = (int64_t)C * (T - 1) * B * per_sample;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int e = (int)(idx % per_sample);
        int64_t rest = idx / per_sample;
        const int b = (int)(rest % B);
        rest /= B;
        const int k = (int)(rest % (T - 1));
        const int c = (int)(rest / (T - 1));
        const int i = e / o, j = e - (e / o) * o;
        float *pa = maps + ((((int64_t)c * T + k) * B + b) * kMapFloats) + (s + i) * kN + (s + j);
        float *pb = maps + ((((int64_t)c * T + k + 1) * B + b) * kMapFloats) + i * kN + j;
        const float m = 0.5f * (*pa + *pb);
        *pa = m;
        *pb = m;
    }
}

// Partial sums over a chunk of samples of (right block of tile k - left block
// of tile k+1): partial[seam][chunk][o*o].
__global__ void __launch_bounds__(256) seam_sums_kernel(const float *__restrict__ maps, int T, int B, int o,
                                                        int chunks, float *__restrict__ partial) {
    const int seam = blockIdx.x;          // c * (T-1) + k
    const int chunk = blockIdx.y;
    const int c = seam / (T - 1), k = seam - c * (T - 1);
    const int s = kN - o;
    const int per = (B + chunks - 1) / chunks;
    const int b0 = chunk * per, b1 = min(B, b0 + per);
    const int oo = o * o;
    const float *ta = maps + (((int64_t)c * T + k) * B) * kMapFloats;
    const float *tb = maps + (((int64_t)c * T + k + 1) * B) * kMapFloats;
    for (int e = threadIdx.x; e < oo; e += blockDim.x) {
        const int i = e / o, j = e - (e / o) * o;
        const int offa = (s + i) * kN + (s + j), offb = i * kN + j;
        float acc = 0.0f;
        for (int b = b0; b < b1; ++b)
            acc += __ldg(ta + (int64_t)b * kMapFloats + offa) - __ldg(tb + (int64_t)b * kMapFloats + offb);
        partial[((int64_t)seam * chunks + chunk) * oo + e] = acc;
    }
}

// sums[seam][e] = sum over chunks of partial[seam][chunk][e]
__global__ void __launch_bounds__(256) seam_reduce_kernel(const float *__restrict__ partial, int64_t n_seams,
                                                          int oo, int chunks, float *__restrict__ sums) {
    const int64_t total = n_seams * oo;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t seam = idx / oo;
        const int e = (int)(idx - seam * oo);
        float acc = 0.0f;
        for (int ch = 0; ch < chunks; ++ch) acc += partial[(seam * chunks + ch) * oo + e];
        sums[idx] = acc;
    }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

// out[seam] = mean_e |sum over chunks of partial[seam][chunk][e] * inv_b|
__global__ void __launch_bounds__(256) seam_finalize_kernel(const float *__restrict__ partial, int oo,
                                                            int chunks, float inv_b, float *__restrict__ out) {
    __shared__ float red[8];
    const int64_t seam = blockIdx.x;
    float local = 0.0f;
    for (int e = threadIdx.x; e < oo; e += blockDim.x) {
        float acc = 0.0f;
        for (int ch = 0; ch < chunks; ++ch) acc += partial[(seam * chunks + ch) * oo + e];
        local += fabsf(acc * inv_b);
    }
    local = warp_sum(local);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = local;
    __syncthreads();
    if (threadIdx.x < 32) {
        float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.0f;
        v = warp_sum(v);
        if (threadIdx.x == 0) out[seam] = v / (float)oo;
    }
}

// One warp per seam, all samples: out[seam] directly, for many seams with few
// samples each (lane e sums entry e, e+32, .. over the samples).
__global__ void __launch_bounds__(256) seam_direct_warp_kernel(const float *__restrict__ maps, int64_t n_seams,
                                                               int T, int B, int o, float inv_b,
                                                               float *__restrict__ out) {
    const int lane = threadIdx.x & 31;
    const int s = kN - o;
    const int oo = o * o;
    for (int64_t seam = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; seam < n_seams;
         seam += ((int64_t)gridDim.x * blockDim.x) >> 5) {
        const int64_t c = seam / (T - 1);
        const int k = (int)(seam - c * (T - 1));
        const float *ta = maps + ((c * T + k) * B) * kMapFloats;
        const float *tb = maps + ((c * T + k + 1) * B) * kMapFloats;
        float local = 0.0f;
        for (int e = lane; e < oo; e += 32) {
            const int i = e / o, j = e - (e / o) * o;
            const float *pa = ta + (s + i) * kN + (s + j), *pb = tb + i * kN + j;
            float acc = 0.0f;
            for (int b = 0; b < B; ++b) acc += __ldg(pa + (int64_t)b * kMapFloats) - __ldg(pb + (int64_t)b * kMapFloats);
            local += fabsf(acc * inv_b);
        }
        local = warp_sum(local);
        if (lane == 0) out[seam] = local / (float)oo;
    }
}

// One CTA per seam, all samples: out[seam] directly (few samples per seam).
// Thread e sums entry e of the block difference over the samples (unrolled,
// so the loads of several samples are in flight together); the CTA then
// reduces |mean| over the entries in a fixed order.
__global__ void __launch_bounds__(256) seam_direct_kernel(const float *__restrict__ maps, int64_t n_seams,
                                                          int T, int B, int o, float inv_b,
                                                          float *__restrict__ out) {
    __shared__ float red[8];
    const int s = kN - o;
    const int oo = o * o;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    for (int64_t seam = blockIdx.x; seam < n_seams; seam += gridDim.x) {
        const int64_t c = seam / (T - 1);
        const int k = (int)(seam - c * (T - 1));
        const float *ta = maps + ((c * T + k) * B) * kMapFloats;
        const float *tb = maps + ((c * T + k + 1) * B) * kMapFloats;
        float local = 0.0f;
        for (int e = threadIdx.x; e < oo; e += blockDim.x) {
            const int i = e / o, j = e - (e / o) * o;
            const float *pa = ta + (s + i) * kN + (s + j), *pb = tb + i * kN + j;
            float acc = 0.0f;
#pragma unroll 8
            for (int b = 0; b < B; ++b) acc += __ldg(pa + (int64_t)b * kMapFloats) - __ldg(pb + (int64_t)b * kMapFloats);
            local += fabsf(acc * inv_b);
        }
        local = warp_sum(local);
        if (lane == 0) red[warp] = local;
        __syncthreads();
        if (warp == 0) {
            float v = lane < nwarps ? red[lane] : 0.0f;
            v = warp_sum(v);
            if (lane == 0) out[seam] = v / (float)oo;
        }
        __syncthreads();
    }
}

int sm_count() {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

}  // namespace

int seam_chunks(int64_t n_seams, int B) {
    // split the samples of a seam over CTAs only when there are too few seams
    // to fill the GPU; 8 samples per chunk at least
    const int64_t target = 4LL * 148;
    if (n_seams >= target / 2 || B <= 8) return 1;
    int64_t ch = (target + n_seams - 1) / n_seams;
    ch = ch < (B + 7) / 8 ? ch : (B + 7) / 8;
    return (int)(ch < 1 ? 1 : ch);
}

cudaError_t launch_seam_project(float *maps, const Tiling &t, cudaStream_t st) {
    const int64_t total = (int64_t)t.C * (t.T - 1) * t.B * t.overlap * t.overlap;
    if (total <= 0) return cudaSuccess;
    int64_t grid = (total + 255) / 256;
    const int64_t cap = (int64_t)sm_count() * 16;
    if (grid > cap) grid = cap;
    seam_project_kernel<<<(int)grid, 256, 0, st>>>(maps, t.C, t.T, t.B, t.overlap);
    return cudaGetLastError();
}

cudaError_t launch_seam_sums(const float *maps, const Tiling &t, float *partial, int chunks, cudaStream_t st) {
    const int64_t n_seams = (int64_t)t.C * (t.T - 1);
    if (n_seams <= 0) return cudaSuccess;
    if (n_seams > 0x7FFFFFFF) return cudaErrorInvalidConfiguration;
    dim3 grid((unsigned)n_seams, (unsigned)chunks);
    seam_sums_kernel<<<grid, 256, 0, st>>>(maps, t.T, t.B, t.overlap, chunks, partial);
    return cudaGetLastError();
}

cudaError_t launch_seam_reduce(const float *partial, const Tiling &t, int chunks, float *sums, cudaStream_t st) {
    const int64_t n_seams = (int64_t)t.C * (t.T - 1);
    const int oo = t.overlap * t.overlap;
    const int64_t total = n_seams * oo;
    if (total <= 0) return cudaSuccess;
    int64_t grid = (total + 255) / 256;
    const int64_t cap = (int64_t)sm_count() * 16;
    if (grid > cap) grid = cap;
    seam_reduce_kernel<<<(int)grid, 256, 0, st>>>(partial, n_seams, oo, chunks, sums);
    return cudaGetLastError();
}

// chunks == 0: `src` is the maps and the discrepancy is computed directly;
// otherwise `src` holds [seam][chunks][o*o] sums.
cudaError_t launch_seam_finalize(const float *src, const Tiling &t, int chunks, double inv_b, float *out,
                                 cudaStream_t st) {
    const int64_t n_seams = (int64_t)t.C * (t.T - 1);
    if (n_seams <= 0) return cudaSuccess;
    if (chunks == 0) {
        const int sms = sm_count();
        if (n_seams >= 4LL * sms) {
            // many seams: a warp each
            int64_t grid = (n_seams * 32 + 255) / 256;
            if (grid > (int64_t)sms * 16) grid = (int64_t)sms * 16;
            seam_direct_warp_kernel<<<(int)grid, 256, 0, st>>>(src, n_seams, t.T, t.B, t.overlap, (float)inv_b,
                                                                out);
        } else {
            // few seams: a CTA each, a thread per overlap entry
            const int oo = t.overlap * t.overlap;
            const int threads = oo >= 256 ? 256 : ((oo + 31) / 32) * 32;
            seam_direct_kernel<<<(int)n_seams, threads, 0, st>>>(src, n_seams, t.T, t.B, t.overlap, (float)inv_b,
                                                                 out);
        }
    } else {
        if (n_seams > 0x7FFFFFFF) return cudaErrorInvalidConfiguration;
        seam_finalize_kernel<<<(unsigned)n_seams, 256, 0, st>>>(src, t.overlap * t.overlap, chunks,
                                                                (float)inv_b, out);
    }
    return cudaGetLastError();
}

}  // namespace tdm
