// Internal declarations of libtdm: context, schedule and kernel launchers.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>
#include <map>
#include <mutex>
#include <string>
#include <utility>
#include <vector>

#include "tdm.h"

namespace tdm {

constexpr int kN = 64;                 // beads per tile
constexpr int kQuadsPerRow = kN / 4;   // 16 column quads per row
constexpr int kUpperQuads = 544;       // row quads (r, q) with 4q + 3 >= r
constexpr int kMapFloats = kN * kN;

// Per DDIM step, float32 coefficients (computed in float64 on the host):
//   fused form   x_p = ka x_t + kx0 x0 + kb (noise part of eps) + ks z
//   step form    x_p = a  x_t + kb eps + ks z
//   stand-in     eps = (x_t - sa x0) * isa1 + s z
struct StepCoef {
    float ka, kx0, kb, ks, a, sa, isa1, pad;
};

// Shape of one call, resolved from tdm_tiling.
struct Tiling {
    int C, T, B, overlap, sync_every;
    int64_t B_total, b_offset, sample_id_base;
    __host__ __device__ int64_t n_maps() const { return (int64_t)C * T * B; }
};

}  // namespace tdm

struct tdm_schedule {
    int device = 0;
    int T_train = 0;
    int S = 0;
    double eta = 0.0;
    std::vector<double> table;           // S x TDM_SCHED_COLS
    tdm::StepCoef *d_coef = nullptr;     // device [S]
};

struct tdm_ctx {
    int device = 0;
    std::string last_error;
    uint32_t *d_flags = nullptr;         // device status word (TDM_FLAG_*)
    float *d_scratch = nullptr;          // partial sums of the seam discrepancy
    size_t scratch_floats = 0;
};

namespace tdm {

// kernel launchers (one .cu file each); every launcher returns cudaGetLastError()
cudaError_t launch_init_noise(float *maps, const Tiling &t, uint64_t seed, cudaStream_t st);
cudaError_t launch_eps_standin(const StepCoef *coef, int step, const float *maps, const float *x0, float s,
                               int tag, uint64_t seed, const Tiling &t, float *eps, cudaStream_t st);
cudaError_t launch_ddim_step(const StepCoef *coef, int step, float *maps, const float *eps_c,
                             const float *eps_u, float w, bool has_eta, bool project, uint64_t seed,
                             const Tiling &t, cudaStream_t st);
cudaError_t launch_ddim_run(const StepCoef *coef, int S, int first, int n_steps, float *maps, const float *x0,
                            float w, float s_c, float s_u, bool has_eta, uint64_t seed, bool init_noise,
                            const Tiling &t, cudaStream_t st);
cudaError_t launch_seam_project(float *maps, const Tiling &t, cudaStream_t st);
cudaError_t launch_seam_sums(const float *maps, const Tiling &t, float *partial, int chunks,
                             cudaStream_t st);
cudaError_t launch_seam_reduce(const float *partial, const Tiling &t, int chunks, float *sums,
                               cudaStream_t st);
cudaError_t launch_seam_finalize(const float *sums, const Tiling &t, int chunks, double inv_b,
                                 float *out, cudaStream_t st);
cudaError_t launch_mds(const float *maps, int64_t n, float *coords, float *eigvals, uint32_t *flags, float *dist,
                       cudaStream_t st);
cudaError_t launch_pdist(const float *coords, int64_t n, float *maps, cudaStream_t st);
cudaError_t launch_refine(const float *maps, int64_t n, float *coords, int iterations, float *stress,
                          cudaStream_t st);
cudaError_t launch_stitch(const float *coords, const Tiling &t, float *chain, float *resid, cudaStream_t st);
cudaError_t launch_philox(const uint32_t *ctr, int64_t n, uint64_t seed, uint32_t *out, cudaStream_t st);
cudaError_t launch_box_muller(const uint32_t *words, int64_t n_pairs, float *z, cudaStream_t st);

// host helpers
int seam_chunks(int64_t n_seams, int B);
int drift_chunks(int64_t tiles, int B);
cudaError_t launch_scan_nonfinite(const float *buf, int64_t n, uint32_t *flags, cudaStream_t st);
cudaError_t launch_fma_rate(float *sink, int64_t sink_floats, int iters, cudaStream_t st, double *fmas);
cudaError_t launch_drift(const float *S, const float *V, const Tiling &t, float *scratch, int chunks,
                         float *tile_sums, float *drift, cudaStream_t st);

}  // namespace tdm
