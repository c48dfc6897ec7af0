// extern "C" entry points of libtdm: argument validation, context, schedule,
// and dispatch to the kernel launchers.  See include/tdm.h for the contract.
#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <new>

#include <nvtx3/nvToolsExt.h>

#include "internal.h"

using tdm::StepCoef;
using tdm::Tiling;

namespace {

tdm_status fail(tdm_ctx *ctx, tdm_status s, const char *fmt, ...) {
    if (ctx != nullptr) {
        char buf[512];
        va_list ap;
        va_start(ap, fmt);
        vsnprintf(buf, sizeof(buf), fmt, ap);
        va_end(ap);
        ctx->last_error = buf;
    }
    return s;
}

tdm_status cuda_fail(tdm_ctx *ctx, cudaError_t e, const char *where) {
    return fail(ctx, TDM_ECUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Makes ctx's device current for the scope of an entry point.
struct DeviceScope {
    int prev = -1;
    cudaError_t err = cudaSuccess;
    explicit DeviceScope(int dev) {
        err = cudaGetDevice(&prev);
        if (err == cudaSuccess && prev != dev) err = cudaSetDevice(dev);
    }
    ~DeviceScope() {
        int cur = -1;
        if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
    }
};

tdm_status check_tiling(tdm_ctx *ctx, const tdm_tiling *in, Tiling *t) {
    if (in == nullptr) return fail(ctx, TDM_EINVAL, "tiling is NULL");
    if (in->C < 0 || in->T < 1 || in->B < 0)
        return fail(ctx, TDM_EINVAL, "tiling: need C >= 0, T >= 1, B >= 0 (got %d, %d, %d)", in->C, in->T, in->B);
    if (in->reserved != 0) return fail(ctx, TDM_EINVAL, "tiling: reserved field must be 0");
    if (in->T > 1 && (in->overlap < 1 || in->overlap > 32))
        return fail(ctx, TDM_EINVAL, "tiling: overlap must be in [1, 32] (got %d)", in->overlap);
    if (in->T == 1 && (in->overlap < 0 || in->overlap > 32))
        return fail(ctx, TDM_EINVAL, "tiling: overlap must be in [0, 32] (got %d)", in->overlap);
    if (in->T > 0xFFFF) return fail(ctx, TDM_EUNSUPPORTED, "tiling: at most 65535 tiles per chain");
    if (in->sync_every < 0) return fail(ctx, TDM_EINVAL, "tiling: sync_every must be >= 0");
    const int64_t B_total = in->B_total == 0 ? in->B : in->B_total;
    if (in->b_offset < 0 || in->sample_id_base < 0 || B_total < in->b_offset + in->B)
        return fail(ctx, TDM_EINVAL, "tiling: need 0 <= b_offset, b_offset + B <= B_total, sample_id_base >= 0");
    // every noise id must fit the 56 bits of the Philox counter
    const long double max_id = (long double)in->sample_id_base +
                               ((long double)in->C * in->T) * (long double)B_total;
    if (max_id > (long double)(1ULL << 56))
        return fail(ctx, TDM_EUNSUPPORTED, "tiling: noise ids exceed 2^56");
    t->C = in->C;
    t->T = in->T;
    t->B = in->B;
    t->overlap = in->overlap;
    t->sync_every = in->sync_every;
    t->B_total = B_total;
    t->b_offset = in->b_offset;
    t->sample_id_base = in->sample_id_base;
    return TDM_OK;
}

tdm_status check_maps(tdm_ctx *ctx, const void *p, const char *name) {
    if (p == nullptr) return fail(ctx, TDM_EINVAL, "%s is NULL", name);
    if (!aligned16(p)) return fail(ctx, TDM_EINVAL, "%s is not 16-byte aligned", name);
    return TDM_OK;
}

tdm_status check_sched(tdm_ctx *ctx, const tdm_schedule *s) {
    if (s == nullptr || s->d_coef == nullptr) return fail(ctx, TDM_EINVAL, "schedule is NULL");
    if (s->device != ctx->device) return fail(ctx, TDM_EINVAL, "schedule belongs to another device");
    return TDM_OK;
}

}  // namespace


// An NVTX range around each entry point (a no-op unless a profiler is attached).
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};

extern "C" {

const char *tdm_status_str(tdm_status s) {
    switch (s) {
        case TDM_OK: return "ok";
        case TDM_EINVAL: return "invalid argument";
        case TDM_ECUDA: return "CUDA error";
        case TDM_ETIMEOUT: return "timed out";
        case TDM_ENONFINITE: return "non-finite value";
        case TDM_EUNSUPPORTED: return "unsupported";
        case TDM_ENOMEM: return "out of device memory";
        case TDM_ENOTCONVERGED: return "eigen-solve did not converge";
        default: return "unknown status";
    }
}

const char *tdm_ctx_last_error(const tdm_ctx *ctx) { return ctx == nullptr ? "" : ctx->last_error.c_str(); }

tdm_status tdm_ctx_create(tdm_ctx **out, int32_t device) {
    NvtxRange nvtx_range_("tdm_ctx_create");
    if (out == nullptr) return TDM_EINVAL;
    *out = nullptr;
    int count = 0;
    if (cudaGetDeviceCount(&count) != cudaSuccess || device < 0 || device >= count) return TDM_EINVAL;
    tdm_ctx *ctx = new (std::nothrow) tdm_ctx();
    if (ctx == nullptr) return TDM_ENOMEM;
    ctx->device = device;
    DeviceScope ds(device);
    if (ds.err != cudaSuccess) {
        delete ctx;
        return TDM_ECUDA;
    }
    // scratch: per-chunk partial sums of the seam discrepancy (<= 1184 seam
    // chunks of up to 32 x 32 entries)
    ctx->scratch_floats = (size_t)1184 * 1024;
    if (cudaMalloc(&ctx->d_flags, sizeof(uint32_t)) != cudaSuccess ||
        cudaMalloc(&ctx->d_scratch, ctx->scratch_floats * sizeof(float)) != cudaSuccess ||
        cudaMemset(ctx->d_flags, 0, sizeof(uint32_t)) != cudaSuccess) {
        cudaFree(ctx->d_flags);
        cudaFree(ctx->d_scratch);
        delete ctx;
        cudaGetLastError();
        return TDM_ENOMEM;
    }
    *out = ctx;
    return TDM_OK;
}

void tdm_ctx_destroy(tdm_ctx *ctx) {
    if (ctx == nullptr) return;
    {
        DeviceScope ds(ctx->device);
        cudaFree(ctx->d_flags);
        cudaFree(ctx->d_scratch);
    }
    delete ctx;
}

tdm_status tdm_ctx_sync(tdm_ctx *ctx, tdm_stream stream, uint32_t *flags_out) {
    NvtxRange nvtx_range_("tdm_ctx_sync");
    if (ctx == nullptr) return TDM_EINVAL;
    DeviceScope ds(ctx->device);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(ctx, e, "stream synchronize");
    uint32_t flags = 0;
    e = cudaMemcpy(&flags, ctx->d_flags, sizeof(flags), cudaMemcpyDeviceToHost);
    if (e == cudaSuccess) e = cudaMemset(ctx->d_flags, 0, sizeof(uint32_t));
    if (e != cudaSuccess) return cuda_fail(ctx, e, "status word");
    if (flags_out != nullptr) *flags_out = flags;
    if (flags & TDM_FLAG_NONFINITE) return fail(ctx, TDM_ENONFINITE, "a scanned buffer held NaN or inf");
    if (flags & TDM_FLAG_MDS_NOT_CONVERGED)
        return fail(ctx, TDM_ENOTCONVERGED, "an MDS eigen-solve reached its iteration cap");
    return TDM_OK;
}

tdm_status tdm_scan_nonfinite(tdm_ctx *ctx, const float *buf, int64_t n, tdm_stream stream) {
    NvtxRange nvtx_range_("tdm_scan_nonfinite");
    if (ctx == nullptr) return TDM_EINVAL;
    if (n < 0) return fail(ctx, TDM_EINVAL, "scan: n < 0");
    if (n == 0) return TDM_OK;
    if (buf == nullptr || (reinterpret_cast<uintptr_t>(buf) & 3u))
        return fail(ctx, TDM_EINVAL, "scan: buf is NULL or not 4-byte aligned");
    DeviceScope ds(ctx->device);
    cudaError_t e = tdm::launch_scan_nonfinite(buf, n, ctx->d_flags, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TDM_OK : cuda_fail(ctx, e, "scan launch");
}

tdm_status tdm_fma_rate(tdm_ctx *ctx, double *fma_per_s, tdm_stream stream) {
    NvtxRange nvtx_range_("tdm_fma_rate");
    if (ctx == nullptr) return TDM_EINVAL;
    if (fma_per_s == nullptr) return fail(ctx, TDM_EINVAL, "fma_rate: output is NULL");
    DeviceScope ds(ctx->device);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaEvent_t ev[2] = {nullptr, nullptr};
    cudaError_t e = cudaEventCreate(&ev[0]);
    if (e == cudaSuccess) e = cudaEventCreate(&ev[1]);
    double fmas = 0.0;
    // one short launch to reach full clocks, then the timed one
    if (e == cudaSuccess) e = tdm::launch_fma_rate(ctx->d_scratch, (int64_t)ctx->scratch_floats, 256, st, &fmas);
    if (e == cudaSuccess) e = cudaEventRecord(ev[0], st);
    if (e == cudaSuccess) e = tdm::launch_fma_rate(ctx->d_scratch, (int64_t)ctx->scratch_floats, 4096, st, &fmas);
    if (e == cudaSuccess) e = cudaEventRecord(ev[1], st);
    if (e == cudaSuccess) e = cudaEventSynchronize(ev[1]);
    float ms = 0.0f;
    if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, ev[0], ev[1]);
    if (ev[0] != nullptr) cudaEventDestroy(ev[0]);
    if (ev[1] != nullptr) cudaEventDestroy(ev[1]);
    if (e != cudaSuccess) return cuda_fail(ctx, e, "fma_rate");
    if (!(ms > 0.0f)) return fail(ctx, TDM_ECUDA, "fma_rate: no elapsed time");
    *fma_per_s = fmas / ((double)ms * 1e-3);
    return TDM_OK;
}

// ---- schedule -----------------------------------------------------------------------

tdm_status tdm_cosine_alphas_bar(int32_t T_train, double s, double *alphas_bar_out) {
    if (T_train < 1 || !(s >= 0.0) || !std::isfinite(s) || alphas_bar_out == nullptr) return TDM_EINVAL;
    constexpr double kHalfPi = 1.5707963267948966;
    constexpr double kMaxBeta = 0.999;
    auto f = [&](double t) {
        const double c = std::cos((t / (double)T_train + s) / (1.0 + s) * kHalfPi);
        return c * c;
    };
    double acc = 1.0, f_prev = f(0.0);
    for (int k = 0; k < T_train; ++k) {
        const double f_next = f((double)k + 1.0);
        const double beta = std::min(1.0 - f_next / f_prev, kMaxBeta);
        acc *= 1.0 - beta;
        alphas_bar_out[k] = acc;
        f_prev = f_next;
    }
    return TDM_OK;
}

tdm_status tdm_init_schedule(tdm_ctx *ctx, tdm_schedule **out, int32_t T_train, double beta_start,
                             double beta_end, const double *alphas_bar_opt, int32_t S, double eta) {
    NvtxRange nvtx_range_("tdm_init_schedule");
    if (ctx == nullptr || out == nullptr) return fail(ctx, TDM_EINVAL, "ctx or out is NULL");
    *out = nullptr;
    if (T_train < 1 || S < 1 || S > T_train || T_train % S != 0)
        return fail(ctx, TDM_EINVAL, "schedule: need 1 <= S, S divides T_train (got T=%d, S=%d)", T_train, S);
    if (!(eta >= 0.0) || !std::isfinite(eta)) return fail(ctx, TDM_EINVAL, "schedule: eta must be >= 0");
    std::vector<double> ab((size_t)T_train);
    if (alphas_bar_opt == nullptr) {
        if (!(beta_start > 0.0 && beta_start < 1.0 && beta_end > 0.0 && beta_end < 1.0))
            return fail(ctx, TDM_EINVAL, "schedule: betas must lie in (0, 1)");
        double acc = 1.0;
        for (int t = 0; t < T_train; ++t) {
            const double b = T_train > 1 ? beta_start + (beta_end - beta_start) * (double)t / (double)(T_train - 1)
                                         : beta_start;
            acc *= (1.0 - b);
            ab[(size_t)t] = acc;
        }
    } else {
        double prev = 1.0;
        for (int t = 0; t < T_train; ++t) {
            const double v = alphas_bar_opt[t];
            if (!(v > 0.0 && v < prev)) return fail(ctx, TDM_EINVAL, "schedule: alphas_bar must decrease in (0, 1)");
            ab[(size_t)t] = prev = v;
        }
    }
    tdm_schedule *s = new (std::nothrow) tdm_schedule();
    if (s == nullptr) return fail(ctx, TDM_ENOMEM, "schedule: host allocation");
    s->device = ctx->device;
    s->T_train = T_train;
    s->S = S;
    s->eta = eta;
    s->table.assign((size_t)S * TDM_SCHED_COLS, 0.0);
    std::vector<StepCoef> coef((size_t)S);
    const int stride = T_train / S;
    for (int i = 0; i < S; ++i) {
        const int tau = i * stride;
        const double ab_t = ab[(size_t)tau];
        const double ab_p = i > 0 ? ab[(size_t)(tau - stride)] : 1.0;
        const double sigma = eta * std::sqrt((1.0 - ab_p) / (1.0 - ab_t)) * std::sqrt(1.0 - ab_t / ab_p);
        const double a = std::sqrt(ab_p) / std::sqrt(ab_t);
        const double dir = 1.0 - ab_p - sigma * sigma;
        const double b = std::sqrt(dir > 0.0 ? dir : 0.0) - std::sqrt(ab_p) * std::sqrt(1.0 - ab_t) / std::sqrt(ab_t);
        const double sa = std::sqrt(ab_t), isa1 = 1.0 / std::sqrt(1.0 - ab_t);
        double *row = &s->table[(size_t)i * TDM_SCHED_COLS];
        row[0] = tau;
        row[1] = ab_t;
        row[2] = ab_p;
        row[3] = sigma;
        row[4] = a;
        row[5] = b;
        row[6] = sa;
        row[7] = isa1;
        StepCoef &c = coef[(size_t)i];
        c.ka = (float)(a + b * isa1);
        c.kx0 = (float)(-b * isa1 * sa);
        c.kb = (float)b;
        c.ks = (float)sigma;
        c.a = (float)a;
        c.sa = (float)sa;
        c.isa1 = (float)isa1;
        c.pad = 0.0f;
    }
    DeviceScope ds(ctx->device);
    cudaError_t e = cudaMalloc(&s->d_coef, sizeof(StepCoef) * (size_t)S);
    if (e == cudaSuccess) e = cudaMemcpy(s->d_coef, coef.data(), sizeof(StepCoef) * (size_t)S, cudaMemcpyHostToDevice);
    if (e != cudaSuccess) {
        cudaFree(s->d_coef);
        delete s;
        return cuda_fail(ctx, e, "schedule upload");
    }
    *out = s;
    return TDM_OK;
}

void tdm_schedule_destroy(tdm_schedule *s) {
    if (s == nullptr) return;
    {
        DeviceScope ds(s->device);
        cudaFree(s->d_coef);
    }
    delete s;
}

tdm_status tdm_schedule_table(const tdm_schedule *s, double *out, int64_t n) {
    NvtxRange nvtx_range_("tdm_schedule_table");
    if (s == nullptr || out == nullptr || n < (int64_t)s->table.size()) return TDM_EINVAL;
    std::memcpy(out, s->table.data(), s->table.size() * sizeof(double));
    return TDM_OK;
}

int32_t tdm_schedule_steps(const tdm_schedule *s) { return s == nullptr ? 0 : s->S; }

// ---- sampler ------------------------------------------------------------------------

tdm_status tdm_init_noise(tdm_ctx *ctx, float *maps, const tdm_tiling *tiling, uint64_t seed, tdm_stream stream) {
    NvtxRange nvtx_range_("tdm_init_noise");
    if (ctx == nullptr) return TDM_EINVAL;
    Tiling t;
    tdm_status s = check_tiling(ctx, tiling, &t);
    if (s != TDM_OK) return s;
    if (t.n_maps() == 0) return TDM_OK;
    if ((s = check_maps(ctx, maps, "maps")) != TDM_OK) return s;
    DeviceScope ds(ctx->device);
    cudaError_t e = tdm::launch_init_noise(maps, t, seed, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TDM_OK : cuda_fail(ctx, e, "init_noise launch");
}

tdm_status tdm_eps_standin(tdm_ctx *ctx, const tdm_schedule *sched, int32_t step, const float *maps,
                           const float *x0, float s_noise, int32_t stream_tag, uint64_t seed,
                           const tdm_tiling *tiling, float *eps_out, tdm_stream stream) {
    NvtxRange nvtx_range_("tdm_eps_standin");
    if (ctx == nullptr) return TDM_EINVAL;
    tdm_status s = check_sched(ctx, sched);
    if (s != TDM_OK) return s;
    Tiling t;
    if ((s = check_tiling(ctx, tiling, &t)) != TDM_OK) return s;
    if (step < 0 || step >= sched->S) return fail(ctx, TDM_EINVAL, "step %d outside [0, %d)", step, sched->S);
    if (stream_tag != TDM_STREAM_EPS_C && stream_tag != TDM_STREAM_EPS_U)
        return fail(ctx, TDM_EINVAL, "stream_tag must be TDM_STREAM_EPS_C or TDM_STREAM_EPS_U");
    if (!std::isfinite(s_noise)) return fail(ctx, TDM_EINVAL, "noise scale is not finite");
    if (t.n_maps() == 0) return TDM_OK;
    if ((s = check_maps(ctx, maps, "maps")) != TDM_OK || (s = check_maps(ctx, x0, "x0")) != TDM_OK ||
        (s = check_maps(ctx, eps_out, "eps_out")) != TDM_OK)
        return s;
    if (eps_out == maps) return fail(ctx, TDM_EINVAL, "eps_out must not alias maps");
    DeviceScope ds(ctx->device);
    cudaError_t e = tdm::launch_eps_standin(sched->d_coef, step, maps, x0, s_noise, stream_tag, seed, t, eps_out,
                                            static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TDM_OK : cuda_fail(ctx, e, "eps_standin launch");
}

tdm_status tdm_seam_project(tdm_ctx *ctx, float *maps, const tdm_tiling *tiling, tdm_stream stream) {
    NvtxRange nvtx_range_("tdm_seam_project");
    if (ctx == nullptr) return TDM_EINVAL;
    Tiling t;
    tdm_status s = check_tiling(ctx, tiling, &t);
    if (s != TDM_OK) return s;
    if (t.n_maps() == 0 || t.T < 2) return TDM_OK;
    if ((s = check_maps(ctx, maps, "maps")) != TDM_OK) return s;
    DeviceScope ds(ctx->device);
    cudaError_t e = tdm::launch_seam_project(maps, t, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TDM_OK : cuda_fail(ctx, e, "seam_project launch");
}

tdm_status tdm_ddim_step(tdm_ctx *ctx, const tdm_schedule *sched, int32_t step, float *maps, const float *eps_c,
                         const float *eps_u, float w, uint64_t seed, const tdm_tiling *tiling, tdm_stream stream) {
    NvtxRange nvtx_range_("tdm_ddim_step");
    if (ctx == nullptr) return TDM_EINVAL;
    tdm_status s = check_sched(ctx, sched);
    if (s != TDM_OK) return s;
    Tiling t;
    if ((s = check_tiling(ctx, tiling, &t)) != TDM_OK) return s;
    if (step < 0 || step >= sched->S) return fail(ctx, TDM_EINVAL, "step %d outside [0, %d)", step, sched->S);
    if (!std::isfinite(w)) return fail(ctx, TDM_EINVAL, "w is not finite");
    if (t.n_maps() == 0) return TDM_OK;    // an empty batch is a no-op, whatever its pointers
    if (w != 0.0f && eps_u == nullptr) return fail(ctx, TDM_EINVAL, "eps_u is NULL but w != 0");
    if ((s = check_maps(ctx, maps, "maps")) != TDM_OK || (s = check_maps(ctx, eps_c, "eps_c")) != TDM_OK)
        return s;
    if (w != 0.0f && (s = check_maps(ctx, eps_u, "eps_u")) != TDM_OK) return s;
    DeviceScope ds(ctx->device);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // the projection, when due after this step, runs inside the step's kernel
    const bool project = t.T > 1 && t.sync_every > 0 && (sched->S - step) % t.sync_every == 0;
    cudaError_t e = tdm::launch_ddim_step(sched->d_coef, step, maps, eps_c, w != 0.0f ? eps_u : nullptr, w,
                                          sched->eta > 0.0, project, seed, t, st);
    return e == cudaSuccess ? TDM_OK : cuda_fail(ctx, e, "ddim_step launch");
}

tdm_status tdm_ddim_run(tdm_ctx *ctx, const tdm_schedule *sched, float *maps, const float *x0, float w, float s_c,
                        float s_u, uint64_t seed, int32_t init_noise, const tdm_tiling *tiling, tdm_stream stream) {
    NvtxRange nvtx_range_("tdm_ddim_run");
    if (ctx == nullptr) return TDM_EINVAL;
    tdm_status s = check_sched(ctx, sched);
    if (s != TDM_OK) return s;
    return tdm_ddim_run_steps(ctx, sched, maps, x0, w, s_c, s_u, seed, init_noise, sched->S - 1, sched->S, tiling,
                              stream);
}

tdm_status tdm_ddim_run_steps(tdm_ctx *ctx, const tdm_schedule *sched, float *maps, const float *x0, float w,
                              float s_c, float s_u, uint64_t seed, int32_t init_noise, int32_t first_step,
                              int32_t n_steps, const tdm_tiling *tiling, tdm_stream stream) {
    NvtxRange nvtx_range_("tdm_ddim_run_steps");
    if (ctx == nullptr) return TDM_EINVAL;
    tdm_status s = check_sched(ctx, sched);
    if (s != TDM_OK) return s;
    if (first_step < 0 || first_step >= sched->S || n_steps < 1 || n_steps > first_step + 1)
        return fail(ctx, TDM_EINVAL, "ddim_run: need 0 <= first_step < S and 1 <= n_steps <= first_step + 1 "
                                     "(got %d, %d, S = %d)", first_step, n_steps, sched->S);
    if (init_noise != 0 && first_step != sched->S - 1)
        return fail(ctx, TDM_EINVAL, "ddim_run: init_noise draws x_T, the state before step S-1 only");
    Tiling t;
    if ((s = check_tiling(ctx, tiling, &t)) != TDM_OK) return s;
    if (!std::isfinite(w) || !std::isfinite(s_c) || !std::isfinite(s_u))
        return fail(ctx, TDM_EINVAL, "w, s_c, s_u must be finite");
    if (t.T > 1 && t.overlap % 4 != 0)
        return fail(ctx, TDM_EUNSUPPORTED, "ddim_run: overlap must be a multiple of 4 (got %d)", t.overlap);
    if (t.n_maps() == 0) return TDM_OK;
    if ((s = check_maps(ctx, maps, "maps")) != TDM_OK || (s = check_maps(ctx, x0, "x0")) != TDM_OK) return s;
    DeviceScope ds(ctx->device);
    cudaError_t e = tdm::launch_ddim_run(sched->d_coef, sched->S, first_step, n_steps, maps, x0, w, s_c, s_u,
                                         sched->eta > 0.0, seed, init_noise != 0, t,
                                         static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TDM_OK : cuda_fail(ctx, e, "ddim_run launch");
}

// ---- refinement ---------------------------------------------------------------------

tdm_status tdm_refine_smacof(tdm_ctx *ctx, const float *maps, int64_t n_maps, float *coords, int32_t iterations,
                             float *stress_out, tdm_stream stream) {
    NvtxRange nvtx_range_("tdm_refine_smacof");
    if (ctx == nullptr) return TDM_EINVAL;
    if (n_maps < 0) return fail(ctx, TDM_EINVAL, "n_maps < 0");
    if (iterations < 0) return fail(ctx, TDM_EINVAL, "iterations < 0");
    if (n_maps == 0) return TDM_OK;
    tdm_status s;
    if ((s = check_maps(ctx, maps, "maps")) != TDM_OK || (s = check_maps(ctx, coords, "coords")) != TDM_OK) return s;
    if (stress_out != nullptr && (reinterpret_cast<uintptr_t>(stress_out) & 3u))
        return fail(ctx, TDM_EINVAL, "stress_out is not 4-byte aligned");
    DeviceScope ds(ctx->device);
    cudaError_t e = tdm::launch_refine(maps, n_maps, coords, iterations, stress_out, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TDM_OK : cuda_fail(ctx, e, "refine launch");
}

// ---- stitching -----------------------------------------------------------------------

tdm_status tdm_kabsch_stitch(tdm_ctx *ctx, const float *coords, const tdm_tiling *tiling, float *chain_out,
                             float *residual_out, tdm_stream stream) {
    NvtxRange nvtx_range_("tdm_kabsch_stitch");
    if (ctx == nullptr) return TDM_EINVAL;
    Tiling t;
    tdm_status s = check_tiling(ctx, tiling, &t);
    if (s != TDM_OK) return s;
    if (t.T > 1 && t.overlap < 3) return fail(ctx, TDM_EINVAL, "stitching needs an overlap of at least 3 beads");
    if (t.n_maps() == 0) return TDM_OK;
    if ((s = check_maps(ctx, coords, "coords")) != TDM_OK || (s = check_maps(ctx, chain_out, "chain_out")) != TDM_OK)
        return s;
    if (residual_out != nullptr && (reinterpret_cast<uintptr_t>(residual_out) & 3u))
        return fail(ctx, TDM_EINVAL, "residual_out is not 4-byte aligned");
    DeviceScope ds(ctx->device);
    cudaError_t e = tdm::launch_stitch(coords, t, chain_out, t.T > 1 ? residual_out : nullptr,
                                       static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TDM_OK : cuda_fail(ctx, e, "stitch launch");
}

// ---- noise primitives ---------------------------------------------------------------

tdm_status tdm_philox4x32(tdm_ctx *ctx, const uint32_t *ctr, int64_t n, uint64_t seed, uint32_t *out,
                          tdm_stream stream) {
    NvtxRange nvtx_range_("tdm_philox4x32");
    if (ctx == nullptr) return TDM_EINVAL;
    if (n < 0) return fail(ctx, TDM_EINVAL, "n < 0");
    if (n == 0) return TDM_OK;
    tdm_status s;
    if ((s = check_maps(ctx, ctr, "ctr")) != TDM_OK || (s = check_maps(ctx, out, "out")) != TDM_OK) return s;
    DeviceScope ds(ctx->device);
    cudaError_t e = tdm::launch_philox(ctr, n, seed, out, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TDM_OK : cuda_fail(ctx, e, "philox launch");
}

tdm_status tdm_box_muller(tdm_ctx *ctx, const uint32_t *words, int64_t n_pairs, float *z, tdm_stream stream) {
    NvtxRange nvtx_range_("tdm_box_muller");
    if (ctx == nullptr) return TDM_EINVAL;
    if (n_pairs < 0) return fail(ctx, TDM_EINVAL, "n_pairs < 0");
    if (n_pairs == 0) return TDM_OK;
    if (words == nullptr || z == nullptr || (reinterpret_cast<uintptr_t>(words) & 7u) ||
        (reinterpret_cast<uintptr_t>(z) & 7u))
        return fail(ctx, TDM_EINVAL, "words and z must be non-NULL and 8-byte aligned");
    DeviceScope ds(ctx->device);
    cudaError_t e = tdm::launch_box_muller(words, n_pairs, z, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TDM_OK : cuda_fail(ctx, e, "box_muller launch");
}

// ---- recovery -----------------------------------------------------------------------

tdm_status tdm_mds_recover(tdm_ctx *ctx, const float *maps, int64_t n_maps, float *coords, float *eigvals_opt,
                           tdm_stream stream) {
    NvtxRange nvtx_range_("tdm_mds_recover");
    if (ctx == nullptr) return TDM_EINVAL;
    if (n_maps < 0) return fail(ctx, TDM_EINVAL, "n_maps < 0");
    if (n_maps == 0) return TDM_OK;
    tdm_status s;
    if ((s = check_maps(ctx, maps, "maps")) != TDM_OK || (s = check_maps(ctx, coords, "coords")) != TDM_OK) return s;
    if (eigvals_opt != nullptr && (reinterpret_cast<uintptr_t>(eigvals_opt) & 3u))
        return fail(ctx, TDM_EINVAL, "eigvals is not 4-byte aligned");
    DeviceScope ds(ctx->device);
    cudaError_t e = tdm::launch_mds(maps, n_maps, coords, eigvals_opt, ctx->d_flags, nullptr,
                                    static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TDM_OK : cuda_fail(ctx, e, "mds launch");
}

tdm_status tdm_mds_reconstruct(tdm_ctx *ctx, const float *maps, int64_t n_maps, float *coords, float *eigvals_opt,
                               float *dist_out, tdm_stream stream) {
    NvtxRange nvtx_range_("tdm_mds_reconstruct");
    if (ctx == nullptr) return TDM_EINVAL;
    if (n_maps < 0) return fail(ctx, TDM_EINVAL, "n_maps < 0");
    if (n_maps == 0) return TDM_OK;
    tdm_status s;
    if ((s = check_maps(ctx, maps, "maps")) != TDM_OK || (s = check_maps(ctx, coords, "coords")) != TDM_OK ||
        (s = check_maps(ctx, dist_out, "dist_out")) != TDM_OK)
        return s;
    if (eigvals_opt != nullptr && (reinterpret_cast<uintptr_t>(eigvals_opt) & 3u))
        return fail(ctx, TDM_EINVAL, "eigvals is not 4-byte aligned");
    DeviceScope ds(ctx->device);
    cudaError_t e = tdm::launch_mds(maps, n_maps, coords, eigvals_opt, ctx->d_flags, dist_out,
                                    static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TDM_OK : cuda_fail(ctx, e, "mds launch");
}

tdm_status tdm_pairwise_dist(tdm_ctx *ctx, const float *coords, int64_t n_maps, float *maps_out, tdm_stream stream) {
    NvtxRange nvtx_range_("tdm_pairwise_dist");
    if (ctx == nullptr) return TDM_EINVAL;
    if (n_maps < 0) return fail(ctx, TDM_EINVAL, "n_maps < 0");
    if (n_maps == 0) return TDM_OK;
    tdm_status s;
    if ((s = check_maps(ctx, coords, "coords")) != TDM_OK || (s = check_maps(ctx, maps_out, "maps_out")) != TDM_OK)
        return s;
    DeviceScope ds(ctx->device);
    cudaError_t e = tdm::launch_pdist(coords, n_maps, maps_out, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TDM_OK : cuda_fail(ctx, e, "pairwise_dist launch");
}

tdm_status tdm_seam_overlap_sums(tdm_ctx *ctx, const float *maps, const tdm_tiling *tiling, float *sums,
                                 tdm_stream stream) {
    NvtxRange nvtx_range_("tdm_seam_overlap_sums");
    if (ctx == nullptr) return TDM_EINVAL;
    Tiling t;
    tdm_status s = check_tiling(ctx, tiling, &t);
    if (s != TDM_OK) return s;
    if (t.T < 2) return fail(ctx, TDM_EINVAL, "seam sums need T >= 2");
    if ((int64_t)t.C * (t.T - 1) == 0) return TDM_OK;
    if ((s = check_maps(ctx, sums, "sums")) != TDM_OK) return s;
    DeviceScope ds(ctx->device);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (t.B == 0) {
        cudaError_t e = cudaMemsetAsync(sums, 0, sizeof(float) * (size_t)t.C * (t.T - 1) * t.overlap * t.overlap, st);
        return e == cudaSuccess ? TDM_OK : cuda_fail(ctx, e, "seam sums clear");
    }
    if ((s = check_maps(ctx, maps, "maps")) != TDM_OK) return s;
    const int64_t n_seams = (int64_t)t.C * (t.T - 1);
    const int oo = t.overlap * t.overlap;
    int chunks = tdm::seam_chunks(n_seams, t.B);
    cudaError_t e;
    if (chunks > 1 && (size_t)n_seams * chunks * oo <= ctx->scratch_floats) {
        e = tdm::launch_seam_sums(maps, t, ctx->d_scratch, chunks, st);
        if (e == cudaSuccess) e = tdm::launch_seam_reduce(ctx->d_scratch, t, chunks, sums, st);
    } else {
        e = tdm::launch_seam_sums(maps, t, sums, 1, st);
    }
    return e == cudaSuccess ? TDM_OK : cuda_fail(ctx, e, "seam sums launch");
}

tdm_status tdm_seam_discrepancy_finalize(tdm_ctx *ctx, const float *sums, const tdm_tiling *tiling, float *out,
                                         tdm_stream stream) {
    NvtxRange nvtx_range_("tdm_seam_discrepancy_finalize");
    if (ctx == nullptr) return TDM_EINVAL;
    Tiling t;
    tdm_status s = check_tiling(ctx, tiling, &t);
    if (s != TDM_OK) return s;
    if (t.T < 2) return fail(ctx, TDM_EINVAL, "seam discrepancy needs T >= 2");
    if (t.B_total < 1) return fail(ctx, TDM_EINVAL, "seam discrepancy needs B_total >= 1");
    if ((int64_t)t.C * (t.T - 1) == 0) return TDM_OK;
    if ((s = check_maps(ctx, sums, "sums")) != TDM_OK || (s = check_maps(ctx, out, "out")) != TDM_OK) return s;
    DeviceScope ds(ctx->device);
    cudaError_t e = tdm::launch_seam_finalize(sums, t, 1, 1.0 / (double)t.B_total, out,
                                              static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TDM_OK : cuda_fail(ctx, e, "seam finalize launch");
}

tdm_status tdm_seam_discrepancy(tdm_ctx *ctx, const float *maps, const tdm_tiling *tiling, float *out,
                                tdm_stream stream) {
    NvtxRange nvtx_range_("tdm_seam_discrepancy");
    if (ctx == nullptr) return TDM_EINVAL;
    Tiling t;
    tdm_status s = check_tiling(ctx, tiling, &t);
    if (s != TDM_OK) return s;
    if (t.T < 2) return fail(ctx, TDM_EINVAL, "seam discrepancy needs T >= 2");
    if (t.B < 1) return fail(ctx, TDM_EINVAL, "seam discrepancy needs B >= 1");
    if ((int64_t)t.C * (t.T - 1) == 0) return TDM_OK;
    if ((s = check_maps(ctx, maps, "maps")) != TDM_OK || (s = check_maps(ctx, out, "out")) != TDM_OK) return s;
    DeviceScope ds(ctx->device);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int64_t n_seams = (int64_t)t.C * (t.T - 1);
    const int oo = t.overlap * t.overlap;
    const int chunks = tdm::seam_chunks(n_seams, t.B);
    const double inv_b = 1.0 / (double)t.B;
    cudaError_t e;
    if (chunks > 1 && (size_t)n_seams * chunks * oo <= ctx->scratch_floats) {
        e = tdm::launch_seam_sums(maps, t, ctx->d_scratch, chunks, st);
        if (e == cudaSuccess) e = tdm::launch_seam_finalize(ctx->d_scratch, t, chunks, inv_b, out, st);
    } else {
        e = tdm::launch_seam_finalize(maps, t, 0, inv_b, out, st);
    }
    return e == cudaSuccess ? TDM_OK : cuda_fail(ctx, e, "seam discrepancy launch");
}

tdm_status tdm_nonoverlap_drift(tdm_ctx *ctx, const float *maps, const float *ref, const tdm_tiling *tiling,
                                float *tile_sums_out, float *drift_out, tdm_stream stream) {
    NvtxRange nvtx_range_("tdm_nonoverlap_drift");
    if (ctx == nullptr) return TDM_EINVAL;
    Tiling t;
    tdm_status s = check_tiling(ctx, tiling, &t);
    if (s != TDM_OK) return s;
    if (t.n_maps() == 0) return TDM_OK;
    if ((s = check_maps(ctx, maps, "maps")) != TDM_OK || (s = check_maps(ctx, ref, "ref")) != TDM_OK ||
        (s = check_maps(ctx, tile_sums_out, "tile_sums_out")) != TDM_OK)
        return s;
    if (drift_out != nullptr && (reinterpret_cast<uintptr_t>(drift_out) & 3u))
        return fail(ctx, TDM_EINVAL, "drift_out is not 4-byte aligned");
    DeviceScope ds(ctx->device);
    const int64_t tiles = (int64_t)t.C * t.T;
    int chunks = tdm::drift_chunks(tiles, t.B);
    if (chunks > 1 && (size_t)tiles * chunks * 2 > ctx->scratch_floats) chunks = 1;
    cudaError_t e = tdm::launch_drift(maps, ref, t, ctx->d_scratch, chunks, tile_sums_out, drift_out,
                                      static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TDM_OK : cuda_fail(ctx, e, "drift launch");
}

}  // extern "C"
