/*
 * tdm.h -- C ABI of the tiled distance-map sampler library (libtdm.so), sm_100a.
 *
 * The library implements the data-parallel hot path of a ParaChromo-style tiled
 * 3D-genome diffusion sampler (ParaChromo paper, mdpi.com/2079-9292/15/13/2750):
 * batched DDIM reverse updates on 64-bead distance maps with classifier-free
 * guidance, the overlap-consistency projection of the 12-bead seam between
 * adjacent tiles (§4.3.2, Algorithm 1), coordinate recovery by classical MDS
 * (the distance-geometry initialisation of §3.1), pairwise-distance
 * reconstruction and the seam discrepancy of §5.5 Eq. (6).  The trained U-Net
 * is replaced by a stand-in noise predictor: the ideal denoiser toward a known
 * x0 plus counter-based Philox noise.  Beside that path: SMACOF coordinate
 * refinement (§3.1), Kabsch stitching of tiles into chains with the per-seam
 * residual (§4.3.2, §5.5 Fig. 4), the non-overlap drift of the
 * synchronisation-frequency sweep (§5.7 Table 8), resumable parts of a run, the
 * cosine schedule of the caller-table path, the noise primitives and a
 * NaN/inf scan.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every function returns a tdm_status; TDM_OK is 0.  Argument errors are
 *    found before any launch and return TDM_EINVAL / TDM_EUNSUPPORTED without
 *    touching device memory.  tdm_ctx_last_error() gives a one-line detail.
 *  - Compute entry points are asynchronous on the caller's stream (a
 *    cudaStream_t passed as tdm_stream; NULL is the legacy default stream).
 *    Launch failures are reported as TDM_ECUDA.
 *  - Every pointer named "device" is device memory owned by the caller; it must
 *    be 16-byte aligned and hold contiguous row-major float32 data.  The library
 *    never frees caller memory and allocates only inside tdm_ctx_create and
 *    tdm_init_schedule; the compute entry points allocate nothing and make no
 *    synchronous copy.
 *  - Beads per tile n is 64.  A map is 64 x 64 float32 (16 KiB).
 *  - Tiled maps are laid out [C][T][B][64][64]: chain c, tile k, sample b.
 *    Reference maps x0 are [C][T][64][64], shared by the B samples of a tile
 *    (§3.3: samples of one condition differ only through their noise).
 *  - The noise id of map (c, k, b) is
 *        g = sample_id_base + (c*T + k) * B_total + b_offset + b
 *    so a run split into sample shards or chunks reproduces the unsplit run.
 */
#ifndef TDM_H
#define TDM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t tdm_status;
#define TDM_OK             0
#define TDM_EINVAL         1  /* bad argument (null, misaligned, out of range) */
#define TDM_ECUDA          2  /* a CUDA runtime call or launch failed */
#define TDM_ETIMEOUT       3  /* reserved: no kernel of this library waits on another */
#define TDM_ENONFINITE     4  /* tdm_scan_nonfinite found NaN or inf (see tdm_ctx_sync) */
#define TDM_EUNSUPPORTED   5  /* valid request this build does not implement */
#define TDM_ENOMEM         6  /* device allocation failed */
#define TDM_ENOTCONVERGED  7  /* an MDS eigen-solve hit its iteration cap (see tdm_ctx_sync) */

/* noise streams of the stand-in and the sampler (Philox counter word 3, top byte) */
#define TDM_STREAM_INIT   0  /* initial state x_T */
#define TDM_STREAM_EPS_C  1  /* conditional eps stream */
#define TDM_STREAM_EPS_U  2  /* unconditional eps stream */
#define TDM_STREAM_ETA    3  /* sigma_i z of DDIM with eta > 0 */

/* device status flags returned by tdm_ctx_sync */
#define TDM_FLAG_MDS_NOT_CONVERGED 0x1u
#define TDM_FLAG_NONFINITE         0x2u   /* raised by tdm_scan_nonfinite */

/* columns of the host schedule table (tdm_schedule_table), one row per DDIM step i */
#define TDM_SCHED_COLS 8   /* tau_i, ab_t, ab_p, sigma_i, a_i, b_i, sqrt(ab_t), 1/sqrt(1-ab_t) */

typedef void *tdm_stream;              /* a cudaStream_t */
typedef struct tdm_ctx tdm_ctx;        /* opaque: device, status word, scratch */
typedef struct tdm_schedule tdm_schedule;  /* opaque: DDIM coefficient table */

/* Shape of a tiled batch.  C chains of T tiles (T = 1: independent, untiled
 * maps), B samples per tile in this call; adjacent tiles share `overlap` beads
 * (12 in ParaChromo §3.2).  The projection runs after every `sync_every`-th
 * DDIM step counted from the start (0: never).  B_total (0 means B) is the
 * number of samples of the whole run when this call holds the slice
 * [b_offset, b_offset + B) of them; sample_id_base offsets every noise id. */
typedef struct tdm_tiling {
    int32_t C;
    int32_t T;
    int32_t B;
    int32_t overlap;
    int32_t sync_every;
    int32_t reserved;     /* must be 0 */
    int64_t B_total;
    int64_t b_offset;
    int64_t sample_id_base;
} tdm_tiling;

/* ---- context ---------------------------------------------------------- */

/* Creates a context on CUDA device `device` (allocates its status word and
 * scratch).  *out receives the handle.  Errors: TDM_EINVAL (out NULL or bad
 * device), TDM_ENOMEM, TDM_ECUDA.  The calls that keep intermediate results
 * in the scratch (tdm_seam_discrepancy, tdm_seam_overlap_sums,
 * tdm_nonoverlap_drift) must not overlap on the GPU for one context: issue
 * them on one stream, or give each stream its own context.  Host threads may share
 * a context, but the message of tdm_ctx_last_error is the context's last one,
 * whichever thread failed: a thread that reads messages should have its own
 * context. */
tdm_status tdm_ctx_create(tdm_ctx **out, int32_t device);

/* Frees everything the context owns.  NULL is ignored. */
void tdm_ctx_destroy(tdm_ctx *ctx);

/* Static message for a status code (never NULL). */
const char *tdm_status_str(tdm_status s);

/* Detail of the last error seen on this context ("" if none). */
const char *tdm_ctx_last_error(const tdm_ctx *ctx);

/* Synchronises `stream`, then reads and clears the context's device status
 * word.  *flags_out (may be NULL) receives the TDM_FLAG_* bits raised since the
 * last call.  Returns TDM_ENONFINITE when TDM_FLAG_NONFINITE was set, else
 * TDM_ENOTCONVERGED when TDM_FLAG_MDS_NOT_CONVERGED was set. */
tdm_status tdm_ctx_sync(tdm_ctx *ctx, tdm_stream stream, uint32_t *flags_out);

/* Scans buf[0 .. n) (device floats, 4-byte aligned, read only) on `stream`
 * and raises TDM_FLAG_NONFINITE in the context's status word when any value
 * is NaN or +-inf; the result is read by tdm_ctx_sync.  Meant for a caller's
 * check of any output (the library's kernels never produce non-finite values
 * from finite inputs).  Errors: TDM_EINVAL (NULL ctx, n < 0, NULL or
 * misaligned buf with n > 0). */
tdm_status tdm_scan_nonfinite(tdm_ctx *ctx, const float *buf, int64_t n, tdm_stream stream);

/* Diagnostics: the device's float32 FMA rate, measured by two launches of a
 * kernel in which every thread of 8 CTAs x 256 threads per SM runs 8
 * independent fmaf chains, the second launch timed with CUDA events on
 * `stream`.  *fma_per_s receives fused multiply-adds per second, one per
 * lane and instruction: the measured denominator of the ALU rooflines (in
 * theory one per CUDA-core lane per clock).  The kernel writes nothing
 * (its guarded store into the context's scratch never fires).  Synchronises
 * `stream`.  Errors: TDM_EINVAL (NULL ctx or output), TDM_ECUDA. */
tdm_status tdm_fma_rate(tdm_ctx *ctx, double *fma_per_s, tdm_stream stream);

/* The cosine alphas-bar table of Nichol & Dhariwal, "Improved Denoising
 * Diffusion Probabilistic Models" (2021, section 3.2), for passing to
 * tdm_init_schedule as alphas_bar_opt: alphas_bar(t) = f(t) / f(0),
 * f(t) = cos^2(((t / T_train) + s) / (1 + s) * pi / 2), each beta clipped at
 * 0.999; entry k is timestep k + 1.  ParaChromo §4.3.2 names a cosine schedule
 * without its constants; s = 0.008 is the published offset.  Host function:
 * alphas_bar_out is a host array [T_train].  Errors: TDM_EINVAL (T_train < 1,
 * s < 0 or not finite, NULL output). */
tdm_status tdm_cosine_alphas_bar(int32_t T_train, double s, double *alphas_bar_out);

/* ---- schedule (ParaChromo §4.1, §5.1.1: reduced-step DDIM) --------------
 * Builds, in float64 on the host, beta_t linear from beta_start to beta_end
 * over T_train steps (or takes alphas_bar_opt[T_train] as given), the DDIM
 * timesteps tau_i = i * T_train / S (i = 0..S-1; alphas_bar before tau_0 is 1)
 * and for every step the coefficients of
 *     x_{tau_{i-1}} = a_i x_{tau_i} + b_i eps + sigma_i z,
 *     sigma_i = eta sqrt((1-ab_p)/(1-ab_t)) sqrt(1-ab_t/ab_p)
 * (Song et al., the pages' ref. [7]); uploads a float32 copy.  The schedule
 * belongs to ctx's device.  Errors: TDM_EINVAL (S < 1, T_train % S != 0,
 * eta < 0, betas outside (0,1), alphas_bar_opt not decreasing in (0,1)). */
tdm_status tdm_init_schedule(tdm_ctx *ctx, tdm_schedule **out, int32_t T_train, double beta_start,
                             double beta_end, const double *alphas_bar_opt, int32_t S, double eta);

void tdm_schedule_destroy(tdm_schedule *sched);

/* Copies the host float64 table, S rows of TDM_SCHED_COLS, into out (host,
 * n_doubles >= S * TDM_SCHED_COLS). */
tdm_status tdm_schedule_table(const tdm_schedule *sched, double *out, int64_t n_doubles);

/* Number of DDIM steps S of the schedule (0 for NULL). */
int32_t tdm_schedule_steps(const tdm_schedule *sched);

/* ---- sampler ----------------------------------------------------------- */

/* Writes the initial state x_T of every map of `tiling` into maps (device,
 * [C][T][B][64][64]): a symmetric N(0,1) field from the INIT stream (Philox
 * step word 0).  Entry (i, j), i <= j, is a Box-Muller normal of row quad
 * (i, j/4); entry (i, j), i > j, repeats entry (j, i). */
tdm_status tdm_init_noise(tdm_ctx *ctx, float *maps, const tdm_tiling *tiling, uint64_t seed,
                          tdm_stream stream);

/* The stand-in noise prediction of one stream at DDIM step `step`
 * (0 <= step < S):
 *     eps_out = (maps - sqrt(ab_t) x0) / sqrt(1 - ab_t) + s * z
 * with z the symmetric normal field of stream `stream_tag` (TDM_STREAM_EPS_C
 * or TDM_STREAM_EPS_U) at Philox step word `step`.  maps, eps_out: device
 * [C][T][B][64][64] (must not overlap); x0: device [C][T][64][64]. */
tdm_status tdm_eps_standin(tdm_ctx *ctx, const tdm_schedule *sched, int32_t step, const float *maps,
                           const float *x0, float s, int32_t stream_tag, uint64_t seed,
                           const tdm_tiling *tiling, float *eps_out, tdm_stream stream);

/* One DDIM reverse step `step` (the loop runs step = S-1 .. 0), in place on
 * maps (device [C][T][B][64][64]):
 *     eps  = (1 + w) eps_c - w eps_u          (classifier-free guidance, ref. [15])
 *     maps = a_i maps + b_i eps + sigma_i z   (z: ETA stream, only when eta > 0)
 * then, when T > 1, sync_every > 0 and (S - step) % sync_every == 0, the
 * overlap projection of tdm_seam_project.  eps_u may be NULL iff w == 0.
 * Every map entry is updated (no symmetry is assumed). */
tdm_status tdm_ddim_step(tdm_ctx *ctx, const tdm_schedule *sched, int32_t step, float *maps,
                         const float *eps_c, const float *eps_u, float w, uint64_t seed,
                         const tdm_tiling *tiling, tdm_stream stream);

/* The whole reverse run in one launch: for step = S-1 .. 0, the stand-in eps
 * of both streams (s_c, s_u; the EPS_U stream is not drawn when w == 0), the
 * guidance combination, the DDIM update and the projection every sync_every
 * steps.  The state is the folded map -- its upper triangle i <= j, which holds
 * every bead pair once -- kept in registers for all S steps; on return maps
 * holds the full symmetric map.  init_noise != 0: x_T is drawn as in
 * tdm_init_noise; otherwise x_T is read from maps (its upper triangle only).
 * x0: device [C][T][64][64].  The overlap must be a multiple of 4 (the state
 * is held in 4-column quads); other overlaps return TDM_EUNSUPPORTED (use
 * tdm_ddim_step).  Results equal the step-by-step path on symmetric input up
 * to float32 rounding. */
tdm_status tdm_ddim_run(tdm_ctx *ctx, const tdm_schedule *sched, float *maps, const float *x0, float w,
                        float s_c, float s_u, uint64_t seed, int32_t init_noise,
                        const tdm_tiling *tiling, tdm_stream stream);

/* Part of the same run: steps first_step, first_step - 1, .., first_step -
 * n_steps + 1 (0 <= first_step < S, 1 <= n_steps <= first_step + 1), with the
 * state read from maps (or x_T drawn when init_noise != 0, allowed only for
 * first_step = S-1) and written back.  The noise is keyed by the step index
 * and the projection follows the steps counted from step S-1, so a run split
 * into parts (the state kept in maps in between, e.g. saved and restored as a
 * checkpoint) follows the whole run: its states equal the whole run's up to
 * the float32 rounding of the state written at each cut, and its final maps
 * (after step 0, which sets them from x0 and that step's own noise) are the
 * same bit for bit.  Errors as tdm_ddim_run, plus TDM_EINVAL for a step range
 * outside the schedule. */
tdm_status tdm_ddim_run_steps(tdm_ctx *ctx, const tdm_schedule *sched, float *maps, const float *x0, float w,
                              float s_c, float s_u, uint64_t seed, int32_t init_noise, int32_t first_step,
                              int32_t n_steps, const tdm_tiling *tiling, tdm_stream stream);

/* Which folded-state quad each lane of the fused run holds (host only; a
 * diagnostic for callers that inspect the launch, and the map that the kernel
 * derives in-kernel from the warp and lane index, with no table in memory).
 * out[w * 32 + l] (host, n >= 544 T entries) receives, for lane l of warp w of
 * a chain-sample's 17 T warps, q | r << 4 | k << 10 | paired << 31: row quad
 * (r, 4q .. 4q+3) of tile k.  A paired lane (l < 16) holds a quad of the
 * overlap block of tile k that the projection averages with the quad of tile
 * k+1 in lane l + 16 of the same warp.  overlap: a multiple of 4 in [4, 32]
 * when T > 1 (ignored when T = 1).  Errors: TDM_EINVAL. */
tdm_status tdm_fused_lane_map(int32_t T, int32_t overlap, uint32_t *out, int64_t n);

/* Overlap-consistency projection, in place (ParaChromo §4.3.2, Algorithm 1):
 * for every chain c, seam k < T-1 and sample b, M = 0.5 * (right block of tile
 * k + left block of tile k+1), the blocks being rows/cols [64-o, 64) and
 * [0, o); M is written to both.  Idempotent.  1 <= overlap <= 32. */
tdm_status tdm_seam_project(tdm_ctx *ctx, float *maps, const tdm_tiling *tiling, tdm_stream stream);

/* ---- coordinate refinement ----------------------------------------------
 * SMACOF stress majorisation of coordinates against their maps (ParaChromo
 * §3.1: distance-geometry initialisation "followed by coordinate refinement";
 * the method is not on the pages -- read as minimising the raw stress
 * sum_{i<j} (|x_i - x_j| - D_ij)^2).  maps: device [n][64][64] (symmetrised
 * as (D + D^T)/2); coords: device [n][64][3], the start (e.g.
 * tdm_mds_recover's output) on entry, the result on return.  Each of the
 * `iterations` steps is the Guttman transform x_i <- (1/64) sum_{j != i}
 * (D_ij / d_ij) (x_i - x_j) (terms with d_ij = 0 left out), which never
 * increases the stress.  stress_out (device [n], may be NULL) receives the
 * final stress. */
tdm_status tdm_refine_smacof(tdm_ctx *ctx, const float *maps, int64_t n_maps, float *coords, int32_t iterations,
                             float *stress_out, tdm_stream stream);

/* ---- stitching ------------------------------------------------------------
 * Kabsch stitching of per-tile coordinates into chains (ParaChromo §4.3.2 last
 * paragraph; §5.5, Fig. 4).  coords: device [C][T][B][64][3] (tile k, sample b
 * of chain c; e.g. tdm_mds_recover's output of a tiled batch).  For every seam,
 * tile k+1 is mapped onto tile k by x -> R x + t with R the orthogonal polar
 * factor of the cross-covariance of the o shared beads (an improper R is
 * allowed: recovered coordinates are defined up to reflection), t matching the
 * centroids; the maps compose along the chain so every tile lands in tile 0's
 * frame.  chain_out: device [C][B][L][3], L = 64 + (T-1)(64-o); an overlap
 * bead is the mean of its two aligned copies.  residual_out: device
 * [C][B][T-1] (may be NULL), the RMSD over the o beads of each seam after the
 * alignment, in the coordinates' units.  Needs overlap >= 3 when T > 1.
 * One pass over the coordinates for chains of any length; no scratch. */
tdm_status tdm_kabsch_stitch(tdm_ctx *ctx, const float *coords, const tdm_tiling *tiling, float *chain_out,
                             float *residual_out, tdm_stream stream);

/* ---- noise primitives ----------------------------------------------------
 * The two stages of every noise stream, on caller data, so that a caller can
 * reproduce any noise value and check the transform's error exhaustively. */

/* out[i] = Philox4x32-10(ctr[i], key = (seed mod 2^32, seed div 2^32)) (Salmon
 * et al., SC'11); ctr, out: device uint32 [n][4], 16-byte aligned. */
tdm_status tdm_philox4x32(tdm_ctx *ctx, const uint32_t *ctr, int64_t n, uint64_t seed, uint32_t *out,
                          tdm_stream stream);

/* The uniform-to-normal transform of every stream: for word pair (a, b) =
 * words[2i], words[2i+1], u1 = 1 - (a>>9) 2^-23, u2 = (b>>9) 2^-23,
 * z[2i] = sqrt(-2 ln u1) cos(2 pi u2), z[2i+1] = sqrt(-2 ln u1) sin(2 pi u2),
 * evaluated with float32 hardware approximations.  words: device uint32
 * [n_pairs][2]; z: device float32 [n_pairs][2]; both 8-byte aligned. */
tdm_status tdm_box_muller(tdm_ctx *ctx, const uint32_t *words, int64_t n_pairs, float *z, tdm_stream stream);

/* ---- recovery ------------------------------------------------------------ */

/* Classical MDS of n_maps maps (device [n][64][64]) into coords (device
 * [n][64][3]) and, if eigvals_opt is not NULL, the top-3 eigenvalues (device
 * [n][3], descending): D <- (D + D^T)/2, B = -1/2 J (D*D) J, top-3 eigenpairs
 * (l_k, v_k) of B by subspace iteration with Rayleigh-Ritz, x_k = v_k
 * sqrt(max(l_k, 0)).  Coordinates are defined up to rotation and reflection.
 * A map whose eigen-solve does not reach its tolerance within the iteration
 * cap keeps its last iterate and raises TDM_FLAG_MDS_NOT_CONVERGED. */
tdm_status tdm_mds_recover(tdm_ctx *ctx, const float *maps, int64_t n_maps, float *coords,
                           float *eigvals_opt, tdm_stream stream);

/* tdm_mds_recover and tdm_pairwise_dist of its coordinates in one pass: the
 * same coordinates, eigenvalues and flags, and dist_out (device
 * [n_maps][64][64], caller-owned, 16-byte aligned) equal to what
 * tdm_pairwise_dist writes for them, bit for bit, without reading the
 * coordinates back from memory. */
tdm_status tdm_mds_reconstruct(tdm_ctx *ctx, const float *maps, int64_t n_maps, float *coords, float *eigvals_opt,
                               float *dist_out, tdm_stream stream);

/* maps_out[m][i][j] = || coords[m][i] - coords[m][j] ||_2 (device; zero diagonal). */
tdm_status tdm_pairwise_dist(tdm_ctx *ctx, const float *coords, int64_t n_maps, float *maps_out,
                             tdm_stream stream);

/* Seam discrepancy, ParaChromo §5.5 Eq. (6): out[c][k] (device [C][T-1]) =
 * mean over the o x o overlap of | mean_b right block of tile k - mean_b left
 * block of tile k+1 |.  Uses context scratch for per-chunk partial sums. */
tdm_status tdm_seam_discrepancy(tdm_ctx *ctx, const float *maps, const tdm_tiling *tiling, float *out,
                                tdm_stream stream);

/* The sharded form of Eq. (6): sums (device [C][T-1][o][o]) = sum over this
 * call's B samples of (right block of tile k - left block of tile k+1).
 * Sums of several shards add up (e.g. an all-reduce across ranks); then
 * tdm_seam_discrepancy_finalize divides by tiling->B_total. */
tdm_status tdm_seam_overlap_sums(tdm_ctx *ctx, const float *maps, const tdm_tiling *tiling, float *sums,
                                 tdm_stream stream);

tdm_status tdm_seam_discrepancy_finalize(tdm_ctx *ctx, const float *sums, const tdm_tiling *tiling,
                                         float *out, tdm_stream stream);

/* ---- non-overlap drift (ParaChromo §5.7, Table 8) ---------------------------
 * How far the synchronised maps moved, outside the overlap blocks, from an
 * independent run of the same seeds.  maps (synchronised) and ref
 * (independent): device [C][T][B][64][64], read only, may alias.  The overlap
 * blocks of tile k are its upper-left o x o block when k > 0 and its
 * lower-right o x o block when k < T-1; all other entries count.
 * tile_sums_out: device [C][T][2] = (sum |maps - ref|, sum |ref|) over the
 * tile's B samples and counted entries.  drift_out (device [C], may be NULL):
 * per chain, sum over its tiles of the first sum / sum of the second (NaN
 * when both are 0, +inf when only the second is).  Sums of several shards of
 * the samples add up.  tiling->sync_every is not used.  When there are few
 * tiles, partial sums over chunks of samples go through context scratch. */
tdm_status tdm_nonoverlap_drift(tdm_ctx *ctx, const float *maps, const float *ref, const tdm_tiling *tiling,
                                float *tile_sums_out, float *drift_out, tdm_stream stream);

/* ---- the same without allocation -------------------------------------------
 * No counterpart in the paper: this entry point exists for callers that cannot
 * call cudaMalloc -- an application whose device memory is all handed to its
 * own pool or arena, a plugin host that forbids allocations outside its own
 * allocator, or a pipeline that cannot afford the synchronisation that
 * cudaMalloc/cudaFree may imply.  It needs no tdm_ctx (creating one allocates).
 *
 * Computes the seam discrepancy of Eq. (6) as tdm_seam_discrepancy does (out:
 * device [C][T-1]; maps: device [C][T][B][64][64]; both caller-owned, 16-byte
 * aligned), on the caller's current CUDA device and stream, and calls no
 * cudaMalloc, cudaFree or allocating routine.  The result agrees with
 * tdm_seam_discrepancy up to the float32 order of the sums.  When the samples
 * of a seam are split into chunks, the partial sums live in one fixed device
 * array of TDM_NOALLOC_SCRATCH_FLOATS floats (1 MiB) compiled into the
 * library: every GPU that loads the library holds it until the process exits.
 * Requests whose partial sums would not fit it (seams x chunks x overlap^2;
 * only overlaps above 16 with few seams) take the one-pass form that needs no
 * partial sums.
 *
 * Set-up and memory: CUDA loads a library's device code lazily by default, so
 * the first call on each device loads this entry point's kernels and, with
 * them, the 1 MiB array (about 1 MiB plus code).  Make that first call before
 * handing the device's memory to a pool, or it may fail with TDM_ECUDA; later
 * calls take no device memory.  Each call outside stream capture looks up the
 * array's device address (cudaGetSymbolAddress) on the current device, so a
 * device reset or another current context is followed.  A call under stream
 * capture uses the address that the last uncaptured call on that device found,
 * and returns TDM_EUNSUPPORTED when there was none: make the first call, and
 * one after any cudaDeviceReset, outside capture.
 *
 * All calls on a device share that array and it keeps the last call's partial
 * sums; each call writes every partial sum it reads before reading it, so no
 * clearing is needed, but calls that overlap on the GPU (on different streams,
 * or from different host threads without ordering) race on it and must be
 * serialised by the caller.
 *
 * Errors: TDM_EINVAL (NULL or misaligned pointers, T < 2, B < 1, overlap
 * outside [1, 32], bad shard fields), TDM_EUNSUPPORTED for a first use under
 * stream capture (above), TDM_ECUDA on a failed launch or symbol lookup.
 * There is no context to hold an error message. */
#define TDM_NOALLOC_SCRATCH_FLOATS 262144
tdm_status tdm_seam_discrepancy_noalloc(const float *maps, const tdm_tiling *tiling, float *out,
                                        tdm_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* TDM_H */
