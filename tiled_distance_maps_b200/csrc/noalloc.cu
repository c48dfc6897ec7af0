// Seam discrepancy for callers that cannot allocate device memory.
//
// Some callers must not call cudaMalloc at all: an application that has handed
// all of the GPU's memory to its own pool or arena (a fresh cudaMalloc would
// fail, or would be made behind the pool's back), a plugin whose host forbids
// allocations outside the host's allocator, or a pipeline that cannot afford
// the device-wide synchronisation that cudaMalloc/cudaFree may imply.  For them
// tdm_seam_discrepancy_noalloc needs no context (creating one allocates) and
// keeps the partial sums of the chunked reduction in a fixed array below, which
// every GPU that loads this library holds until the process exits.
#include <map>
#include <mutex>

#include "internal.h"

// Partial sums of the chunked Eq. (6) reduction, shared by every call on a
// device.  Its host-side name is only a stand-in: host code passes the device
// address obtained from cudaGetSymbolAddress.
static __device__ __align__(256) float g_noalloc_scratch[TDM_NOALLOC_SCRATCH_FLOATS];

namespace {

std::mutex g_scratch_mu;
std::map<int, float *> g_scratch_addr;    // device index -> address seen by the last uncaptured call

// Device address of g_noalloc_scratch on the current device `dev`.  A call
// outside stream capture looks it up again (cheap once the module is loaded),
// so a device reset or another current context is followed; a call under
// capture takes the address of the last uncaptured call on that device, and
// fails when there was none (the lookup may load the module, which a capture
// must not see).
cudaError_t scratch_address(int dev, cudaStream_t st, float **out) {
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    cudaError_t e = cudaStreamIsCapturing(st, &cap);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (cap == cudaStreamCaptureStatusNone) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev] = static_cast<float *>(p);
    }
    const auto it = g_scratch_addr.find(dev);
    if (it == g_scratch_addr.end()) return cudaErrorStreamCaptureUnsupported;
    *out = it->second;
    return cudaSuccess;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" tdm_status tdm_seam_discrepancy_noalloc(const float *maps, const tdm_tiling *tiling, float *out,
                                                   tdm_stream stream) {
    if (tiling == nullptr || maps == nullptr || out == nullptr || !aligned16(maps) || !aligned16(out))
        return TDM_EINVAL;
    const tdm_tiling &in = *tiling;
    if (in.C < 0 || in.T < 2 || in.B < 1 || in.overlap < 1 || in.overlap > 32 || in.reserved != 0 ||
        in.sync_every < 0 || in.b_offset < 0 || in.sample_id_base < 0)
        return TDM_EINVAL;
    tdm::Tiling t;
    t.C = in.C;
    t.T = in.T;
    t.B = in.B;
    t.overlap = in.overlap;
    t.sync_every = in.sync_every;
    t.B_total = in.B_total == 0 ? in.B : in.B_total;
    t.b_offset = in.b_offset;
    t.sample_id_base = in.sample_id_base;
    if (t.B_total < t.b_offset + t.B) return TDM_EINVAL;
    const int64_t n_seams = (int64_t)t.C * (t.T - 1);
    if (n_seams == 0) return TDM_OK;

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const double inv_b = 1.0 / (double)t.B;
    const int chunks = tdm::seam_chunks(n_seams, t.B);
    const int64_t need = n_seams * chunks * (int64_t)t.overlap * t.overlap;
    cudaError_t e;
    if (chunks <= 1 || need > TDM_NOALLOC_SCRATCH_FLOATS) {
        // one warp (or CTA) per seam over all samples: no partial sums, no
        // scratch; also the form for requests whose partial sums would not
        // fit the fixed array
        e = tdm::launch_seam_finalize(maps, t, 0, inv_b, out, st);
    } else {
        int dev = 0;
        e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return TDM_ECUDA;
        float *scratch = nullptr;
        e = scratch_address(dev, st, &scratch);
        if (e == cudaErrorStreamCaptureUnsupported) return TDM_EUNSUPPORTED;
        if (e != cudaSuccess) return TDM_ECUDA;
        // every partial sum that the finalisation reads is written first by
        // the sums kernel, so nothing has to start at zero
        e = tdm::launch_seam_sums(maps, t, scratch, chunks, st);
        if (e == cudaSuccess) e = tdm::launch_seam_finalize(scratch, t, chunks, inv_b, out, st);
    }
    return e == cudaSuccess ? TDM_OK : TDM_ECUDA;
}
