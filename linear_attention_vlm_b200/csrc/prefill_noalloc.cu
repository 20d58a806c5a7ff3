// gdn_prefill_noalloc: the prefill for callers that cannot allocate device
// memory, e.g. a serving loop that reserves all of its device memory at
// start-up and forbids any later cudaMalloc, or a host program that has no
// way to hand the library a workspace pointer.  Instead of a caller-supplied
// workspace it uses one fixed scratch array compiled into libgdn.so.
#include <cuda_runtime.h>

#include <mutex>

#include "gdn.h"
#include "gdn_internal.h"

namespace {

constexpr size_t kScratchBytes = GDN_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

// The scratch.  Every GPU that loads libgdn.so holds these bytes until the
// process exits.  In host code this name is only a host-side stand-in for the
// array: its address is not a device address, so it is never passed to a
// kernel; the device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) uint8_t g_noalloc_scratch[kScratchBytes];

std::mutex g_mu;
void *g_scratch_dev[kMaxDevices] = {};   // device address of the array, per device

// Device address of the scratch on the current device, looked up once per
// device (with that device current) and cached.
int scratch_on_current_device(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return gdn::note_cuda_error(e);
    if (dev < 0 || dev >= kMaxDevices) return GDN_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_dev[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return gdn::note_cuda_error(e);
        g_scratch_dev[dev] = p;
    }
    *out = g_scratch_dev[dev];
    return GDN_OK;
}

}  // namespace

extern "C" int gdn_prefill_noalloc(const void *q, const void *k, const void *v, const float *g,
                                   const float *beta, const float *state_in, void *out,
                                   float *state_out, const int32_t *cu_seqlens, int num_seqs,
                                   int64_t total_tokens, int H, int dk, int dv, int chunk,
                                   int dtype, void *stream) {
    const size_t need = gdn_prefill_workspace_size(num_seqs, total_tokens, H, dk, dv, chunk, dtype);
    if (need > kScratchBytes) return GDN_ERR_WORKSPACE;   // request larger than the fixed scratch
    void *ws = nullptr;
    if (need > 0) {
        const int st = scratch_on_current_device(&ws);
        if (st != GDN_OK) return st;
    }
    // gdn_prefill validates every argument, clears the status word at the
    // start of the scratch and launches the same kernels as with a
    // caller-owned workspace.
    return gdn_prefill(q, k, v, g, beta, state_in, out, state_out, cu_seqlens, num_seqs,
                       total_tokens, H, dk, dv, chunk, dtype, ws, need > 0 ? kScratchBytes : 0,
                       stream);
}

extern "C" int gdn_noalloc_read_status(void *stream, int32_t *code) {
    if (code) *code = 0;
    void *ws = nullptr;
    const int st = scratch_on_current_device(&ws);
    if (st != GDN_OK) return st;
    // the status word is the first int32 of the scratch, as it is the first
    // int32 of a caller-owned workspace for gdn_prefill
    return gdn_read_status(static_cast<const int32_t *>(ws), stream, code);
}
