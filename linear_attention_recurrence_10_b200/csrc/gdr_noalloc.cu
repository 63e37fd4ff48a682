// gdr_noalloc.cu -- gdr_prefill_chunked_noalloc: the chunked prefill for
// callers that cannot hand the library a workspace.
//
// Some callers have no way to allocate device memory on the path where they
// run the prefill: a runtime that gives all free device memory to its own
// pools when it starts, or a plain C caller that embeds this library without
// any memory manager.  For them the workspace comes from a fixed array in the
// library's own device memory instead.  The array is a file-scope __device__
// object, so every GPU that loads the library holds it until the process exits.
//
// In host code `g_prefill_scratch` names a host-side stand-in, not a device
// address.  Its device address is looked up once per device, with that device
// current, through cudaGetSymbolAddress; the prefill kernels only ever see
// that address.  The lookup is cached per device index for the life of the
// process: it belongs to the device's primary context, so callers that reset
// the device (cudaDeviceReset) or run in a context of their own are not
// served by this entry point.
#include <mutex>

#include "gdr.h"
#include "gdr_common.cuh"

namespace {

constexpr size_t kScratchBytes = gdr::prefill_tc_ws_bytes(GDR_PREFILL_NOALLOC_MAX_SEQS);

static __device__ __align__(256) unsigned char g_prefill_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_lock;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device, resolved on the
// first call made with that device current.  nullptr if the lookup fails.
void *scratch_on_current_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> guard(g_lock);
    if (!g_scratch_addr[dev]) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_prefill_scratch) != cudaSuccess) {
            (void)cudaGetLastError();
            return nullptr;
        }
        g_scratch_addr[dev] = ptr;
    }
    return g_scratch_addr[dev];
}

// The calls that run on the tensor cores write the scratch status word; the
// others (CUDA-core shapes, no sequences) leave it alone.
bool writes_status_word(const gdr_prefill_args *a) {
    return a->n_seq > 0 && a->in_dtype == GDR_BF16 && a->d_k == 128 &&
           (a->chunk == 0 || a->chunk == 64);
}

}  // namespace

extern "C" gdr_status gdr_prefill_chunked_noalloc(const gdr_prefill_args *args,
                                                   gdr_stream_t stream) {
    if (!args) return GDR_ERR_INVALID_ARG;
    if (args->n_seq > GDR_PREFILL_NOALLOC_MAX_SEQS) return GDR_ERR_WORKSPACE;
    void *scratch = scratch_on_current_device();
    if (!scratch) return GDR_ERR_CUDA;
    // Everything the kernels read from the scratch is written first by the same
    // call (the status word is cleared and the sequence order rebuilt), so the
    // previous call's contents never leak into this one.
    const gdr_status st = gdr_prefill_chunked(args, scratch, kScratchBytes, stream);
    if (st != GDR_OK || writes_status_word(args)) return st;
    // A call that does not write the status word still leaves it reading 0.
    if (cudaMemsetAsync(scratch, 0, sizeof(int32_t), (cudaStream_t)stream) != cudaSuccess) {
        (void)cudaGetLastError();
        return GDR_ERR_CUDA;
    }
    return GDR_OK;
}

extern "C" gdr_status gdr_prefill_noalloc_status(int32_t *status, gdr_stream_t stream) {
    if (!status) return GDR_ERR_INVALID_ARG;
    void *scratch = scratch_on_current_device();
    if (!scratch) return GDR_ERR_CUDA;
    if (cudaMemcpyAsync(status, scratch, sizeof(int32_t), cudaMemcpyDefault,
                        (cudaStream_t)stream) != cudaSuccess) {
        (void)cudaGetLastError();
        return GDR_ERR_CUDA;
    }
    return GDR_OK;
}
