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
// that address.
#include <mutex>

#include "gdr.h"

namespace {

constexpr size_t kScratchBytes =
    ((16 + 4 * (size_t)GDR_PREFILL_NOALLOC_MAX_SEQS) + 255) & ~(size_t)255;

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
    return gdr_prefill_chunked(args, scratch, kScratchBytes, stream);
}
