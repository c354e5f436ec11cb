// no_alloc.cu -- falcon_fwd_chunk for callers that cannot allocate device memory.
//
// Some callers have no way to allocate device memory at the point where they run the
// forward pass: a plugin handed raw device pointers by a host runtime that offers no
// allocator, a serving loop that must not make a cudaMalloc (it can synchronise the
// device and stall other streams), or a process whose device memory is already carved up
// by a pool it does not control. For them this file keeps the chunk pass's scratch in a
// fixed, file-scope device array instead of a caller-provided workspace.
//
// The array is part of the library's device image: every GPU that loads the library
// holds its kFalconStaticScratchBytes until the process exits. Host code never uses the
// array's name as a pointer (on the host it names a stand-in, not device memory): once
// per device, with that device current, the first call resolves the device address with
// cudaGetSymbolAddress and keeps it.
#include <mutex>

#include <cuda_runtime.h>

#include "falcon.h"

namespace {

constexpr size_t kFalconStaticScratchBytes = FALCON_NOALLOC_SCRATCH_BYTES;  // 32 MiB per device
constexpr int kMaxScratchDevices = 64;

static __device__ __align__(256) unsigned char g_chunk_scratch[kFalconStaticScratchBytes];

std::mutex g_scratch_mu;
void *g_scratch_ptr[kMaxScratchDevices] = {};

// Device address of the scratch array on the current device, resolved once per device;
// nullptr when the device cannot be queried or the symbol cannot be resolved.
void *scratch_on_current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxScratchDevices) return nullptr;
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_chunk_scratch) != cudaSuccess || !ptr) return nullptr;
        g_scratch_ptr[dev] = ptr;
    }
    return g_scratch_ptr[dev];
}

}  // namespace

extern "C" {

FALCON_API falcon_status_t falcon_fwd_chunk_noalloc(const falcon_args_t *args, falcon_stream_t stream) {
    // Argument errors are reported by falcon_fwd_chunk itself; a size of 0 means no scratch.
    // falcon_fwd_chunk decides what the array's size allows: a sequence split that needs more
    // is refused before anything runs, and the regression rules' two-pass path runs only when
    // every block's tiles fit (their single-kernel path otherwise).
    const size_t need = falcon_workspace_size(args);
    if (need == 0) return falcon_fwd_chunk(args, nullptr, 0, stream);
    void *ws = scratch_on_current_device();
    if (!ws) return FALCON_ERR_CUDA;
    // Nothing in the scratch has to start at zero: every byte a call reads (the pieces'
    // state increments and decays, the segment start states, the cached keys, the blocks'
    // tiles) is written earlier in the same call, so stale contents of a previous call are
    // never read.
    return falcon_fwd_chunk(args, ws, kFalconStaticScratchBytes, stream);
}

}  // extern "C"
