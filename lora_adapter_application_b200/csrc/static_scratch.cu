// lora_build_segments_static: the batch grouping without caller-provided
// scratch memory.
//
// Some callers cannot allocate device memory at the point where they group a
// batch: code running inside a memory pool that owns every byte of the
// device, host callbacks and plugin hooks that must not call cudaMalloc (it
// can synchronise the device or fail under a pool's quota), and runtimes that
// only hand out the input and output buffers.  This entry point takes the
// same ids and lora_meta arrays as lora_build_segments, but its scratch lives
// in one fixed array of LORA_STATIC_SCRATCH_BYTES bytes compiled into the
// library, so nothing is allocated by the call.
//
// How the array is used:
//   * Every device that loads the library holds its own copy until the
//     process exits.
//   * Host code cannot take the array's address directly (the host symbol is
//     only a stand-in).  The first call on each device, with that device
//     current, asks the runtime for the device address once
//     (cudaGetSymbolAddress) and remembers it; make that first call before
//     any stream capture.
//   * All calls share the array and it keeps whatever the last call left.
//     The grouping overwrites every scratch word it later reads, so nothing
//     has to be cleared between calls.  Calls that overlap on the GPU (on
//     different streams, or from several threads without ordering) race on
//     the array and corrupt each other's result: order them on one stream.
#include "kernels.cuh"

#include <mutex>

namespace {

constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char lora_static_scratch[LORA_STATIC_SCRATCH_BYTES];

std::mutex g_mutex;
void *g_addr[kMaxDevices] = {};

// Device address of the array on the current device (looked up once).
int static_scratch_address(void **out) {
    int dev = 0;
    const cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return lora::cuda_rc(e);
    if (dev < 0 || dev >= kMaxDevices) return lora::cuda_fail("device index beyond the static scratch table");
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_addr[dev] == nullptr) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, lora_static_scratch);
        if (e != cudaSuccess) return lora::cuda_rc(e);
        if (p == nullptr) return lora::cuda_fail("cudaGetSymbolAddress returned no address");
        g_addr[dev] = p;
    }
    *out = g_addr[dev];
    return LORA_OK;
}

}  // namespace

extern "C" {

int lora_build_segments_static(const int32_t *ids, const lora_meta *meta, int32_t *status,
                               void *stream) {
    if (!meta || !status) return LORA_ERR_NULL;
    if (meta->T < 0 || meta->N < 1) return LORA_ERR_SHAPE;
    const size_t need = lora_segments_scratch_bytes(meta->T, meta->N);
    if (need > (size_t)LORA_STATIC_SCRATCH_BYTES) return LORA_ERR_WORKSPACE;
    void *scratch = nullptr;
    if (need > 0) {
        const int rc = static_scratch_address(&scratch);
        if (rc != LORA_OK) return rc;
    }
    return lora_build_segments(ids, meta, scratch, need, status, stream);
}

}  // extern "C"
