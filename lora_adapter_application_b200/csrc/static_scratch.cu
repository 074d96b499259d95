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
//     only a stand-in).  Every call, with its device current, asks the
//     runtime for the device address (cudaGetSymbolAddress) - cheap once the
//     module is loaded; the first call on a device may load it, so make one
//     call per device before any stream capture.  Nothing is cached, so the
//     address is never stale (after a cudaDeviceReset, say).
//   * All calls share the array and it keeps whatever the last call left.
//     The grouping overwrites every scratch word it later reads, so nothing
//     has to be cleared between calls.  Calls that overlap on the GPU (on
//     different streams, or from several threads without ordering) race on
//     the array and corrupt each other's result: order them on one stream.
#include "kernels.cuh"


namespace {

static __device__ __align__(256) unsigned char lora_static_scratch[LORA_STATIC_SCRATCH_BYTES];

// Device address of the array on the current device.
int static_scratch_address(void **out) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, lora_static_scratch);
    if (e != cudaSuccess) return lora::cuda_rc(e);
    if (p == nullptr) return lora::cuda_fail("cudaGetSymbolAddress returned no address");
    *out = p;
    return LORA_OK;
}

}  // namespace

extern "C" {

int lora_build_segments_static(const int32_t *ids, const lora_meta *meta, int32_t *status,
                               void *stream) {
    // the checks of lora_build_segments come first, before any size arithmetic
    const int rc0 = lora::check_meta_args(meta);
    if (rc0 != LORA_OK) return rc0;
    if (!status || (meta->T > 0 && !ids)) return LORA_ERR_NULL;
    const size_t need = lora_segments_scratch_bytes(meta->T, meta->N);
    if (need > (size_t)LORA_STATIC_SCRATCH_BYTES) return LORA_ERR_WORKSPACE;
    void *scratch = nullptr;
    const int rc = static_scratch_address(&scratch);
    if (rc != LORA_OK) return rc;
    return lora_build_segments(ids, meta, need > 0 ? scratch : nullptr, need, status, stream);
}

}  // extern "C"
