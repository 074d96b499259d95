// Adapter slots: loading one adapter into a slot of the stacked tensors, and
// the host policy that picks the slot (page "LoRA hot load and adapter
// routing", adapter lifecycle: load -> check the rank -> copy to the GPU ->
// evict the least recently used adapter when the GPU slots are full; page
// "Multi-LoRA Serving", section 3.2: max_loras adapters resident on the GPU).
//
// lora_load_adapter moves the adapter with the copy engines on the caller's
// stream (one 1-D copy per A slice, one pitched copy per B slice, pitched
// zero-fills for the rank padding) and writes the slot's rank and alpha with
// a one-thread kernel, so the whole load is stream-ordered, needs no host
// synchronisation and can be captured into a CUDA graph (for device sources).
//
// lora_slot_cache is a plain host structure: adapter key -> slot, a use clock
// per slot, and a pin count per slot (a slot that a batch in flight reads
// cannot be chosen as a victim).
#include "kernels.cuh"

#include <cstdint>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

namespace lora {
namespace {

__global__ void slot_meta_kernel(int32_t *ranks, float *alphas, int n, int r, float alpha) {
    ranks[n] = r;
    alphas[n] = alpha;
}

}  // namespace
}  // namespace lora

struct lora_slot_cache {
    std::mutex mu;
    int32_t n_slots = 0;
    uint64_t clock = 0;
    std::vector<int64_t> key;     // adapter held by each slot (-1: free)
    std::vector<uint64_t> used;   // clock of the last acquire
    std::vector<int32_t> pins;    // batches in flight that read the slot
};

extern "C" {

int lora_load_adapter(const lora_slice *slices, int32_t n_slices, int32_t d_in, int32_t r_max,
                      int32_t N, int32_t n, int32_t r, const void *const *src_A,
                      const void *const *src_B, float alpha, int32_t *ranks, float *alphas,
                      lora_dtype dtype, void *stream) {
    if (!slices || !src_A || !src_B || !ranks || !alphas) return LORA_ERR_NULL;
    if (dtype != LORA_BF16 && dtype != LORA_FP32) return LORA_ERR_DTYPE;
    if (n_slices < 1 || n_slices > LORA_MAX_SLICES || d_in < 1 || N < 1 || N > LORA_MAX_ADAPTERS ||
        n < 0 || n >= N)
        return LORA_ERR_SHAPE;
    if (r_max < 1 || r_max > LORA_MAX_RANK || r < 1 || r > r_max) return LORA_ERR_RANK;
    const size_t e = dtype == LORA_BF16 ? 2 : 4;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    for (int s = 0; s < n_slices; ++s) {
        const lora_slice &sl = slices[s];
        if (!sl.A || !sl.B || !src_A[s] || !src_B[s]) return LORA_ERR_NULL;
        if (sl.d_out < 1) return LORA_ERR_SHAPE;
    }
    cudaError_t err = cudaSuccess;
    for (int s = 0; s < n_slices && err == cudaSuccess; ++s) {
        const lora_slice &sl = slices[s];
        // A_s[n]: r rows of d_in, then r_max - r rows of zeros
        unsigned char *a = (unsigned char *)sl.A + (size_t)n * r_max * d_in * e;
        err = cudaMemcpyAsync(a, src_A[s], (size_t)r * d_in * e, cudaMemcpyDefault, st);
        if (err == cudaSuccess && r < r_max)
            err = cudaMemsetAsync(a + (size_t)r * d_in * e, 0, (size_t)(r_max - r) * d_in * e, st);
        // B_s[n]: d_out rows of r_max; the first r columns from the source, the rest zero
        unsigned char *b = (unsigned char *)sl.B + (size_t)n * sl.d_out * r_max * e;
        if (err == cudaSuccess)
            err = cudaMemcpy2DAsync(b, (size_t)r_max * e, src_B[s], (size_t)r * e, (size_t)r * e,
                                    (size_t)sl.d_out, cudaMemcpyDefault, st);
        if (err == cudaSuccess && r < r_max)
            err = cudaMemset2DAsync(b + (size_t)r * e, (size_t)r_max * e, 0, (size_t)(r_max - r) * e,
                                    (size_t)sl.d_out, st);
    }
    if (err != cudaSuccess) return lora::cuda_rc(err);
    lora::slot_meta_kernel<<<1, 1, 0, st>>>(ranks, alphas, n, r, alpha);
    return lora::cuda_rc(cudaGetLastError());
}

lora_slot_cache *lora_slot_cache_create(int32_t n_slots) {
    if (n_slots < 1 || n_slots > LORA_MAX_ADAPTERS) return nullptr;
    lora_slot_cache *c = new (std::nothrow) lora_slot_cache;
    if (!c) return nullptr;
    c->n_slots = n_slots;
    c->key.assign(n_slots, -1);
    c->used.assign(n_slots, 0);
    c->pins.assign(n_slots, 0);
    return c;
}

void lora_slot_cache_destroy(lora_slot_cache *c) { delete c; }

int lora_slot_cache_acquire(lora_slot_cache *c, int64_t key, int32_t *slot, int32_t *resident) {
    if (!c || !slot || !resident) return LORA_ERR_NULL;
    if (key < 0) return LORA_ERR_SHAPE;
    std::lock_guard<std::mutex> lock(c->mu);
    ++c->clock;
    int victim = -1;
    for (int i = 0; i < c->n_slots; ++i) {
        if (c->key[i] == key) {   // a hit: the adapter is already in slot i
            c->used[i] = c->clock;
            ++c->pins[i];
            *slot = i;
            *resident = 1;
            return LORA_OK;
        }
    }
    // a miss: the lowest free slot, else the least recently used slot nobody pins
    for (int i = 0; i < c->n_slots && victim < 0; ++i)
        if (c->key[i] < 0) victim = i;
    if (victim < 0)
        for (int i = 0; i < c->n_slots; ++i)
            if (c->pins[i] == 0 && (victim < 0 || c->used[i] < c->used[victim])) victim = i;
    if (victim < 0) return LORA_ERR_CAPACITY;   // every slot is pinned by a batch in flight
    c->key[victim] = key;
    c->used[victim] = c->clock;
    c->pins[victim] = 1;
    *slot = victim;
    *resident = 0;
    return LORA_OK;
}

int lora_slot_cache_release(lora_slot_cache *c, int32_t slot) {
    if (!c) return LORA_ERR_NULL;
    std::lock_guard<std::mutex> lock(c->mu);
    if (slot < 0 || slot >= c->n_slots || c->pins[slot] <= 0) return LORA_ERR_SHAPE;
    --c->pins[slot];
    return LORA_OK;
}

int64_t lora_slot_cache_key(lora_slot_cache *c, int32_t slot) {
    if (!c) return -1;
    std::lock_guard<std::mutex> lock(c->mu);
    if (slot < 0 || slot >= c->n_slots) return -1;
    return c->key[slot];
}

int lora_slot_cache_evict(lora_slot_cache *c, int64_t key) {
    if (!c) return LORA_ERR_NULL;
    std::lock_guard<std::mutex> lock(c->mu);
    for (int i = 0; i < c->n_slots; ++i)
        if (c->key[i] == key) {
            if (c->pins[i] > 0) return LORA_ERR_CAPACITY;
            c->key[i] = -1;
            c->used[i] = 0;
            return LORA_OK;
        }
    return LORA_ERR_SHAPE;
}

}  // extern "C"
