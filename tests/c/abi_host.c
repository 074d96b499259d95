/* A C99 caller of the library's host-only entry points: sizes, status strings,
 * the segment plan and the slot cache.  No device work, so it runs without a
 * GPU; tests/test_c_abi_host.py compiles it against include/lora_delta.h,
 * links the built library and checks what it prints. */
#include <stdio.h>

#include "lora_delta.h"

int main(void) {
    int32_t mg = 0, mc = 0, rt = 16, mr = 64, slot = -1, resident = -1, slot2 = -1;
    int rc;
    int64_t cols[2] = {28672, 8192};
    uint8_t flags[2] = {0, 0};
    lora_slot_cache *cache;

    printf("version %d\n", lora_version());
    printf("status %s\n", lora_status_string(LORA_ERR_SHAPE));
    if (lora_meta_capacity(1024, 100, 16, 0, LORA_LONG_TILE, &mg, &mc) != LORA_OK) return 1;
    printf("capacity %d %d\n", (int)mg, (int)mc);
    printf("scratch %lu\n", (unsigned long)lora_segments_scratch_bytes(77431, 8));
    if (lora_segment_plan(8192, cols, 2, 148, LORA_LONG_TILE, &rt, &mr, flags) != LORA_OK) return 2;
    printf("plan %d %d %d %d\n", (int)rt, (int)mr, (int)flags[0], (int)flags[1]);
    printf("plan_null %d\n", lora_segment_plan(8192, NULL, 2, 148, LORA_LONG_TILE, &rt, &mr, NULL));

    cache = lora_slot_cache_create(2);
    if (!cache) return 3;
    if (lora_slot_cache_acquire(cache, 42, &slot, &resident) != LORA_OK) return 4;
    printf("acquire %d %d %lld\n", (int)slot, (int)resident, (long long)lora_slot_cache_key(cache, slot));
    if (lora_slot_cache_acquire(cache, 42, &slot2, &resident) != LORA_OK) return 5;
    printf("again %d %d\n", (int)slot2, (int)resident);
    printf("evict_pinned %d\n", lora_slot_cache_evict(cache, 42));
    lora_slot_cache_release(cache, slot);
    lora_slot_cache_release(cache, slot2);
    rc = lora_slot_cache_evict(cache, 42);   /* before the key is read */
    printf("evict %d %lld\n", rc, (long long)lora_slot_cache_key(cache, slot));
    lora_slot_cache_destroy(cache);
    return 0;
}
