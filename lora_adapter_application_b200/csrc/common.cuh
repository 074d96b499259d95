// Shared device helpers and launch parameter blocks of the multi-LoRA delta
// kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "lora_delta.h"

namespace lora {

constexpr unsigned FULL = 0xffffffffu;

// ----------------------------------------------------------- element access
__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

__device__ __forceinline__ float load_elem(const float *p) { return *p; }
__device__ __forceinline__ float load_elem(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
__device__ __forceinline__ void store_elem(float *p, float v) { *p = v; }
__device__ __forceinline__ void store_elem(__nv_bfloat16 *p, float v) { *p = __float2bfloat16_rn(v); }

// Two fp32 values packed as bf16x2 (low half = first), round-to-nearest-even.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

// ----------------------------------------------------------- launch blocks
struct Slices {
    const void *A[LORA_MAX_SLICES];
    const void *B[LORA_MAX_SLICES];
    int32_t d_out[LORA_MAX_SLICES];
    int32_t col_off[LORA_MAX_SLICES];
    int32_t cat_off[LORA_MAX_SLICES + 1];   // offsets of the slices in the concatenated column space
    int32_t n;
};

// Which rows a unit of work covers: a gathered tile, or a slice of rows_per_tile
// rows of a contiguous tile.
struct Tiles {
    const int32_t *counts;        // [4]
    const int32_t *grow;
    const int4 *gather;           // {id, q0, cnt, 0}
    const int4 *contig;           // {id, row0, cnt, 0}
    int32_t max_gather;           // units [0, max_gather) are gathered tiles
    int32_t max_contig;           // then max_contig * subs units of contiguous tiles
    int32_t subs;                 // units per contiguous tile (0 = skip contiguous tiles)
    int32_t rows_per_unit;        // rows of one unit (rows_per_tile)
    int32_t use_gather;           // 0 = skip gathered tiles
};

// Resolve unit u: returns the row count (0 = nothing to do), adapter id and
// fills rows[0..cnt) through `row_of(q)`.
struct Unit {
    int32_t id;
    int32_t cnt;
    int32_t base;     // gathered: first index into grow; contiguous: first row
    bool gathered;
    __device__ __forceinline__ int32_t row(const Tiles &t, int q) const {
        return gathered ? t.grow[base + q] : base + q;
    }
};

__device__ __forceinline__ Unit resolve_unit(const Tiles &t, int u) {
    Unit r{0, 0, 0, true};
    if (u < t.max_gather) {
        if (!t.use_gather || u >= t.counts[1]) return r;
        int4 g = t.gather[u];
        r.id = g.x; r.base = g.y; r.cnt = g.z; r.gathered = true;
        return r;
    }
    if (t.subs == 0) return r;
    u -= t.max_gather;
    int tile = u / t.subs, sub = u - tile * t.subs;
    if (tile >= t.counts[2]) return r;
    int4 c = t.contig[tile];
    int first = sub * t.rows_per_unit;
    if (first >= c.z) return r;
    r.id = c.x; r.base = c.y + first; r.cnt = min(t.rows_per_unit, c.z - first); r.gathered = false;
    return r;
}

// Units that exist in this batch, numbered without gaps: the gathered tiles
// first, then rows_per_unit-row slices of the contiguous tiles (a slice past
// its tile's end resolves to cnt = 0).  Read from the device-side counts, so a
// persistent grid walks only real work.
__device__ __forceinline__ int n_live_units(const Tiles &t) {
    const int ng = t.use_gather ? min(t.counts[1], t.max_gather) : 0;
    const int nc = t.subs ? min(t.counts[2], t.max_contig) : 0;
    return ng + nc * t.subs;
}

__device__ __forceinline__ Unit resolve_live_unit(const Tiles &t, int v) {
    Unit r{0, 0, 0, true};
    const int ng = t.use_gather ? min(t.counts[1], t.max_gather) : 0;
    if (v < ng) {
        const int4 g = t.gather[v];
        r.id = g.x; r.base = g.y; r.cnt = g.z; r.gathered = true;
        return r;
    }
    v -= ng;
    const int tile = v / t.subs, sub = v - tile * t.subs;
    const int4 c = t.contig[tile];
    const int first = sub * t.rows_per_unit;
    if (first >= c.z) return r;
    r.id = c.x; r.base = c.y + first; r.cnt = min(t.rows_per_unit, c.z - first); r.gathered = false;
    return r;
}

}  // namespace lora
