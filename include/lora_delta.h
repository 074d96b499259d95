/*
 * lora_delta.h - C ABI of the B200 (sm_100a) multi-LoRA delta library.
 *
 * One batched pass applies a different low-rank adapter to every row of a
 * batch:
 *
 *     y_i[off_s + c] += (alpha / r_n) * sum_k B_s[n][c][k] * (sum_j A_s[n][k][j] * x_i[j]),
 *     n = ids[i];  rows with ids[i] == -1 are left untouched.
 *
 * Naming follows the page "Multi-LoRA Serving: one base, many adapters",
 * section 3.1 (Delta W = B A, B in R^{d_out x r}, A in R^{r x d_in},
 * y = W x + B(A x) * alpha/r).  The adapters of all N resident slots are stacked
 * into one tensor per projection and picked per row by an integer id (page
 * "LoRA service: multi-adapter dynamic loading", section 2: A_all
 * [N_adapters, r, d] plus a per-request adapter id; page "LoRA hot load and
 * adapter routing": per-request lora_ids where None means the base model).
 * The shared base product W x is not part of this library: y arrives holding
 * it and leaves holding it plus the delta (merge step of the page "Multi-LoRA
 * Serving", section 2 flowchart: y_i = base_i + delta_i).
 *
 * Conventions for every entry point
 *   - Pointers named d_* or documented "device" are device memory owned by the
 *     caller.  The library allocates nothing, keeps no pointer after a call
 *     returns, and never synchronises the stream.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  All work
 *     is enqueued on it; a call returns as soon as it is enqueued.
 *   - The return value reports only what the host can see (lora_status).
 *     Problems found on the device (an id outside [-1, N), a rank outside
 *     [1, r_max], a full tile list) are OR-ed into the int32 device word
 *     `status` (LORA_DEV_* bits); the affected rows are skipped, never trapped.
 *   - Element type: LORA_BF16 (x, y, A, B all bf16, fp32 accumulation) or
 *     LORA_FP32 (all fp32).  Rounding into y happens once, round-to-nearest-even.
 *   - Layouts are row-major with element strides:
 *         x      [T][ld_x]            d_in columns used
 *         A_s    [N][r_max][d_in]     rank rows k >= r_n are padding: they may be read
 *                                     (up to r_n rounded up to 8) but never affect the
 *                                     result, whatever they hold (NaN included)
 *         B_s    [N][d_out_s][r_max]  rank columns k >= r_n are padding, as for A
 *         y      [T][ld_y]            slice s owns columns col_off_s .. +d_out_s; slices
 *                                     that overlap, or run past ld_y, are LORA_ERR_SHAPE;
 *                                     y must not overlap x
 *         ranks  [N] int32 device,    r_n in [1, r_max]
 *         alphas [N] fp32 device,     alpha_n of adapter n; the library scales adapter n's
 *                                     delta by alpha_n / r_n (page "Multi-LoRA Serving",
 *                                     3.1: y = W x + B(A x) * alpha / r), computed on the
 *                                     device in fp32 from alphas[n] and ranks[n]
 *
 * Tuning overrides (environment, read at each call; unset = the library's own
 * choice).  They change only the launch shape: results stay within the same
 * tolerance of the exact value, and a fixed setting gives bit-identical results
 * from run to run.  A value outside the range is ignored.
 *   LORA_BG_BLOCKS      1 to 4096: blocks of the gathered-tile kernel's persistent
 *                       grid (default: one per SM)
 *   LORA_BG_ITEM_COLS   32 to 8192, a multiple of 32: output columns of one expand item
 *   LORA_BG_KSPLIT      1 or 2: pieces a fused call's shrink items are split into along
 *                       d_in (default 2 for batches small enough to leave most SMs idle
 *                       in the shrink, else 1)
 *   LORA_BG_TC          1: fused calls whose tiles have at most 16 rows run on the
 *                       tensor-core gathered-tile kernel (tcgen05 MMAs, TMA copies,
 *                       accumulators in tensor memory) instead of the mma.sync one;
 *                       off by default (correct, slower on the decode layer set)
 *   LORA_BT_COLS        128 to 512, a multiple of 128: output columns of one expand
 *                       item of the tensor-core gathered-tile kernel
 *   LORA_TC_CLUSTER     1, 2, 4 or 8: blocks per cluster of the tensor-core kernel;
 *                       when the shape cannot use it, the contiguous tiles run on
 *                       the gathered-tile kernel instead
 *   LORA_TC_STAGES      2 to 6: depth of the tensor-core kernel's load ring (ignored
 *                       when shared memory cannot hold that many stages)
 *   LORA_TC_ROUTE       1: lora_add_linear gives contiguous tiles to the tensor-core
 *                       kernel whenever it qualifies; 2: never (the gathered-tile
 *                       kernel takes every row).  Default: the tensor-core kernel unless
 *                       the batch has fewer 128-row tiles than SMs and the layer's
 *                       slices total 8192 or more output columns (lora_segment_plan
 *                       follows the same setting)
 *   LORA_TC_LOAD_ROWS   8 to 128, a power of two: rows per x / y load box
 *   LORA_TC_STORE_ROWS  8 to 128, a power of two: rows per y store box
 *
 * Test hook (environment, read at each call; never set it in production):
 *   LORA_DEBUG_STALL=1  the gathered-tile kernel's expand items wait, with a bound of
 *                       a few ms, for one shrink signal more than their unit gives:
 *                       the waits run out, LORA_DEV_TIMEOUT is set, the call's
 *                       results are unreliable, and the kernel still completes (the
 *                       context stays usable).
 */
#ifndef LORA_DELTA_H
#define LORA_DELTA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LORA_API __attribute__((visibility("default")))
#else
#define LORA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Host-detected status, returned by every entry point. */
typedef enum {
    LORA_OK = 0,
    LORA_ERR_NULL = -1,       /* a required pointer is NULL */
    LORA_ERR_DTYPE = -2,      /* unknown element type */
    LORA_ERR_SHAPE = -3,      /* a size or stride is out of range or inconsistent */
    LORA_ERR_RANK = -4,       /* r_max outside [1, LORA_MAX_RANK] */
    LORA_ERR_ALIGN = -5,      /* reserved: misaligned data takes a slower path instead */
    LORA_ERR_WORKSPACE = -6,  /* scratch or workspace smaller than required */
    LORA_ERR_CAPACITY = -7,   /* a tile-list capacity below lora_meta_capacity() */
    LORA_ERR_CUDA = -8        /* a CUDA launch failed (cudaGetLastError) */
} lora_status;

/* Bits OR-ed into the device status word. */
#define LORA_DEV_BAD_ID        1  /* id outside [-1, N): that row is treated as -1 */
#define LORA_DEV_TILE_OVERFLOW 2  /* tile list full: the rows of dropped tiles are untouched */
#define LORA_DEV_BAD_RANK      4  /* ranks[n] outside [1, r_max]: rows of adapter n untouched */
#define LORA_DEV_TIMEOUT       8  /* a bounded wait ran out: the call's results are unreliable */

typedef enum { LORA_BF16 = 0, LORA_FP32 = 1 } lora_dtype;

#define LORA_MAX_ROWS    131072  /* rows per call */
#define LORA_MAX_ADAPTERS  4096  /* adapter slots N */
#define LORA_MAX_RANK       128  /* r_max */
#define LORA_MAX_SLICES       8  /* output slices of one linear layer */
#define LORA_LONG_TILE      128  /* rows per contiguous tile */
#define LORA_MAX_TILE_ROWS   64  /* rows per gathered tile (lora_meta.rows_per_tile) */

/*
 * Batch metadata: the grouping of rows by adapter id (page "Multi-LoRA
 * Serving", section 2 flowchart "group rows by adapter id", section 3.2; page
 * "LoRA hot load and adapter routing", LoraBatchInfo) made concrete.  The
 * struct lives in host memory; every array it points to is device memory of
 * the stated size, written by lora_build_segments and read by the compute
 * entry points.
 *
 *   perm          [T]      rows with a valid id ordered by (id, row), then the others by row
 *   seg_start     [N+1]    seg_start[n] = number of valid rows with id < n
 *   seg_adapter   [N]      ids with at least one row, ascending (counts[0] of them)
 *   counts        [4]      n_seg, n_gather_tiles, n_contig_tiles, n_gathered_rows
 *   grow          [T]      rows outside long runs, grouped by id (perm order)
 *   gather_tiles  [max_gather_tiles][4]  {id, first index into grow, rows, 0}
 *   contig_tiles  [max_contig_tiles][4]  {id, first row, rows, 0}
 *
 * A run is a maximal block of consecutive rows with one id (a prompt during
 * prefill).  Runs of at least min_run rows (min_run > 0) are cut into
 * contiguous tiles of at most long_tile rows; every other row is gathered,
 * and each id's gathered rows are cut into tiles of at most rows_per_tile.
 * The fused kernel reads a tile's adapter once for all of the tile's rows, but
 * a tile's shrink runs on one SM and its expand waits for it: 16-row tiles
 * measured best on decode batches (64-row tiles were 8 % slower on a
 * Llama-3-8B layer set at 1024 rows).  lora_segment_plan gives rows_per_tile
 * and min_run for a batch whose layers all take the fused kernel for every row.
 */
typedef struct {
    int32_t T;
    int32_t N;
    int32_t rows_per_tile;      /* 1 .. LORA_MAX_TILE_ROWS */
    int32_t min_run;            /* 0 = no contiguous tiles, else >= 1 */
    int32_t long_tile;          /* LORA_LONG_TILE */
    int32_t max_gather_tiles;   /* capacity, >= lora_meta_capacity() */
    int32_t max_contig_tiles;   /* capacity, >= lora_meta_capacity() */
    int32_t *perm;
    int32_t *seg_start;
    int32_t *seg_adapter;
    int32_t *counts;
    int32_t *grow;
    int32_t *gather_tiles;
    int32_t *contig_tiles;
} lora_meta;

/* One output slice of a linear layer (q, k, v of a fused QKV; gate, up of a
 * fused gate/up; or the single output of o/down).  A and B are device
 * pointers to the stacked adapters of that slice. */
typedef struct {
    const void *A;      /* [N][r_max][d_in] */
    const void *B;      /* [N][d_out][r_max] */
    int32_t d_out;
    int32_t col_off;    /* first column of this slice in y */
} lora_slice;

/* Library version (major*10000 + minor*100 + patch). */
LORA_API int lora_version(void);

/* Human-readable name of a lora_status value. */
LORA_API const char *lora_status_string(int status);

/* The CUDA failure behind the last LORA_ERR_CUDA returned on the calling
 * thread ("cudaErrorName: description", or the failing driver step); an empty
 * string if there was none.  The text stays valid until the thread's next
 * failing call.  No counterpart in the pages: a diagnostic of this library. */
LORA_API const char *lora_last_error(void);

/*
 * Tile-list capacities that always suffice for a batch of T rows over N
 * slots: *max_gather >= T/rows_per_tile + N, *max_contig >= T/long_tile +
 * T/min_run.  Returns LORA_ERR_SHAPE on out-of-range arguments.
 */
LORA_API int lora_meta_capacity(int32_t T, int32_t N, int32_t rows_per_tile, int32_t min_run,
                       int32_t long_tile, int32_t *max_gather, int32_t *max_contig);

/* Device scratch bytes lora_build_segments needs for T rows over N slots,
 * each part rounded up to 256 bytes: per-chunk id counts (4 * (N+1) per 2048
 * rows), one byte per row, 12 bytes per 32 rows (run bitmaps and offsets) and
 * 16 bytes per 2048 rows (per-block totals).  0 when T <= 2048, or T <= 8192
 * and N <= 1023: the grouping then runs in one thread block, in shared memory.
 * Also 0 for T outside [0, LORA_MAX_ROWS] or N outside [1, LORA_MAX_ADAPTERS]
 * (lora_build_segments then returns LORA_ERR_SHAPE). */
LORA_API size_t lora_segments_scratch_bytes(int32_t T, int32_t N);

/*
 * Group the rows of a batch by adapter id and write the tile lists into the
 * arrays of *meta (see lora_meta).  ids: device int32 [meta->T].
 * scratch: device memory of lora_segments_scratch_bytes() bytes (may be NULL
 * when that is 0); its contents on entry do not matter.  status: device int32,
 * receives LORA_DEV_BAD_ID / LORA_DEV_TILE_OVERFLOW.  Deterministic: equal ids
 * give bit-identical metadata.
 */
LORA_API int lora_build_segments(const int32_t *ids, const lora_meta *meta, void *scratch,
                        size_t scratch_bytes, int32_t *status, void *stream);

/*
 * Bytes of the scratch array compiled into the library for
 * lora_build_segments_static (1 MiB per device that loads the library).
 */
#define LORA_STATIC_SCRATCH_BYTES (1 << 20)

/*
 * lora_build_segments without caller-provided scratch memory.  The pages have
 * no counterpart: this exists for callers that cannot allocate device memory
 * when they group a batch (a pool that owns all device memory, callbacks and
 * hooks that must not call cudaMalloc, runtimes that only hand over input and
 * output buffers).  Same ids, meta and status as lora_build_segments, same
 * results; the scratch is one library-owned array of
 * LORA_STATIC_SCRATCH_BYTES bytes per device, so nothing is allocated.
 *   - Returns what lora_build_segments returns for the same meta (checked
 *     first), then LORA_ERR_WORKSPACE when lora_segments_scratch_bytes(T, N)
 *     exceeds LORA_STATIC_SCRATCH_BYTES (use lora_build_segments then).
 *   - Every call (that device current) asks the CUDA runtime for the array's
 *     device address; the first call on a device may load the library's
 *     module there, so make one call on each device before any stream
 *     capture.  Nothing is cached across calls, so a cudaDeviceReset between
 *     calls leaves no stale address behind.
 *   - Every call uses the same array; calls that overlap on the GPU race and
 *     corrupt each other: keep them ordered (one stream).
 */
LORA_API int lora_build_segments_static(const int32_t *ids, const lora_meta *meta,
                                        int32_t *status, void *stream);

/* Bytes of the fp32 intermediate v = A x that lora_sgmv_shrink writes and
 * lora_sgmv_expand reads: n_slices * T * r_max * 4. */
LORA_API size_t lora_shrink_workspace_bytes(int32_t T, int32_t r_max, int32_t n_slices);

/*
 * Shrink (page "Multi-LoRA Serving", section 3.4: add_shrink, the rank-r
 * v = A x, grouped per adapter).  For every row i with a valid id n and every
 * slice s: v[(s*T + i)*r_max + k] = sum_j A_s[n][k][j] x_i[j] for k < r_n, in
 * fp32.  Entries of rows without an adapter, and k >= r_n, are not written.
 * v: device fp32 [n_slices][T][r_max].
 */
LORA_API int lora_sgmv_shrink(float *v, const void *x, int64_t ld_x, int32_t d_in,
                     const lora_slice *slices, int32_t n_slices, int32_t r_max,
                     const int32_t *ranks, const lora_meta *meta, lora_dtype dtype,
                     int32_t *status, void *stream);

/*
 * Expand and merge (page "Multi-LoRA Serving", section 3.4: add_expand,
 * delta = B v * alpha/r, grouped per adapter, added into the base output).
 * For every row i with a valid id n: y_i[col_off_s + c] += (alphas[n] / r_n) *
 * sum_{k < r_n} B_s[n][c][k] v[(s*T + i)*r_max + k].  v as written by
 * lora_sgmv_shrink.
 */
LORA_API int lora_sgmv_expand(void *y, int64_t ld_y, const float *v, const lora_slice *slices,
                     int32_t n_slices, int32_t r_max, const int32_t *ranks,
                     const float *alphas, const lora_meta *meta, lora_dtype dtype,
                     int32_t *status, void *stream);

/*
 * Bytes of the workspace lora_bgmv_fused and lora_add_linear take for a batch
 * grouped into *meta and a layer of n_slices slices with rank slots r_max: a
 * 256-byte head of control words, one int per unit of work (tile capacity of
 * the meta, rounded up to 256 bytes), then room for v: the larger of
 * [2][n_slices][T][r_max] fp32 (a small batch's shrink items may be split in two
 * along d_in, each half with its own partial v) and, per unit and slice, a bf16 hi + lo pair of 16
 * rows by r_max rounded up to 16 ranks (the tensor-core gathered-tile kernel's
 * form).  0 for invalid arguments.
 *
 * The workspace belongs to the caller.  Its head must hold zeros before the
 * first call that uses it (allocate it zero-filled, or cudaMemset it once);
 * every call leaves the head at zero again when its kernel completes, so one
 * workspace serves call after call, CUDA graph replays included.  Calls that
 * share a workspace must not overlap on the GPU (keep them on one stream).
 */
LORA_API size_t lora_linear_workspace_bytes(const lora_meta *meta, int32_t n_slices, int32_t r_max);

/*
 * Fused shrink + expand for every tile (BGMV: page "Multi-LoRA Serving",
 * section 3.2, SGMV/BGMV-style grouped products), in one kernel launch: a
 * thread block reduces A x for all rows of a tile (up to 64 rows of one
 * adapter) and 32 of its ranks, its warps splitting the input columns, and
 * warps then expand the tile's output columns in small items, each starting as
 * soon as its tile is reduced.  v passes between the two through the workspace
 * (it stays in L2; only x, y and the adapters' live ranks cross HBM).  Same result as
 * lora_sgmv_shrink followed by lora_sgmv_expand.  workspace: device memory of
 * lora_linear_workspace_bytes() bytes, 256-byte aligned (LORA_ERR_WORKSPACE
 * otherwise; see there for its contract).
 */
LORA_API int lora_bgmv_fused(void *y, int64_t ld_y, const void *x, int64_t ld_x, int32_t d_in,
                    const lora_slice *slices, int32_t n_slices, int32_t r_max,
                    const int32_t *ranks, const float *alphas, const lora_meta *meta,
                    void *workspace, size_t workspace_bytes, lora_dtype dtype,
                    int32_t *status, void *stream);

/*
 * add_lora_linear (page "Multi-LoRA Serving", section 3.4: one call serves a
 * whole heterogeneous batch, shrink then expand, no per-adapter loop): applies
 * every slice of one linear layer (fused QKV, gate/up, or a single output) to
 * y in place.  Gathered tiles (decode rows) take the fused BGMV kernel;
 * contiguous tiles (prompt runs) take the tensor-core SGMV kernel when the
 * data is bf16, except when the batch has fewer 128-row tiles than the GPU has
 * SMs and the layer's slices total 8192 or more output columns: then the fused
 * BGMV kernel takes every row in one launch (it spreads a wide layer's columns
 * over every SM; LORA_TC_ROUTE overrides; lora_segment_plan gives the segment
 * build that suits this route); everything else takes the general kernel.
 * Same result as
 * lora_bgmv_fused; the same workspace contract.  When both kinds of tiles are
 * present the gathered ones run on a library-owned second stream, forked from
 * and joined back into `stream` with events (also under stream capture); each
 * caller stream gets a second stream of its own, created by the first such
 * call on that stream, so make that call before capturing the stream.
 */
LORA_API int lora_add_linear(void *y, int64_t ld_y, const void *x, int64_t ld_x, int32_t d_in,
                    const lora_slice *slices, int32_t n_slices, int32_t r_max,
                    const int32_t *ranks, const float *alphas, const lora_meta *meta,
                    void *workspace, size_t workspace_bytes, lora_dtype dtype,
                    int32_t *status, void *stream);

/*
 * Segment-build plan for one batch that will run through lora_add_linear
 * (page "Multi-LoRA Serving", section 3.2: SGMV for prompt segments and BGMV
 * for single rows in one heterogeneous batch; which rows become segments is the
 * scheduler's choice).  Host only: no device work, no stream.
 *
 *   T            rows of the batch, 0..LORA_MAX_ROWS
 *   layer_cols   host array of n_layers entries: per layer the total output
 *                columns of its slices (sum of d_out); may be NULL when n_layers
 *                is 0
 *   sms          SMs of the device the batch runs on, or 0 for the current device
 *   long_tile    rows per contiguous tile the meta will use, 1..LORA_LONG_TILE
 *   rows_per_tile, min_run  in: the caller's choice for this batch (min_run 0 =
 *                no contiguous tiles); out: the plan
 *   all_gathered optional host array of n_layers bytes (NULL to skip): 1 where
 *                lora_add_linear sends every row of that layer to the fused
 *                BGMV kernel, 0 where the tensor-core kernel may take its
 *                contiguous tiles
 *
 * A layer routes all rows to the fused BGMV kernel when the batch has fewer
 * long_tile-row tiles than SMs and the layer is 8192 or more columns wide (the
 * rule lora_add_linear applies; LORA_TC_ROUTE = 1 / 2 forces 0 / 1 for every
 * layer).  When every layer does and min_run > 0, contiguous runs would only be
 * cut back into gathered tiles, so the plan is min_run = 0 with 32-row tiles;
 * otherwise the caller's values come back unchanged.  Returns LORA_ERR_NULL
 * for a missing pointer, LORA_ERR_SHAPE for T, n_layers (0..4096), sms,
 * long_tile, rows_per_tile (1..LORA_MAX_TILE_ROWS), min_run (>= 0) or a
 * layer's columns (>= 1) out of range, with nothing written.
 */
LORA_API int lora_segment_plan(int32_t T, const int64_t *layer_cols, int32_t n_layers, int32_t sms,
                               int32_t long_tile, int32_t *rows_per_tile, int32_t *min_run,
                               uint8_t *all_gathered);


/*
 * Adapter slots (page "LoRA hot load and adapter routing", adapter lifecycle:
 * load, check the rank, copy to the GPU, evict the least recently used adapter
 * when the slots are full; page "Multi-LoRA Serving", section 3.2: max_loras
 * adapters resident, max_lora_rank the slot size).
 *
 * lora_load_adapter: put one adapter of rank r into slot n of every slice's
 * stacked tensors, on `stream`:
 *     A_s[n][0:r][:]     = src_A[s]  ([r][d_in] row-major)
 *     A_s[n][r:r_max][:] = 0
 *     B_s[n][:][0:r]     = src_B[s]  ([d_out_s][r] row-major)
 *     B_s[n][:][r:r_max] = 0
 *     ranks[n] = r, alphas[n] = alpha   (device words, written by a kernel)
 * slices[s].A / .B are the stacks ([N][r_max][d_in], [N][d_out_s][r_max]);
 * col_off is not used.  src_A[s] / src_B[s] may be device memory or pinned
 * host memory (the copy engines read them); they must stay valid until the
 * stream reaches the call.  Everything is enqueued on the stream: batches
 * enqueued after it on that stream see the new adapter, batches enqueued before
 * it see the old one.  Returns LORA_ERR_RANK for r outside [1, r_max],
 * LORA_ERR_SHAPE for n outside [0, N).
 */
LORA_API int lora_load_adapter(const lora_slice *slices, int32_t n_slices, int32_t d_in,
                               int32_t r_max, int32_t N, int32_t n, int32_t r,
                               const void *const *src_A, const void *const *src_B, float alpha,
                               int32_t *ranks, float *alphas, lora_dtype dtype, void *stream);

/*
 * Host policy for the slots: which slot holds which adapter (a caller-chosen
 * key >= 0), least recently used first out.  Thread-safe; host memory only.
 *   acquire  the adapter's slot and one pin on it.  *resident = 1: the slot
 *            already holds the adapter; 0: the slot was given to it (a free slot
 *            first, else the least recently acquired slot with no pins) and the
 *            caller must load it (lora_load_adapter).  LORA_ERR_CAPACITY when
 *            every slot is pinned.
 *   release  one pin (a batch that read the slot has completed).
 *   key      the key a slot holds, -1 if free.
 *   evict    free the adapter's slot (LORA_ERR_CAPACITY while pinned).
 */
typedef struct lora_slot_cache lora_slot_cache;
LORA_API lora_slot_cache *lora_slot_cache_create(int32_t n_slots);
LORA_API void lora_slot_cache_destroy(lora_slot_cache *cache);
LORA_API int lora_slot_cache_acquire(lora_slot_cache *cache, int64_t key, int32_t *slot,
                                     int32_t *resident);
LORA_API int lora_slot_cache_release(lora_slot_cache *cache, int32_t slot);
LORA_API int64_t lora_slot_cache_key(lora_slot_cache *cache, int32_t slot);
LORA_API int lora_slot_cache_evict(lora_slot_cache *cache, int64_t key);

/*
 * Merge / unmerge one adapter into a dense base weight (page "LoRA service:
 * multi-adapter dynamic loading", section 1: W' = W + B A for a single-tenant
 * deployment, with the scale alpha / r of page "Multi-LoRA Serving", 3.1):
 *     W[o][i] += sign * (alphas[n] / r_n) * sum_{k < r_n} B[n][o][k] A[n][k][i]
 * for o < d_out, i < d_in.  W: device [d_out][ld_w] (row o = output feature o,
 * as in y = W x); A [N][r_max][d_in] and B [N][d_out][r_max]: one slice's
 * stacks; n: the slot; sign: +1 merges, -1 unmerges.  fp32 products and
 * accumulation, W rounded once (round-to-nearest-even); unmerging a merged
 * adapter restores W up to that rounding.  ranks[n] outside [1, r_max] sets
 * LORA_DEV_BAD_RANK and leaves W unchanged.  Padding ranks never affect W.
 */
LORA_API int lora_merge_adapter(void *W, int64_t ld_w, int32_t d_out, int32_t d_in, const void *A,
                                const void *B, int32_t N, int32_t r_max, int32_t n,
                                const int32_t *ranks, const float *alphas, int32_t sign,
                                lora_dtype dtype, int32_t *status, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* LORA_DELTA_H */
