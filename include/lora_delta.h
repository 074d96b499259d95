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
 *         A_s    [N][r_max][d_in]     rank rows k >= r_n are padding, never read
 *         B_s    [N][d_out_s][r_max]  rank columns k >= r_n are padding, never read
 *         y      [T][ld_y]            slice s owns columns col_off_s .. +d_out_s; slices
 *                                     that overlap, or run past ld_y, are LORA_ERR_SHAPE
 *         ranks  [N] int32 device,    r_n in [1, r_max]
 *         scales [N] fp32 device,     alpha / r_n (page "Multi-LoRA Serving", 3.1)
 *
 * Tuning overrides (environment, read at each call; unset = the library's own
 * choice).  They change only the launch shape: results stay within the same
 * tolerance of the exact value, and a fixed setting gives bit-identical results
 * from run to run.  A value outside the range is ignored.
 *   LORA_BG_CLUSTER     1, 2, 4 or 8: blocks per cluster of the gathered-tile kernel
 *   LORA_BG_STAGES      2 or 3: stages of the gathered-tile kernel's 72 KB load ring
 *   LORA_TC_CLUSTER     1, 2, 4 or 8: blocks per cluster of the tensor-core kernel;
 *                       when the shape cannot use it, the contiguous tiles run on
 *                       the gathered-tile kernel instead
 *   LORA_TC_STAGES      2 to 6: depth of the tensor-core kernel's load ring (ignored
 *                       when shared memory cannot hold that many stages)
 *   LORA_TC_LOAD_ROWS   8 to 128, a power of two: rows per x / y load box
 *   LORA_TC_STORE_ROWS  8 to 128, a power of two: rows per y store box
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
#define LORA_DEV_TIMEOUT       8  /* a bounded on-chip wait ran out: the block's rows are unreliable */

typedef enum { LORA_BF16 = 0, LORA_FP32 = 1 } lora_dtype;

#define LORA_MAX_ROWS    131072  /* rows per call */
#define LORA_MAX_ADAPTERS  4096  /* adapter slots N */
#define LORA_MAX_RANK       128  /* r_max */
#define LORA_MAX_SLICES       8  /* output slices of one linear layer */
#define LORA_LONG_TILE      128  /* rows per contiguous tile */

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
 */
typedef struct {
    int32_t T;
    int32_t N;
    int32_t rows_per_tile;      /* 1 .. 16 */
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
 * and N <= 1023: the grouping then runs in one thread block, in shared memory. */
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
 *   - Returns LORA_ERR_WORKSPACE when lora_segments_scratch_bytes(T, N)
 *     exceeds LORA_STATIC_SCRATCH_BYTES (use lora_build_segments then).
 *   - The first call on a device (that device current) looks up the array's
 *     device address; make it before any stream capture.
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
 * For every row i with a valid id n: y_i[col_off_s + c] += scales[n] *
 * sum_{k < r_n} B_s[n][c][k] v[(s*T + i)*r_max + k].  v as written by
 * lora_sgmv_shrink.
 */
LORA_API int lora_sgmv_expand(void *y, int64_t ld_y, const float *v, const lora_slice *slices,
                     int32_t n_slices, int32_t r_max, const int32_t *ranks,
                     const float *scales, const lora_meta *meta, lora_dtype dtype,
                     int32_t *status, void *stream);

/*
 * Fused shrink + expand for every tile (BGMV: page "Multi-LoRA Serving",
 * section 3.2, SGMV/BGMV-style grouped products).  The rank-r intermediate of
 * each tile never leaves the chip: a cluster of thread blocks reduces A x
 * through distributed shared memory and expands from there.  Same result as
 * lora_sgmv_shrink followed by lora_sgmv_expand.
 */
LORA_API int lora_bgmv_fused(void *y, int64_t ld_y, const void *x, int64_t ld_x, int32_t d_in,
                    const lora_slice *slices, int32_t n_slices, int32_t r_max,
                    const int32_t *ranks, const float *scales, const lora_meta *meta,
                    lora_dtype dtype, int32_t *status, void *stream);

/*
 * add_lora_linear (page "Multi-LoRA Serving", section 3.4: one call serves a
 * whole heterogeneous batch, shrink then expand, no per-adapter loop): applies
 * every slice of one linear layer (fused QKV, gate/up, or a single output) to
 * y in place.  Gathered tiles (decode rows) take the fused BGMV kernel;
 * contiguous tiles (prompt runs) take the tensor-core SGMV kernel when the
 * data is bf16; everything else takes the general kernel.  Same result as
 * lora_bgmv_fused.  When both kinds of tiles are present the gathered ones run
 * on a library-owned second stream, forked from and joined back into `stream`
 * with events (also under stream capture); the first such call on a device
 * creates that stream and its events, so make it before any capture.
 */
LORA_API int lora_add_linear(void *y, int64_t ld_y, const void *x, int64_t ld_x, int32_t d_in,
                    const lora_slice *slices, int32_t n_slices, int32_t r_max,
                    const int32_t *ranks, const float *scales, const lora_meta *meta,
                    lora_dtype dtype, int32_t *status, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* LORA_DELTA_H */
