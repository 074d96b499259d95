/*
 * Multi-LoRA delta oracle: plain, slow, obviously correct CPU statement of the
 * method, in fp64.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the smoke check and the CPU
 * baseline leg of the benchmark may load this file's library.  The product
 * path (the CUDA library under lora_adapter_application_b200/) never calls it,
 * and this file shares no code, header, table or helper with it.
 *
 * What it computes (page "Multi-LoRA Serving: one base, many adapters",
 * section 3.1, the equation y = Wx + B(Ax)*alpha/r with B in R^{d x r},
 * A in R^{r x k}; section 2, the per-row formula y_i = W x_i + B_a(i) A_a(i) x_i
 * * alpha/r; page "LoRA service: multi-adapter dynamic loading", section 2,
 * adapters stacked as [N_adapters, r, d] and selected per request by an integer
 * id; page "LoRA hot load and adapter routing", "LoraBatchInfo" paragraph:
 * an id of None means the base model only):
 *
 *   for every row i with 0 <= id[i] < N, adapter n = id[i], rank r_n:
 *       v[k]          = sum_j A[n][k][j] * x[i][j]                 k < r_n
 *       y[i][off_s+c] = y0[i][off_s+c] + (alpha/r_n) * sum_k B[n][c][k] * v[k]
 *   rows with id == -1 (or any id outside [0,N)) keep y0 unchanged.
 *
 * Inputs are bf16 or fp32 bit patterns, widened exactly to double.  The result
 * is returned unrounded in fp64.  The oracle follows the pages' naive loop
 * (page "LoRA hot load ...", "batched LoRA" listing: per adapter, gather rows,
 * two small products, add into the base output) but loops per row, which gives
 * the same sums because every row is computed on its own.
 *
 * The segment builder statement (oracle_build_segments) is the grouping step
 * "group rows by adapter id" of the page "Multi-LoRA Serving", section 2
 * flowchart and section 3.2, made concrete as a stable counting sort plus the
 * tile lists the library's kernels walk.  Its tile rules are this library's own
 * contract; the pages fix only the grouping.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_BF16 0
#define ORACLE_FP32 1

/* bf16 is the upper half of an IEEE binary32: widening is exact. */
static double widen(int dtype, const void *base, int64_t idx)
{
    if (dtype == ORACLE_FP32)
        return (double)((const float *)base)[idx];
    uint32_t u = (uint32_t)((const uint16_t *)base)[idx] << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/*
 * Delta application for the rows listed in rows[0..n_rows) (rows == NULL means
 * all T rows in order).  y_out is [n_rows x ld_y] fp64 and receives, for each
 * listed row, y0's row widened plus the delta of every slice.
 *
 * Layouts (all row-major, as stacked by the page "LoRA service", section 2):
 *   x        [T][ld_x]               row i at x + i*ld_x, d_in used columns
 *   A[s]     [N][r_max][d_in]        adapter n, rank row k, input column j
 *   B[s]     [N][d_out[s]][r_max]    adapter n, output column c, rank k
 *   y0       [T][ld_y]               slice s owns columns col_off[s] .. +d_out[s]
 * ranks[n] is r_n (0 < r_n <= r_max); rank rows k >= r_n are padding, never read.
 * Returns 0, or -1 on a bad argument.
 */
int oracle_lora_apply(int dtype, const void *x, int64_t ld_x, int32_t d_in,
                      int32_t n_slices, const void *const *A, const void *const *B,
                      const int32_t *d_out, const int32_t *col_off,
                      int32_t N, int32_t r_max, const int32_t *ranks, double alpha,
                      const int32_t *ids, int32_t T, const int32_t *rows, int32_t n_rows,
                      const void *y0, int64_t ld_y, double *y_out)
{
    if (dtype != ORACLE_BF16 && dtype != ORACLE_FP32)
        return -1;
    if (T < 0 || n_rows < 0 || d_in <= 0 || n_slices <= 0 || N <= 0 || r_max <= 0 || r_max > 1024)
        return -1;
    int32_t count = rows ? n_rows : T;

#pragma omp parallel for schedule(dynamic, 4)
    for (int32_t q = 0; q < count; ++q) {
        int32_t i = rows ? rows[q] : q;
        double *yo = y_out + (int64_t)q * ld_y;
        for (int64_t c = 0; c < ld_y; ++c)
            yo[c] = widen(dtype, y0, (int64_t)i * ld_y + c);

        int32_t n = ids[i];
        if (n < 0 || n >= N)
            continue;                       /* base model only: no change */
        int32_t r = ranks[n];
        if (r <= 0 || r > r_max)
            continue;                       /* rejected adapter: no change */
        double scale = alpha / (double)r;   /* alpha / r, page 3 section 3.1 */

        double v[1024];
        for (int32_t s = 0; s < n_slices; ++s) {
            /* shrink: v = A_n x_i */
            for (int32_t k = 0; k < r; ++k) {
                double acc = 0.0;
                for (int32_t j = 0; j < d_in; ++j)
                    acc += widen(dtype, A[s], ((int64_t)n * r_max + k) * d_in + j) *
                           widen(dtype, x, (int64_t)i * ld_x + j);
                v[k] = acc;
            }
            /* expand and merge: y_i += scale * B_n v */
            for (int32_t c = 0; c < d_out[s]; ++c) {
                double acc = 0.0;
                for (int32_t k = 0; k < r; ++k)
                    acc += widen(dtype, B[s], ((int64_t)n * d_out[s] + c) * r_max + k) * v[k];
                yo[col_off[s] + c] += scale * acc;
            }
        }
    }
    return 0;
}

/*
 * The shrink alone (page "Multi-LoRA Serving", section 3.4: add_shrink, the
 * rank-r v = A x): v_out[q][s][k] = sum_j A_s[n][k][j] * x_i[j] for the listed
 * rows, k < r_n, in fp64; entries of rows without a valid adapter, and k >= r_n,
 * are set to 0.  v_out is [n_rows][n_slices][r_max].
 */
int oracle_lora_shrink(int dtype, const void *x, int64_t ld_x, int32_t d_in,
                       int32_t n_slices, const void *const *A, int32_t N, int32_t r_max,
                       const int32_t *ranks, const int32_t *ids, const int32_t *rows,
                       int32_t n_rows, double *v_out)
{
    if (dtype != ORACLE_BF16 && dtype != ORACLE_FP32)
        return -1;
    if (n_rows < 0 || d_in <= 0 || n_slices <= 0 || N <= 0 || r_max <= 0)
        return -1;
#pragma omp parallel for schedule(dynamic, 4)
    for (int32_t q = 0; q < n_rows; ++q) {
        int32_t i = rows[q];
        double *vo = v_out + (int64_t)q * n_slices * r_max;
        for (int64_t e = 0; e < (int64_t)n_slices * r_max; ++e)
            vo[e] = 0.0;
        int32_t n = ids[i];
        if (n < 0 || n >= N)
            continue;
        int32_t r = ranks[n];
        if (r <= 0 || r > r_max)
            continue;
        for (int32_t s = 0; s < n_slices; ++s)
            for (int32_t k = 0; k < r; ++k) {
                double acc = 0.0;
                for (int32_t j = 0; j < d_in; ++j)
                    acc += widen(dtype, A[s], ((int64_t)n * r_max + k) * d_in + j) *
                           widen(dtype, x, (int64_t)i * ld_x + j);
                vo[s * r_max + k] = acc;
            }
    }
    return 0;
}

/*
 * Grouping of rows by adapter id, and the work lists.
 *
 *   valid(i)      = 0 <= ids[i] < N
 *   perm          = valid rows ordered by (ids[i], i), then the other rows by i
 *   seg_start[n]  = number of valid rows with id < n      (n = 0..N)
 *   seg_adapter   = the ids n with at least one row, ascending; counts[0] = how many
 *
 *   A "run" is a maximal stretch of perm positions inside one segment whose
 *   rows are consecutive integers (that is, a maximal block of equal ids in
 *   the original row order).  A run is long when min_run > 0 and its length is
 *   at least min_run.
 *
 *   contiguous tiles: each long run, in position order, cut every long_tile
 *       rows: {n, first row, count}.                         counts[2] = how many
 *   gathered rows:   grow = the rows of the non-long positions, in perm order;
 *       counts[3] = how many.
 *   gathered tiles:  each segment's gathered rows, cut every rows_per_tile:
 *       {n, first index into grow, count}.                    counts[1] = how many
 *
 * Tiles are written as 4 int32 {adapter, start, count, 0}.  Returns the bit set
 * of problems found: 1 = an id outside [-1, N), 2 = a tile list over capacity
 * (tiles beyond capacity are dropped).
 */
int oracle_build_segments(const int32_t *ids, int32_t T, int32_t N,
                          int32_t rows_per_tile, int32_t min_run, int32_t long_tile,
                          int32_t max_gather_tiles, int32_t max_contig_tiles,
                          int32_t *perm, int32_t *seg_start, int32_t *seg_adapter,
                          int32_t *counts, int32_t *grow,
                          int32_t *gather_tiles, int32_t *contig_tiles)
{
    int status = 0;
    int32_t pos = 0;

    for (int32_t i = 0; i < T; ++i)
        if (ids[i] < -1 || ids[i] >= N)
            status |= 1;

    /* stable grouping by id: for each id in turn, its rows in row order */
    for (int32_t n = 0; n < N; ++n) {
        seg_start[n] = pos;
        for (int32_t i = 0; i < T; ++i)
            if (ids[i] == n)
                perm[pos++] = i;
    }
    seg_start[N] = pos;
    int32_t P = pos;
    for (int32_t i = 0; i < T; ++i)
        if (ids[i] < 0 || ids[i] >= N)
            perm[pos++] = i;

    int32_t n_seg = 0;
    for (int32_t n = 0; n < N; ++n)
        if (seg_start[n + 1] > seg_start[n])
            seg_adapter[n_seg++] = n;

    /* runs over the grouped positions */
    char *is_long = (char *)calloc(P > 0 ? P : 1, 1);
    int32_t n_contig = 0;
    int32_t p = 0;
    while (p < P) {
        int32_t q = p + 1;
        while (q < P && ids[perm[q]] == ids[perm[p]] && perm[q] == perm[q - 1] + 1)
            ++q;
        int32_t len = q - p;
        if (min_run > 0 && len >= min_run) {
            for (int32_t u = p; u < q; ++u)
                is_long[u] = 1;
            for (int32_t off = 0; off < len; off += long_tile) {
                int32_t cnt = len - off < long_tile ? len - off : long_tile;
                if (n_contig < max_contig_tiles) {
                    int32_t *t = contig_tiles + 4 * (int64_t)n_contig;
                    t[0] = ids[perm[p]];
                    t[1] = perm[p] + off;
                    t[2] = cnt;
                    t[3] = 0;
                } else {
                    status |= 2;
                }
                ++n_contig;
            }
        }
        p = q;
    }

    /* gathered rows, segment by segment */
    int32_t n_short = 0, n_gather = 0;
    for (int32_t n = 0; n < N; ++n) {
        int32_t first = n_short;
        for (int32_t u = seg_start[n]; u < seg_start[n + 1]; ++u)
            if (!is_long[u])
                grow[n_short++] = perm[u];
        int32_t cnt_n = n_short - first;
        for (int32_t off = 0; off < cnt_n; off += rows_per_tile) {
            int32_t cnt = cnt_n - off < rows_per_tile ? cnt_n - off : rows_per_tile;
            if (n_gather < max_gather_tiles) {
                int32_t *t = gather_tiles + 4 * (int64_t)n_gather;
                t[0] = n;
                t[1] = first + off;
                t[2] = cnt;
                t[3] = 0;
            } else {
                status |= 2;
            }
            ++n_gather;
        }
    }
    free(is_long);

    counts[0] = n_seg;
    counts[1] = n_gather < max_gather_tiles ? n_gather : max_gather_tiles;
    counts[2] = n_contig < max_contig_tiles ? n_contig : max_contig_tiles;
    counts[3] = n_short;
    return status;
}

/*
 * Merged weight (page "LoRA service: multi-adapter dynamic loading", section 1:
 * a single-tenant deployment folds the adapter into the base weight,
 * W' = W + B A; the scale alpha / r of page "Multi-LoRA Serving", section 3.1),
 * in fp64:
 *   out[o][i] = W[o][i] + sign * (alpha / r) * sum_{k < r} B[o][k] * A[k][i]
 * for o < d_out, i < d_in.  W is [d_out][ld_w]; A is one adapter [r_max][d_in]
 * and B one adapter [d_out][r_max] (rank rows / columns k >= r are padding,
 * never read); out is [d_out][d_in].  Returns 0, or -1 on a bad argument.
 */
int oracle_lora_merge(int dtype, const void *W, int64_t ld_w, int32_t d_out, int32_t d_in,
                      const void *A, const void *B, int32_t r_max, int32_t r, double alpha,
                      int32_t sign, double *out)
{
    if (dtype != ORACLE_BF16 && dtype != ORACLE_FP32)
        return -1;
    if (d_out <= 0 || d_in <= 0 || ld_w < d_in || r <= 0 || r > r_max || (sign != 1 && sign != -1))
        return -1;
    double s = (double)sign * alpha / (double)r;
#pragma omp parallel for schedule(static)
    for (int32_t o = 0; o < d_out; ++o)
        for (int32_t i = 0; i < d_in; ++i) {
            double acc = 0.0;
            for (int32_t k = 0; k < r; ++k)
                acc += widen(dtype, B, (int64_t)o * r_max + k) * widen(dtype, A, (int64_t)k * d_in + i);
            out[(int64_t)o * d_in + i] = widen(dtype, W, (int64_t)o * ld_w + i) + s * acc;
        }
    return 0;
}

/* Adapter parameter count r(d + k) against the full d*k (page "Multi-LoRA
 * Serving", section 3.1, last paragraph). */
int64_t oracle_lora_param_count(int64_t d, int64_t k, int64_t r) { return r * (d + k); }

/* Adapter memory 2 * num_layers * r * hidden * dtype_bytes (page "LoRA
 * service", section 7). */
int64_t oracle_adapter_bytes(int64_t num_layers, int64_t r, int64_t hidden, int64_t dtype_bytes)
{
    return 2 * num_layers * r * hidden * dtype_bytes;
}

/* Host threads used by oracle_lora_apply (OpenMP over rows). */
#ifdef _OPENMP
#include <omp.h>
void oracle_set_threads(int n) { if (n > 0) omp_set_num_threads(n); }
int oracle_max_threads(void) { return omp_get_max_threads(); }
#else
void oracle_set_threads(int n) { (void)n; }
int oracle_max_threads(void) { return 1; }
#endif
