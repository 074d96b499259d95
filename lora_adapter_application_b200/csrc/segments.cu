// Grouping of a batch's rows by adapter id, and the tile lists the compute
// kernels walk ("group rows by adapter id", page "Multi-LoRA Serving",
// section 2 flowchart and section 3.2; LoraBatchInfo of page "LoRA hot load
// and adapter routing").
//
// A stable counting sort.  Up to SEG_SMALL_T rows one thread block does it
// all in a single launch (decode batches).  Above that:
//   seg_hist     one block per chunk of SEG_CHUNK rows: per-chunk id histogram
//   seg_scan     one block: totals -> seg_start, seg_adapter, per-chunk bases
//   seg_scatter  one warp per chunk: stable ranks with __match_any_sync
//   seg_tiles    one block: runs, contiguous tiles, gathered rows and tiles
// No block ever waits for another block: the phases are separate launches.
#include "common.cuh"

#include <climits>

namespace lora {

constexpr int SEG_THREADS = 1024;
constexpr int SEG_CHUNK = 2048;
constexpr int SEG_SMALL_T = 2048;
constexpr int SEG_HIST_THREADS = 512;

__device__ __forceinline__ int bin_of(int id, int N) { return (id >= 0 && id < N) ? id : N; }

// Exclusive prefix sum over the SEG_THREADS threads of the block.  sm: 33 ints.
__device__ int block_excl_sum(int v, int *total, int *sm) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int t = __shfl_up_sync(FULL, incl, o);
        if (lane >= o) incl += t;
    }
    if (lane == 31) sm[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int w = sm[lane];
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int t = __shfl_up_sync(FULL, wi, o);
            if (lane >= o) wi += t;
        }
        sm[lane] = wi - w;
        if (lane == 31) sm[32] = wi;
    }
    __syncthreads();
    int res = sm[warp] + incl - v;
    *total = sm[32];
    __syncthreads();
    return res;
}

// For each thread, the minimum of v over the threads after it (INT_MAX if none).
__device__ int block_excl_suffix_min(int v, int *sm) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int t = __shfl_down_sync(FULL, incl, o);
        if (lane + o < 32) incl = min(incl, t);
    }
    if (lane == 0) sm[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int wi = sm[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int t = __shfl_down_sync(FULL, wi, o);
            if (lane + o < 32) wi = min(wi, t);
        }
        sm[lane] = wi;
    }
    __syncthreads();
    int within = __shfl_down_sync(FULL, incl, 1);
    if (lane == 31) within = INT_MAX;
    int after = warp < 31 ? sm[warp + 1] : INT_MAX;
    __syncthreads();
    return min(within, after);
}

// Turn per-id counts hist[0..N] (bin N = rows without a valid id) into start
// offsets; write seg_start, seg_adapter and counts[0].  Whole block.
__device__ void seg_scan_block(int *hist, int N, int32_t *seg_start, int32_t *seg_adapter,
                               int32_t *counts, int *sm33) {
    const int tid = threadIdx.x;
    const int bpt = (N + SEG_THREADS - 1) / SEG_THREADS;
    const int lo = min(tid * bpt, N), hi = min(lo + bpt, N);
    int s = 0, nz = 0;
    for (int b = lo; b < hi; ++b) {
        s += hist[b];
        nz += hist[b] > 0;
    }
    int P, nseg;
    int pre = block_excl_sum(s, &P, sm33);
    int zpre = block_excl_sum(nz, &nseg, sm33);
    for (int b = lo; b < hi; ++b) {
        int c = hist[b];
        seg_start[b] = pre;
        hist[b] = pre;
        pre += c;
        if (c > 0) seg_adapter[zpre++] = b;
    }
    if (tid == 0) {
        seg_start[N] = P;
        hist[N] = P;
        counts[0] = nseg;
    }
}

// Stable placement of rows [lo, hi) by one warp, starting at base[bin].
__device__ void scatter_warp(const int32_t *ids, int lo, int hi, int N, int *base, int32_t *perm) {
    const int lane = threadIdx.x & 31;
    for (int i0 = lo; i0 < hi; i0 += 32) {
        const int i = i0 + lane;
        const bool v = i < hi;
        const int key = v ? bin_of(ids[i], N) : N + 1 + lane;
        const unsigned m = __match_any_sync(FULL, key);
        const int rank = __popc(m & ((1u << lane) - 1u));
        const int pos = v ? base[key] + rank : 0;
        __syncwarp();
        if (v) {
            perm[pos] = i;
            if (rank == 0) base[key] += __popc(m);
        }
        __syncwarp();
    }
}

__device__ __forceinline__ uint32_t bit_range(int a, int b) {   // bits [a, b), 0 <= a < b <= 32
    uint32_t hi = b >= 32 ? 0xffffffffu : ((1u << b) - 1u);
    return hi & ~((1u << a) - 1u);
}

struct TileOut {
    int32_t *grow;
    int4 *gather;
    int4 *contig;
    int32_t *counts;
    int32_t *status;
    int max_gather, max_contig;
    int R, min_run, LT;
};

// Runs, contiguous tiles, gathered rows and gathered tiles (see lora_meta).
// Whole block.  brkw/lngw/aux: ceil(P/32) words of shared memory each.
__device__ void dev_tiles(const int32_t *ids, const int32_t *perm, const int32_t *seg_start, int N,
                          const TileOut &o, uint32_t *brkw, uint32_t *lngw, int *aux, int *sm33) {
    const int tid = threadIdx.x;
    const int P = seg_start[N];
    const int W = (P + 31) >> 5;

    // 1. run starts: a new id, or a row that does not follow the previous one
    for (int w = tid; w < W; w += SEG_THREADS) {
        const int p0 = w * 32;
        int prev_row = -2, prev_id = -2;
        if (p0 > 0) {
            prev_row = perm[p0 - 1];
            prev_id = ids[prev_row];
        }
        uint32_t bits = 0;
        for (int b = 0; b < 32 && p0 + b < P; ++b) {
            const int row = perm[p0 + b];
            const int id = ids[row];
            if (id != prev_id || row != prev_row + 1) bits |= 1u << b;
            prev_row = row;
            prev_id = id;
        }
        brkw[w] = bits;
        lngw[w] = 0;
    }
    __syncthreads();

    // aux[w] = first run start at a position >= 32*w (P if none)
    const int wpt = (W + SEG_THREADS - 1) / SEG_THREADS;
    const int w_lo = min(tid * wpt, W), w_hi = min(w_lo + wpt, W);
    int first = INT_MAX;
    for (int w = w_lo; w < w_hi; ++w)
        if (brkw[w]) {
            first = w * 32 + __ffs(brkw[w]) - 1;
            break;
        }
    int nxt = min(block_excl_suffix_min(first, sm33), P);
    for (int w = w_hi - 1; w >= w_lo; --w) {
        if (brkw[w]) nxt = w * 32 + __ffs(brkw[w]) - 1;
        aux[w] = nxt;
    }
    __syncthreads();

    auto run_end = [&](int p) -> int {
        const int w = p >> 5, b = p & 31;
        const uint32_t rest = b == 31 ? 0u : (brkw[w] & (0xffffffffu << (b + 1)));
        if (rest) return min(w * 32 + __ffs(rest) - 1, P);
        return (w + 1 < W) ? aux[w + 1] : P;
    };

    // 2. long runs
    if (o.min_run > 0) {
        for (int w = tid; w < W; w += SEG_THREADS) {
            uint32_t bits = brkw[w];
            while (bits) {
                const int b = __ffs(bits) - 1;
                bits &= bits - 1;
                const int p = w * 32 + b, e = run_end(p);
                if (e - p >= o.min_run) {
                    for (int ww = p >> 5; ww <= (e - 1) >> 5; ++ww) {
                        const int a = max(p, ww * 32) - ww * 32, z = min(e, ww * 32 + 32) - ww * 32;
                        atomicOr(&lngw[ww], bit_range(a, z));
                    }
                }
            }
        }
    }
    __syncthreads();

    bool overflow = false;

    // 3. contiguous tiles, in position order
    int my_ct = 0;
    for (int w = w_lo; w < w_hi; ++w) {
        uint32_t bits = brkw[w] & lngw[w];
        while (bits) {
            const int b = __ffs(bits) - 1;
            bits &= bits - 1;
            const int p = w * 32 + b;
            my_ct += (run_end(p) - p + o.LT - 1) / o.LT;
        }
    }
    int n_contig;
    int cbase = block_excl_sum(my_ct, &n_contig, sm33);
    for (int w = w_lo; w < w_hi; ++w) {
        uint32_t bits = brkw[w] & lngw[w];
        while (bits) {
            const int b = __ffs(bits) - 1;
            bits &= bits - 1;
            const int p = w * 32 + b, len = run_end(p) - p;
            const int row0 = perm[p], id = ids[row0];
            for (int off = 0; off < len; off += o.LT, ++cbase) {
                if (cbase < o.max_contig)
                    o.contig[cbase] = make_int4(id, row0 + off, min(o.LT, len - off), 0);
                else
                    overflow = true;
            }
        }
    }

    // 4. gathered rows (positions outside long runs), in position order
    auto short_bits = [&](int w) -> uint32_t {
        const int rem = P - w * 32;
        const uint32_t valid = rem >= 32 ? 0xffffffffu : ((1u << rem) - 1u);
        return ~lngw[w] & valid;
    };
    int my_sh = 0;
    for (int w = w_lo; w < w_hi; ++w) my_sh += __popc(short_bits(w));
    int n_short;
    int sbase = block_excl_sum(my_sh, &n_short, sm33);
    for (int w = w_lo; w < w_hi; ++w) {
        aux[w] = sbase;
        uint32_t bits = short_bits(w);
        while (bits) {
            const int b = __ffs(bits) - 1;
            bits &= bits - 1;
            o.grow[sbase++] = perm[w * 32 + b];
        }
    }
    __syncthreads();

    // 5. gathered tiles: each id's gathered rows cut every R rows
    auto short_before = [&](int q) -> int {
        if (q >= P) return n_short;
        const int w = q >> 5, b = q & 31;
        return aux[w] + __popc(short_bits(w) & ((1u << b) - 1u));
    };
    const int spt = (N + SEG_THREADS - 1) / SEG_THREADS;
    const int n_lo = min(tid * spt, N), n_hi = min(n_lo + spt, N);
    int my_gt = 0;
    for (int n = n_lo; n < n_hi; ++n) {
        const int cnt = short_before(seg_start[n + 1]) - short_before(seg_start[n]);
        my_gt += (cnt + o.R - 1) / o.R;
    }
    int n_gather;
    int gbase = block_excl_sum(my_gt, &n_gather, sm33);
    for (int n = n_lo; n < n_hi; ++n) {
        const int g0 = short_before(seg_start[n]);
        const int cnt = short_before(seg_start[n + 1]) - g0;
        for (int off = 0; off < cnt; off += o.R, ++gbase) {
            if (gbase < o.max_gather)
                o.gather[gbase] = make_int4(n, g0 + off, min(o.R, cnt - off), 0);
            else
                overflow = true;
        }
    }
    if (overflow) atomicOr(o.status, LORA_DEV_TILE_OVERFLOW);
    if (tid == 0) {
        o.counts[1] = min(n_gather, o.max_gather);
        o.counts[2] = min(n_contig, o.max_contig);
        o.counts[3] = n_short;
    }
}

struct SegArgs {
    const int32_t *ids;
    int T, N;
    int32_t *perm, *seg_start, *seg_adapter;
    int *ws;   // [n_chunks][N+1] (multi-block path)
    TileOut out;
};

// Everything in one block (T <= SEG_SMALL_T).
__global__ void __launch_bounds__(SEG_THREADS) seg_small_kernel(SegArgs a) {
    extern __shared__ int sm[];
    int *sm33 = sm;
    int *hist = sm + 64;
    const int W = (a.T + 31) >> 5;
    uint32_t *brkw = reinterpret_cast<uint32_t *>(hist + a.N + 1);
    uint32_t *lngw = brkw + W;
    int *aux = reinterpret_cast<int *>(lngw + W);
    const int tid = threadIdx.x;

    for (int b = tid; b <= a.N; b += SEG_THREADS) hist[b] = 0;
    __syncthreads();
    bool bad = false;
    for (int i = tid; i < a.T; i += SEG_THREADS) {
        const int id = a.ids[i];
        bad |= (id < -1 || id >= a.N);
        atomicAdd(&hist[bin_of(id, a.N)], 1);
    }
    if (bad) atomicOr(a.out.status, LORA_DEV_BAD_ID);
    __syncthreads();
    seg_scan_block(hist, a.N, a.seg_start, a.seg_adapter, a.out.counts, sm33);
    __syncthreads();
    if (tid < 32) scatter_warp(a.ids, 0, a.T, a.N, hist, a.perm);
    __syncthreads();
    dev_tiles(a.ids, a.perm, a.seg_start, a.N, a.out, brkw, lngw, aux, sm33);
}

__global__ void __launch_bounds__(SEG_HIST_THREADS) seg_hist_kernel(SegArgs a) {
    extern __shared__ int hist[];
    const int c = blockIdx.x, lo = c * SEG_CHUNK, hi = min(lo + SEG_CHUNK, a.T);
    for (int b = threadIdx.x; b <= a.N; b += blockDim.x) hist[b] = 0;
    __syncthreads();
    bool bad = false;
    for (int i = lo + threadIdx.x; i < hi; i += blockDim.x) {
        const int id = a.ids[i];
        bad |= (id < -1 || id >= a.N);
        atomicAdd(&hist[bin_of(id, a.N)], 1);
    }
    if (bad) atomicOr(a.out.status, LORA_DEV_BAD_ID);
    __syncthreads();
    for (int b = threadIdx.x; b <= a.N; b += blockDim.x) a.ws[(size_t)c * (a.N + 1) + b] = hist[b];
}

__global__ void __launch_bounds__(SEG_THREADS) seg_scan_kernel(SegArgs a, int n_chunks) {
    extern __shared__ int sm[];
    int *sm33 = sm;
    int *tot = sm + 64;
    const int stride = a.N + 1;
    for (int b = threadIdx.x; b <= a.N; b += SEG_THREADS) {
        int run = 0;
        for (int c = 0; c < n_chunks; ++c) {
            const int t = a.ws[(size_t)c * stride + b];
            a.ws[(size_t)c * stride + b] = run;
            run += t;
        }
        tot[b] = run;
    }
    __syncthreads();
    seg_scan_block(tot, a.N, a.seg_start, a.seg_adapter, a.out.counts, sm33);
    __syncthreads();
    for (int b = threadIdx.x; b <= a.N; b += SEG_THREADS) {
        const int base = tot[b];
        for (int c = 0; c < n_chunks; ++c) a.ws[(size_t)c * stride + b] += base;
    }
}

__global__ void __launch_bounds__(32) seg_scatter_kernel(SegArgs a) {
    extern __shared__ int base[];
    const int c = blockIdx.x, lo = c * SEG_CHUNK, hi = min(lo + SEG_CHUNK, a.T);
    for (int b = threadIdx.x; b <= a.N; b += 32) base[b] = a.ws[(size_t)c * (a.N + 1) + b];
    __syncwarp();
    scatter_warp(a.ids, lo, hi, a.N, base, a.perm);
}

__global__ void __launch_bounds__(SEG_THREADS) seg_tiles_kernel(SegArgs a) {
    extern __shared__ int sm[];
    int *sm33 = sm;
    const int W = (a.T + 31) >> 5;
    uint32_t *brkw = reinterpret_cast<uint32_t *>(sm + 64);
    uint32_t *lngw = brkw + W;
    int *aux = reinterpret_cast<int *>(lngw + W);
    dev_tiles(a.ids, a.perm, a.seg_start, a.N, a.out, brkw, lngw, aux, sm33);
}

size_t segments_scratch_bytes(int T, int N) {
    if (T <= SEG_SMALL_T) return 0;
    const size_t n_chunks = (T + SEG_CHUNK - 1) / SEG_CHUNK;
    return n_chunks * (size_t)(N + 1) * sizeof(int);
}

int launch_build_segments(const int32_t *ids, const lora_meta *m, void *scratch,
                          size_t scratch_bytes, int32_t *status, cudaStream_t st) {
    SegArgs a;
    a.ids = ids;
    a.T = m->T;
    a.N = m->N;
    a.perm = m->perm;
    a.seg_start = m->seg_start;
    a.seg_adapter = m->seg_adapter;
    a.ws = static_cast<int *>(scratch);
    a.out.grow = m->grow;
    a.out.gather = reinterpret_cast<int4 *>(m->gather_tiles);
    a.out.contig = reinterpret_cast<int4 *>(m->contig_tiles);
    a.out.counts = m->counts;
    a.out.status = status;
    a.out.max_gather = m->max_gather_tiles;
    a.out.max_contig = m->max_contig_tiles;
    a.out.R = m->rows_per_tile;
    a.out.min_run = m->min_run;
    a.out.LT = m->long_tile;

    const int W = (a.T + 31) / 32;
    if (a.T <= SEG_SMALL_T) {
        const size_t smem = (64 + (size_t)a.N + 1 + 3 * (size_t)W) * sizeof(int);
        if (smem > 48 * 1024)
            cudaFuncSetAttribute(seg_small_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem);
        seg_small_kernel<<<1, SEG_THREADS, smem, st>>>(a);
    } else {
        if (scratch == nullptr || scratch_bytes < segments_scratch_bytes(a.T, a.N))
            return LORA_ERR_WORKSPACE;
        const int n_chunks = (a.T + SEG_CHUNK - 1) / SEG_CHUNK;
        const size_t bins = (size_t)a.N + 1;
        seg_hist_kernel<<<n_chunks, SEG_HIST_THREADS, bins * sizeof(int), st>>>(a);
        const size_t scan_smem = (64 + bins) * sizeof(int);
        seg_scan_kernel<<<1, SEG_THREADS, scan_smem, st>>>(a, n_chunks);
        seg_scatter_kernel<<<n_chunks, 32, bins * sizeof(int), st>>>(a);
        const size_t tile_smem = (64 + 3 * (size_t)W) * sizeof(int);
        if (tile_smem > 48 * 1024)
            cudaFuncSetAttribute(seg_tiles_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)tile_smem);
        seg_tiles_kernel<<<1, SEG_THREADS, tile_smem, st>>>(a);
    }
    return cudaGetLastError() == cudaSuccess ? LORA_OK : LORA_ERR_CUDA;
}

}  // namespace lora
