// Grouping of a batch's rows by adapter id, and the tile lists the compute
// kernels walk ("group rows by adapter id", page "Multi-LoRA Serving",
// section 2 flowchart and section 3.2; LoraBatchInfo of page "LoRA hot load
// and adapter routing").
//
// A stable counting sort.  One thread block does it all in a single launch
// up to SEG_SMALL_T rows, or up to SEG_ONE_BLOCK_T rows when N < 1024 (then at
// least 8 warps rank rows in parallel; measured on B200 at 3000-8192 rows:
// 15-26 us in one block against 33-40 us in seven launches).  Above that:
//   seg_hist     one block per chunk of SEG_CHUNK rows: per-chunk id histogram
//   seg_scan     one block, a warp per id: chunk offsets by warp scans; totals
//                -> seg_start, seg_adapter
//   seg_scatter  one block per chunk: every warp ranks its share of the rows
//   seg_runs     one block per TW_WORDS x 32 positions: run starts as bits,
//                the block's first and last run start
//   seg_long     per block: runs through its positions (neighbours from the
//                other blocks' first / last starts), long-run bits, counts of
//                contiguous tiles and gathered rows
//   seg_emit     per block: contiguous tiles, gathered rows, per-word offsets
//   seg_gtiles   one block: each id's gathered rows cut into tiles
// No block ever waits for another block: the phases are separate launches.
#include "kernels.cuh"

#include <climits>

namespace lora {

constexpr int SEG_THREADS = 1024;
constexpr int SEG_CHUNK = 2048;
constexpr int SEG_SMALL_T = 2048;
constexpr int SEG_ONE_BLOCK_T = 8192, SEG_ONE_BLOCK_N = 1023;

// The whole grouping in one block (shared memory only, no scratch)?
__host__ __device__ constexpr bool one_block(int T, int N) {
    return T <= SEG_SMALL_T || (T <= SEG_ONE_BLOCK_T && N <= SEG_ONE_BLOCK_N);
}
constexpr int SEG_HIST_THREADS = 512;
// ints of scan scratch in front of a kernel's other shared arrays (33 long longs)
constexpr int SEG_SCAN_WORDS = 80;

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

// block_excl_sum for 64-bit values.  sm: 33 long longs.
__device__ long long block_excl_sum64(long long v, long long *total, long long *sm) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    long long incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        long long t = __shfl_up_sync(FULL, incl, o);
        if (lane >= o) incl += t;
    }
    if (lane == 31) sm[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        long long w = sm[lane];
        long long wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            long long t = __shfl_up_sync(FULL, wi, o);
            if (lane >= o) wi += t;
        }
        sm[lane] = wi - w;
        if (lane == 31) sm[32] = wi;
    }
    __syncthreads();
    long long res = sm[warp] + incl - v;
    *total = sm[32];
    __syncthreads();
    return res;
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
    // one block scan for both prefix sums: rows (high word) and non-empty ids (low word)
    long long tot2;
    const long long pre2 = block_excl_sum64(((long long)s << 32) | nz, &tot2, reinterpret_cast<long long *>(sm33));
    const int P = (int)(tot2 >> 32), nseg = (int)(tot2 & 0xffffffffll);
    int pre = (int)(pre2 >> 32), zpre = (int)(pre2 & 0xffffffffll);
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

// Lanes of the warp whose key equals this lane's key.  One ballot per key bit
// (keys < 2^nbits); a hardware match instruction is far slower here.
__device__ __forceinline__ unsigned equal_lanes(int key, int nbits) {
    unsigned eq = FULL;
    for (int b = 0; b < nbits; ++b) {
        const unsigned m = __ballot_sync(FULL, (key >> b) & 1);
        eq &= ((key >> b) & 1) ? m : ~m;
    }
    return eq;
}

// Stable placement of rows [lo, hi) by one warp, starting at base[bin].  Also
// records, for every placed row, whether it starts a run: a row starts a run
// when the row before it (in row order) has another id.  Because the grouping
// is stable, that is the same as "the previous position holds another id or a
// row that is not the previous row".
__device__ void scatter_warp(const int32_t *ids, int lo, int hi, int N, int *base, int32_t *perm,
                             uint8_t *brkb) {
    const int lane = threadIdx.x & 31;
    const int nbits = 32 - __clz(N + 1 + 32);
    for (int i0 = lo; i0 < hi; i0 += 32) {
        const int i = i0 + lane;
        const bool v = i < hi;
        const int id = v ? ids[i] : 0;
        int prev = __shfl_up_sync(FULL, id, 1);
        if (lane == 0) prev = i > 0 ? ids[i - 1] : INT_MIN;
        const int key = v ? bin_of(id, N) : N + 1 + lane;
        const unsigned m = equal_lanes(key, nbits);
        const int rank = __popc(m & ((1u << lane) - 1u));
        const int pos = v ? base[key] + rank : 0;
        __syncwarp();
        if (v) {
            perm[pos] = i;
            if (key < N) brkb[pos] = (i == 0 || prev != id) ? 1 : 0;
            if (rank == 0) base[key] += __popc(m);
        }
        __syncwarp();
    }
}

// Exclusive prefix over the block's warps of one value per warp (taken from
// lane 0), and the total.  All threads of the block call it.  wsum: 33 ints.
__device__ int warp_excl_scan(int v, int *total, int *wsum) {
    constexpr int NW = SEG_THREADS / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) wsum[warp] = v;
    __syncthreads();
    if (warp == 0) {
        const int x = lane < NW ? wsum[lane] : 0;
        int incl = x;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(FULL, incl, o);
            if (lane >= o) incl += t;
        }
        wsum[lane] = incl - x;
        if (lane == 31) wsum[32] = incl;
    }
    __syncthreads();
    const int r = wsum[warp];
    *total = wsum[32];
    __syncthreads();
    return r;
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

// Shared-memory words used by dev_tiles: 4 arrays of ceil(P/32) words plus 64.
__host__ __device__ constexpr int tiles_smem_words(int T) { return 64 + 4 * ((T + 31) / 32); }

// Runs, contiguous tiles, gathered rows and gathered tiles (see lora_meta).
// Whole block; every loop over positions runs one position per lane and packs
// flags into 32-bit words with ballots, so no thread walks positions serially.
//   perm, ids  : global or shared
//   brkb[p]    : 1 if position p starts a run (p < P)
//   sm         : tiles_smem_words(T) words of shared memory
__device__ void dev_tiles(const int32_t *ids, const int32_t *perm, const uint8_t *brkb,
                          const int32_t *seg_start, int N, const TileOut &o, int *sm) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int NW = SEG_THREADS / 32;
    const int P = seg_start[N];
    const int W = (P + 31) >> 5;
    int *wsum = sm;                                   // 64 ints: per-warp values
    uint32_t *brkw = reinterpret_cast<uint32_t *>(sm + 64);
    uint32_t *lngw = brkw + W;
    int *nxt = reinterpret_cast<int *>(lngw + W);      // first run start at a position >= 32w (P if none)
    int *prv = nxt + W;                                // last run start at a position < 32w (-1 if none)
    const uint32_t lt = (1u << lane) - 1u;

    // word ranges per warp, contiguous so that per-warp order is position order
    const int wpw = (W + NW - 1) / NW;
    const int wl = min(warp * wpw, W), wh = min(wl + wpw, W);
    bool overflow = false;

    // no contiguous tiles: every valid position is gathered, in position order
    const bool all_gathered = o.min_run <= 0;
    if (all_gathered) {
        if (tid == 0) o.counts[2] = 0;
    } else {
    // 1. pack run starts
    for (int w = warp; w < W; w += NW) {
        const int p = w * 32 + lane;
        const uint32_t word = __ballot_sync(FULL, p < P && brkb[p]);
        if (lane == 0) brkw[w] = word;
    }
    __syncthreads();

    // 2. nxt[] (suffix) and prv[] (prefix) over words
    {
        int first = INT_MAX, last = -1;
        for (int w = wl + lane; w < wh; w += 32) {
            const uint32_t b = brkw[w];
            if (b) {
                first = min(first, w * 32 + __ffs(b) - 1);
                last = max(last, w * 32 + 31 - __clz(b));
            }
        }
#pragma unroll
        for (int o2 = 16; o2 > 0; o2 >>= 1) {
            first = min(first, __shfl_xor_sync(FULL, first, o2));
            last = max(last, __shfl_xor_sync(FULL, last, o2));
        }
        if (lane == 0) {
            wsum[warp] = first;
            wsum[32 + warp] = last;
        }
        __syncthreads();
        if (warp == 0) {   // exclusive suffix-min of firsts, exclusive prefix-max of lasts
            const int f = wsum[lane], l = wsum[32 + lane];
            int sf = f, pl = l;
#pragma unroll
            for (int o2 = 1; o2 < 32; o2 <<= 1) {
                const int tf = __shfl_down_sync(FULL, sf, o2);
                if (lane + o2 < 32) sf = min(sf, tf);
                const int tl = __shfl_up_sync(FULL, pl, o2);
                if (lane >= o2) pl = max(pl, tl);
            }
            int after = __shfl_down_sync(FULL, sf, 1);
            if (lane == 31) after = INT_MAX;
            int before = __shfl_up_sync(FULL, pl, 1);
            if (lane == 0) before = -1;
            __syncwarp();
            wsum[lane] = min(after, P);
            wsum[32 + lane] = before;
        }
        __syncthreads();
        const int after = wsum[warp], before = wsum[32 + warp];
        // backward over my words, 32 at a time: suffix minimum of first starts
        int carry = after;
        const int nchunk = (wh - wl + 31) / 32;
        for (int c = nchunk - 1; c >= 0; --c) {
            const int w = wl + c * 32 + lane;
            int f = INT_MAX;
            if (w < wh && brkw[w]) f = w * 32 + __ffs(brkw[w]) - 1;
            int incl = f;
#pragma unroll
            for (int o2 = 1; o2 < 32; o2 <<= 1) {
                const int t = __shfl_down_sync(FULL, incl, o2);
                if (lane + o2 < 32) incl = min(incl, t);
            }
            if (w < wh) nxt[w] = min(incl, carry);
            carry = min(carry, __shfl_sync(FULL, incl, 0));
        }
        // forward: prefix maximum of last starts (strictly before the word)
        carry = before;
        for (int c = 0; c < nchunk; ++c) {
            const int w = wl + c * 32 + lane;
            int l = -1;
            if (w < wh && brkw[w]) l = w * 32 + 31 - __clz(brkw[w]);
            int incl = l;
#pragma unroll
            for (int o2 = 1; o2 < 32; o2 <<= 1) {
                const int t = __shfl_up_sync(FULL, incl, o2);
                if (lane >= o2) incl = max(incl, t);
            }
            int excl = __shfl_up_sync(FULL, incl, 1);
            if (lane == 0) excl = -1;
            if (w < wh) prv[w] = max(carry, excl);
            carry = max(carry, __shfl_sync(FULL, incl, 31));
        }
    }
    __syncthreads();

    auto run_end = [&](int p) -> int {   // first run start after p, or P
        const int w = p >> 5, b = p & 31;
        const uint32_t rest = b == 31 ? 0u : (brkw[w] & (0xffffffffu << (b + 1)));
        if (rest) return w * 32 + __ffs(rest) - 1;
        return (w + 1 < W) ? nxt[w + 1] : P;
    };
    auto run_start = [&](int p) -> int {   // last run start at or before p
        const int w = p >> 5, b = p & 31;
        const uint32_t upto = brkw[w] & (b == 31 ? 0xffffffffu : ((2u << b) - 1u));
        if (upto) return w * 32 + 31 - __clz(upto);
        return prv[w];
    };

    // 3. long positions: the run through the position has at least min_run rows
    for (int w = warp; w < W; w += NW) {
        const int p = w * 32 + lane;
        bool lg = false;
        if (o.min_run > 0 && p < P) lg = run_end(p) - run_start(p) >= o.min_run;
        const uint32_t word = __ballot_sync(FULL, lg);
        if (lane == 0) lngw[w] = word;
    }
    __syncthreads();

    // 4. contiguous tiles: long runs in position order, cut every LT rows
    {
        int cnt = 0;
        for (int w = wl; w < wh; ++w) {
            const int p = w * 32 + lane;
            int k = 0;
            if (((brkw[w] & lngw[w]) >> lane) & 1u) k = (run_end(p) - p + o.LT - 1) / o.LT;
            cnt += k;
        }
#pragma unroll
        for (int o2 = 16; o2 > 0; o2 >>= 1) cnt += __shfl_xor_sync(FULL, cnt, o2);
        int n_contig;
        int base = warp_excl_scan(cnt, &n_contig, wsum);
        for (int w = wl; w < wh; ++w) {
            const int p = w * 32 + lane;
            int len = 0, k = 0;
            if (((brkw[w] & lngw[w]) >> lane) & 1u) {
                len = run_end(p) - p;
                k = (len + o.LT - 1) / o.LT;
            }
            int incl = k;
#pragma unroll
            for (int o2 = 1; o2 < 32; o2 <<= 1) {
                const int t = __shfl_up_sync(FULL, incl, o2);
                if (lane >= o2) incl += t;
            }
            int idx = base + incl - k;
            if (k) {
                const int row0 = perm[p], id = ids[row0];
                for (int off = 0; off < len; off += o.LT, ++idx) {
                    if (idx < o.max_contig)
                        o.contig[idx] = make_int4(id, row0 + off, min(o.LT, len - off), 0);
                    else
                        overflow = true;
                }
            }
            base += __shfl_sync(FULL, incl, 31);
        }
        if (tid == 0) o.counts[2] = min(n_contig, o.max_contig);
    }
    __syncthreads();
    }   // min_run > 0

    // 5. gathered rows: positions outside long runs, in position order
    int *gpre = prv;   // reused: gathered rows before word w
    auto short_bits = [&](int w) -> uint32_t {
        const int rem = P - w * 32;
        const uint32_t valid = rem >= 32 ? 0xffffffffu : ((1u << rem) - 1u);
        return ~lngw[w] & valid;
    };
    int n_short;
    if (all_gathered) {   // the gathered rows are perm[0:P]
        for (int p = tid; p < P; p += SEG_THREADS) o.grow[p] = perm[p];
        n_short = P;
    } else {
        int cnt = 0;
        for (int w = wl + lane; w < wh; w += 32) cnt += __popc(short_bits(w));
#pragma unroll
        for (int o2 = 16; o2 > 0; o2 >>= 1) cnt += __shfl_xor_sync(FULL, cnt, o2);
        int base = warp_excl_scan(cnt, &n_short, wsum);
        for (int w = wl; w < wh; ++w) {
            const uint32_t bits = short_bits(w);
            if ((bits >> lane) & 1u) o.grow[base + __popc(bits & lt)] = perm[w * 32 + lane];
            if (lane == 0) gpre[w] = base;
            base += __popc(bits);
        }
        __syncthreads();
    }

    // 6. gathered tiles: each id's gathered rows cut every R rows
    auto short_before = [&](int q) -> int {
        if (all_gathered) return min(q, P);
        if (q >= P) return n_short;
        const int w = q >> 5, b = q & 31;
        return gpre[w] + __popc(short_bits(w) & ((1u << b) - 1u));
    };
    {
        const int spt = (N + SEG_THREADS - 1) / SEG_THREADS;
        const int n_lo = min(tid * spt, N), n_hi = min(n_lo + spt, N);
        int my_gt = 0;
        for (int n = n_lo; n < n_hi; ++n) {
            const int c = short_before(seg_start[n + 1]) - short_before(seg_start[n]);
            my_gt += (c + o.R - 1) / o.R;
        }
        int n_gather;
        int gbase = block_excl_sum(my_gt, &n_gather, wsum);
        for (int n = n_lo; n < n_hi; ++n) {
            const int g0 = short_before(seg_start[n]);
            const int c = short_before(seg_start[n + 1]) - g0;
            for (int off = 0; off < c; off += o.R, ++gbase) {
                if (gbase < o.max_gather)
                    o.gather[gbase] = make_int4(n, g0 + off, min(o.R, c - off), 0);
                else
                    overflow = true;
            }
        }
        if (tid == 0) {
            o.counts[1] = min(n_gather, o.max_gather);
            o.counts[3] = n_short;
        }
    }
    if (overflow) atomicOr(o.status, LORA_DEV_TILE_OVERFLOW);
}

struct SegArgs {
    const int32_t *ids;
    int T, N;
    int32_t *perm, *seg_start, *seg_adapter;
    int *ws;          // [n_chunks][N+1] (multi-block path)
    uint8_t *brkb;    // [T]            (multi-block path)
    // multi-block tile passes: per word of 32 positions, and per block of TW_WORDS words
    uint32_t *brkw;   // [W] run-start bits
    uint32_t *lngw;   // [W] long-run bits
    int *gpre;        // [W] gathered rows before word w
    int4 *blk;        // [B] {first run start, last run start, contiguous tiles, gathered rows}
    int W, B;
    TileOut out;
};

constexpr int TW_WORDS = 64;      // words per block of the multi-block tile passes
constexpr int TW_THREADS = 256;   // 8 warps x 8 words

// Warps that rank rows in parallel: each keeps a private count per id, so the
// counts must fit the shared-memory budget.
__host__ __device__ constexpr int rank_warps(int N) {
    return (8192 / (N + 1)) >= 32 ? 32 : ((8192 / (N + 1)) < 1 ? 1 : 8192 / (N + 1));
}

// Stable placement of rows [lo, hi) by up to 32 warps.  Warp w ranks the rows
// [lo + w*rpw, lo + (w+1)*rpw); hw[w][b] holds its private count of id b on
// entry, and is turned into its first position (base[b] plus the counts of
// warps before it).  Whole block.
__device__ void scatter_block(const int32_t *ids, int lo, int hi, int N, const int *base, int *hw,
                              int nwr, int32_t *perm, uint8_t *brkb) {
    const int tid = threadIdx.x, warp = tid >> 5;
    const int rpw = (hi - lo + nwr - 1) / nwr;
    for (int b = tid; b <= N; b += blockDim.x) {
        int run = base[b];
        for (int w = 0; w < nwr; ++w) {
            const int c = hw[w * (N + 1) + b];
            hw[w * (N + 1) + b] = run;
            run += c;
        }
    }
    __syncthreads();
    if (warp < nwr) {
        const int wl = lo + warp * rpw, wh = min(wl + rpw, hi);
        if (wl < wh) scatter_warp(ids, wl, wh, N, hw + warp * (N + 1), perm, brkb);
    }
}

// Per-warp id counts of rows [lo, hi) into hw[w][*] (zeroed here).  Whole block.
__device__ bool count_block(const int32_t *ids, int lo, int hi, int N, int *hw, int nwr) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int e = tid; e < nwr * (N + 1); e += blockDim.x) hw[e] = 0;
    __syncthreads();
    bool bad = false;
    if (warp < nwr) {
        const int rpw = (hi - lo + nwr - 1) / nwr;
        const int wl = lo + warp * rpw, wh = min(wl + rpw, hi);
        for (int i = wl + lane; i < wh; i += 32) {
            const int id = ids[i];
            bad |= (id < -1 || id >= N);
            atomicAdd(&hw[warp * (N + 1) + bin_of(id, N)], 1);
        }
    }
    __syncthreads();
    return bad;
}

// Everything in one block (T <= SEG_SMALL_T); ids, perm and the run starts
// stay in shared memory.
__global__ void __launch_bounds__(SEG_THREADS) seg_small_kernel(SegArgs a) {
    extern __shared__ int sm[];
    int *sm33 = sm;
    // ranking warps: at most one per 32 rows (each per-id loop below walks them)
    const int nwr = min(rank_warps(a.N), max(1, (a.T + 31) / 32));
    int *hist = sm + SEG_SCAN_WORDS;                      // N+1
    int *hw = hist + ((a.N + 1 + 3) & ~3);                // nwr * (N+1)
    int *ids_s = hw + ((nwr * (a.N + 1) + 3) & ~3);       // T
    int *perm_s = ids_s + a.T;                            // T
    int *tsm = perm_s + a.T;                              // tiles_smem_words(T)
    uint8_t *brk_s = reinterpret_cast<uint8_t *>(tsm + tiles_smem_words(a.T));   // T bytes
    const int tid = threadIdx.x;

    for (int i = tid; i < a.T; i += SEG_THREADS) ids_s[i] = a.ids[i];
    __syncthreads();
    if (count_block(ids_s, 0, a.T, a.N, hw, nwr)) atomicOr(a.out.status, LORA_DEV_BAD_ID);
    for (int b = tid; b <= a.N; b += SEG_THREADS) {
        int t = 0;
        for (int w = 0; w < nwr; ++w) t += hw[w * (a.N + 1) + b];
        hist[b] = t;
    }
    __syncthreads();
    seg_scan_block(hist, a.N, a.seg_start, a.seg_adapter, a.out.counts, sm33);
    __syncthreads();
    scatter_block(ids_s, 0, a.T, a.N, hist, hw, nwr, perm_s, brk_s);
    __syncthreads();
    for (int i = tid; i < a.T; i += SEG_THREADS) a.perm[i] = perm_s[i];
    // hist holds seg_start[0..N] (scan above, read-only since): the tile pass reads
    // it from shared memory instead of the global copy this block just wrote
    dev_tiles(ids_s, perm_s, brk_s, hist, a.N, a.out, tsm);
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
    int *tot = sm + SEG_SCAN_WORDS;
    const int stride = a.N + 1, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    // per id: exclusive offsets of the chunks (chunk order), 32 chunks per warp step
    for (int b = warp; b <= a.N; b += SEG_THREADS / 32) {
        int carry = 0;
        for (int c0 = 0; c0 < n_chunks; c0 += 32) {
            const int c = c0 + lane;
            const int v = c < n_chunks ? a.ws[(size_t)c * stride + b] : 0;
            int incl = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(FULL, incl, o);
                if (lane >= o) incl += t;
            }
            if (c < n_chunks) a.ws[(size_t)c * stride + b] = carry + incl - v;
            carry += __shfl_sync(FULL, incl, 31);
        }
        if (lane == 0) tot[b] = carry;
    }
    __syncthreads();
    seg_scan_block(tot, a.N, a.seg_start, a.seg_adapter, a.out.counts, sm33);
}

__global__ void __launch_bounds__(SEG_THREADS) seg_scatter_kernel(SegArgs a) {
    extern __shared__ int sm[];
    const int nwr = rank_warps(a.N);
    int *base = sm;                                   // N+1
    int *hw = sm + ((a.N + 1 + 3) & ~3);              // nwr * (N+1)
    const int c = blockIdx.x, lo = c * SEG_CHUNK, hi = min(lo + SEG_CHUNK, a.T);
    for (int b = threadIdx.x; b <= a.N; b += SEG_THREADS)   // id start + rows of earlier chunks
        base[b] = a.seg_start[b] + a.ws[(size_t)c * (a.N + 1) + b];
    count_block(a.ids, lo, hi, a.N, hw, nwr);
    scatter_block(a.ids, lo, hi, a.N, base, hw, nwr, a.perm, a.brkb);
}

// ---------------------------------------------------------------- multi-block tile passes
// Block b covers words [b*TW_WORDS, (b+1)*TW_WORDS) of the P valid positions;
// warp w of a block takes TW_WORDS/8 consecutive words, one word (32
// positions, one per lane) at a time, so per-warp order is position order.

// Sum / min / max of one int per thread over a TW_THREADS block.  sm: 8 ints.
template <class Op>
__device__ int tw_reduce(int v, int *sm, Op op) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = op(v, __shfl_xor_sync(FULL, v, o));
    __syncthreads();
    if (lane == 0) sm[warp] = v;
    __syncthreads();
    v = sm[0];
    for (int w = 1; w < TW_THREADS / 32; ++w) v = op(v, sm[w]);
    return v;
}

__global__ void __launch_bounds__(TW_THREADS) seg_runs_kernel(SegArgs a) {
    __shared__ int red[8];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int P = a.seg_start[a.N];
    int first = INT_MAX, last = -1;
    for (int i = 0; i < TW_WORDS / 8; ++i) {
        const int w = blockIdx.x * TW_WORDS + warp * (TW_WORDS / 8) + i;
        if (w >= a.W) break;
        const int p = w * 32 + lane;
        const uint32_t word = __ballot_sync(FULL, p < P && a.brkb[p]);
        if (lane == 0) a.brkw[w] = word;
        if (word) {
            first = min(first, w * 32 + __ffs(word) - 1);
            last = max(last, w * 32 + 31 - __clz(word));
        }
    }
    first = tw_reduce(first, red, [](int x, int y) { return min(x, y); });
    last = tw_reduce(last, red, [](int x, int y) { return max(x, y); });
    if (threadIdx.x == 0) a.blk[blockIdx.x] = make_int4(first, last, 0, 0);
}

// Run bits of this block's words plus the neighbouring runs outside the block.
struct RunWords {
    uint32_t bw[TW_WORDS];
    int nx[TW_WORDS + 1];    // first run start at a position >= 32 (w0 + i)
    int pv[TW_WORDS];        // last run start at a position < 32 (w0 + i)
};

// Fills rw for block blockIdx.x (whole block).  red: 8 ints.
__device__ void load_run_words(const SegArgs &a, int P, RunWords &rw, int *red) {
    const int tid = threadIdx.x, w0 = blockIdx.x * TW_WORDS;
    // first start after this block and last start before it, from the block table
    int after = INT_MAX, before = -1;
    for (int b = tid; b < a.B; b += TW_THREADS) {
        const int4 e = a.blk[b];
        if (b > (int)blockIdx.x) after = min(after, e.x);
        if (b < (int)blockIdx.x) before = max(before, e.y);
    }
    after = tw_reduce(after, red, [](int x, int y) { return min(x, y); });
    before = tw_reduce(before, red, [](int x, int y) { return max(x, y); });
    for (int i = tid; i < TW_WORDS; i += TW_THREADS) rw.bw[i] = (w0 + i < a.W) ? a.brkw[w0 + i] : 0u;
    __syncthreads();
    if (tid == 0) {   // suffix minimum of first starts, prefix maximum of last starts (64 steps)
        int nx = min(after, P);
        rw.nx[TW_WORDS] = nx;
        for (int i = TW_WORDS - 1; i >= 0; --i) {
            if (rw.bw[i]) nx = (w0 + i) * 32 + __ffs(rw.bw[i]) - 1;
            rw.nx[i] = nx;
        }
        int pv = before;
        for (int i = 0; i < TW_WORDS; ++i) {
            rw.pv[i] = pv;
            if (rw.bw[i]) pv = (w0 + i) * 32 + 31 - __clz(rw.bw[i]);
        }
    }
    __syncthreads();
}

__device__ __forceinline__ int rw_run_end(const RunWords &rw, int w0, int p) {   // first start after p
    const int i = (p >> 5) - w0, b = p & 31;
    const uint32_t rest = b == 31 ? 0u : (rw.bw[i] & (0xffffffffu << (b + 1)));
    return rest ? (p & ~31) + __ffs(rest) - 1 : rw.nx[i + 1];
}
__device__ __forceinline__ int rw_run_start(const RunWords &rw, int w0, int p) {   // last start <= p
    const int i = (p >> 5) - w0, b = p & 31;
    const uint32_t upto = rw.bw[i] & (b == 31 ? 0xffffffffu : ((2u << b) - 1u));
    return upto ? (p & ~31) + 31 - __clz(upto) : rw.pv[i];
}

__global__ void __launch_bounds__(TW_THREADS) seg_long_kernel(SegArgs a) {
    __shared__ RunWords rw;
    __shared__ int red[8];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int P = a.seg_start[a.N], w0 = blockIdx.x * TW_WORDS;
    load_run_words(a, P, rw, red);
    int tiles = 0, shorts = 0;
    for (int i = 0; i < TW_WORDS / 8; ++i) {
        const int li = warp * (TW_WORDS / 8) + i, w = w0 + li;
        if (w >= a.W) break;
        const int p = w * 32 + lane;
        bool lg = false;
        int k = 0;
        if (p < P) {
            const int e = rw_run_end(rw, w0, p);
            lg = a.out.min_run > 0 && e - rw_run_start(rw, w0, p) >= a.out.min_run;
            if (lg && ((rw.bw[li] >> lane) & 1u)) k = (e - p + a.out.LT - 1) / a.out.LT;
        }
        const uint32_t word = __ballot_sync(FULL, lg);
        if (lane == 0) a.lngw[w] = word;
        tiles += k;
        shorts += (p < P && !lg) ? 1 : 0;
    }
    tiles = tw_reduce(tiles, red, [](int x, int y) { return x + y; });
    shorts = tw_reduce(shorts, red, [](int x, int y) { return x + y; });
    if (threadIdx.x == 0) {
        a.blk[blockIdx.x].z = tiles;
        a.blk[blockIdx.x].w = shorts;
    }
}

__global__ void __launch_bounds__(TW_THREADS) seg_emit_kernel(SegArgs a) {
    __shared__ RunWords rw;
    __shared__ int red[8];
    __shared__ int wt[8], wsh[8];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int P = a.seg_start[a.N], w0 = blockIdx.x * TW_WORDS;
    const uint32_t lt = (1u << lane) - 1u;
    // tiles and gathered rows of the blocks before this one
    int tb = 0, sb = 0;
    for (int b = tid; b < (int)blockIdx.x; b += TW_THREADS) {
        const int4 e = a.blk[b];
        tb += e.z;
        sb += e.w;
    }
    tb = tw_reduce(tb, red, [](int x, int y) { return x + y; });
    sb = tw_reduce(sb, red, [](int x, int y) { return x + y; });
    load_run_words(a, P, rw, red);
    // per-warp totals (its words are consecutive), then the warp's base
    int wtiles = 0, wshort = 0;
    for (int i = 0; i < TW_WORDS / 8; ++i) {
        const int li = warp * (TW_WORDS / 8) + i, w = w0 + li;
        if (w >= a.W) break;
        const int p = w * 32 + lane;
        const uint32_t lw = a.lngw[w];
        if (p < P && ((rw.bw[li] & lw) >> lane) & 1u)
            wtiles += (rw_run_end(rw, w0, p) - p + a.out.LT - 1) / a.out.LT;
        if (p < P && !((lw >> lane) & 1u)) ++wshort;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        wtiles += __shfl_xor_sync(FULL, wtiles, o);
        wshort += __shfl_xor_sync(FULL, wshort, o);
    }
    if (lane == 0) {
        wt[warp] = wtiles;
        wsh[warp] = wshort;
    }
    __syncthreads();
    int tbase = tb, sbase = sb;
    for (int v = 0; v < warp; ++v) {
        tbase += wt[v];
        sbase += wsh[v];
    }
    bool overflow = false;
    for (int i = 0; i < TW_WORDS / 8; ++i) {
        const int li = warp * (TW_WORDS / 8) + i, w = w0 + li;
        if (w >= a.W) break;
        const int p = w * 32 + lane;
        const uint32_t lw = a.lngw[w];
        const uint32_t valid = P - w * 32 >= 32 ? 0xffffffffu : (P > w * 32 ? ((1u << (P - w * 32)) - 1u) : 0u);
        // contiguous tiles of the long runs starting in this word
        int len = 0, k = 0;
        if (((rw.bw[li] & lw & valid) >> lane) & 1u) {
            len = rw_run_end(rw, w0, p) - p;
            k = (len + a.out.LT - 1) / a.out.LT;
        }
        int incl = k;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(FULL, incl, o);
            if (lane >= o) incl += t;
        }
        int idx = tbase + incl - k;
        if (k) {
            const int row0 = a.perm[p], id = a.ids[row0];
            for (int off = 0; off < len; off += a.out.LT, ++idx) {
                if (idx < a.out.max_contig)
                    a.out.contig[idx] = make_int4(id, row0 + off, min(a.out.LT, len - off), 0);
                else
                    overflow = true;
            }
        }
        tbase += __shfl_sync(FULL, incl, 31);
        // gathered rows
        const uint32_t sbits = ~lw & valid;
        if ((sbits >> lane) & 1u) a.out.grow[sbase + __popc(sbits & lt)] = a.perm[p];
        if (lane == 0) a.gpre[w] = sbase;
        sbase += __popc(sbits);
    }
    if (overflow) atomicOr(a.out.status, LORA_DEV_TILE_OVERFLOW);
}

__global__ void __launch_bounds__(SEG_THREADS) seg_gtiles_kernel(SegArgs a) {
    __shared__ int sm33[33];
    const int tid = threadIdx.x;
    const int P = a.seg_start[a.N];
    int n_contig = 0, n_short = 0;
    for (int b = 0; b < a.B; ++b) {   // the block table is small (T / 2048 entries)
        const int4 e = a.blk[b];
        n_contig += e.z;
        n_short += e.w;
    }
    auto short_before = [&](int q) -> int {
        if (q >= P) return n_short;
        const int w = q >> 5, bit = q & 31;
        const int rem = P - w * 32;
        const uint32_t valid = rem >= 32 ? 0xffffffffu : ((1u << rem) - 1u);
        return a.gpre[w] + __popc(~a.lngw[w] & valid & ((1u << bit) - 1u));
    };
    const int spt = (a.N + SEG_THREADS - 1) / SEG_THREADS;
    const int n_lo = min(tid * spt, a.N), n_hi = min(n_lo + spt, a.N);
    int my_gt = 0;
    for (int n = n_lo; n < n_hi; ++n) {
        const int c = short_before(a.seg_start[n + 1]) - short_before(a.seg_start[n]);
        my_gt += (c + a.out.R - 1) / a.out.R;
    }
    int n_gather;
    int gbase = block_excl_sum(my_gt, &n_gather, sm33);
    bool overflow = false;
    for (int n = n_lo; n < n_hi; ++n) {
        const int g0 = short_before(a.seg_start[n]);
        const int c = short_before(a.seg_start[n + 1]) - g0;
        for (int off = 0; off < c; off += a.out.R, ++gbase) {
            if (gbase < a.out.max_gather)
                a.out.gather[gbase] = make_int4(n, g0 + off, min(a.out.R, c - off), 0);
            else
                overflow = true;
        }
    }
    if (tid == 0) {
        a.out.counts[1] = min(n_gather, a.out.max_gather);
        a.out.counts[2] = min(n_contig, a.out.max_contig);
        a.out.counts[3] = n_short;
        if (n_contig > a.out.max_contig) overflow = true;
    }
    if (overflow) atomicOr(a.out.status, LORA_DEV_TILE_OVERFLOW);
}

static size_t ws_bytes(int T, int N) {   // size_t throughout: no int overflow for any T, N
    const size_t n_chunks = ((size_t)T + SEG_CHUNK - 1) / SEG_CHUNK;
    return (n_chunks * ((size_t)N + 1) * sizeof(int) + 255) & ~(size_t)255;
}

static size_t round256(size_t b) { return (b + 255) & ~(size_t)255; }
static int tw_words(int T) { return (int)(((int64_t)T + 31) / 32); }
static int tw_blocks(int T) { return (tw_words(T) + TW_WORDS - 1) / TW_WORDS; }

// per-chunk id counts | run-start byte per row | 3 words per 32 rows | 4 ints per block
size_t segments_scratch_bytes(int T, int N) {
    if (one_block(T, N)) return 0;
    return ws_bytes(T, N) + round256((size_t)T) + round256((size_t)12 * tw_words(T)) +
           round256((size_t)16 * tw_blocks(T));
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
    a.brkb = nullptr;
    a.brkw = a.lngw = nullptr;
    a.gpre = nullptr;
    a.blk = nullptr;
    a.W = tw_words(m->T);
    a.B = tw_blocks(m->T);
    if (scratch) {
        uint8_t *p = static_cast<uint8_t *>(scratch) + ws_bytes(m->T, m->N);
        a.brkb = p;
        p += round256((size_t)m->T);
        a.brkw = reinterpret_cast<uint32_t *>(p);
        a.lngw = a.brkw + a.W;
        a.gpre = reinterpret_cast<int *>(a.lngw + a.W);
        p += round256((size_t)12 * a.W);
        a.blk = reinterpret_cast<int4 *>(p);
    }
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

    if (one_block(a.T, a.N)) {
        const size_t nwr = rank_warps(a.N);
        const size_t smem = (SEG_SCAN_WORDS + (((size_t)a.N + 1 + 3) & ~(size_t)3) +
                             ((nwr * (a.N + 1) + 3) & ~(size_t)3) + 2 * (size_t)a.T +
                             tiles_smem_words(a.T)) * sizeof(int) + (size_t)a.T;
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
        const size_t scan_smem = (SEG_SCAN_WORDS + bins) * sizeof(int);
        seg_scan_kernel<<<1, SEG_THREADS, scan_smem, st>>>(a, n_chunks);
        const size_t scat_smem =
            ((((size_t)a.N + 1 + 3) & ~(size_t)3) + (size_t)rank_warps(a.N) * bins) * sizeof(int);
        if (scat_smem > 48 * 1024)
            cudaFuncSetAttribute(seg_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)scat_smem);
        seg_scatter_kernel<<<n_chunks, SEG_THREADS, scat_smem, st>>>(a);
        seg_runs_kernel<<<a.B, TW_THREADS, 0, st>>>(a);
        seg_long_kernel<<<a.B, TW_THREADS, 0, st>>>(a);
        seg_emit_kernel<<<a.B, TW_THREADS, 0, st>>>(a);
        seg_gtiles_kernel<<<1, SEG_THREADS, 0, st>>>(a);
    }
    return cuda_rc(cudaGetLastError());
}

}  // namespace lora
