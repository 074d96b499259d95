// Fused multi-LoRA BGMV over gathered rows, bf16, ranks up to 64 (page
// "Multi-LoRA Serving", section 3.2: rows grouped per adapter, BGMV-style
// grouped products; section 3.4: add_shrink then add_expand in one call).
//
// Unit of work = up to 64 rows that share an adapter (a gathered tile, or a
// piece of a contiguous tile).  All rows of a unit share one stream of the
// adapter's A and B, so an adapter with up to 64 rows in the batch is read
// from HBM once.  One persistent launch runs two phases:
//
//   shrink   a cluster of C thread blocks takes a unit; block c reduces 1/C
//            of the input columns: v_part[rows][S*r8] = x[rows][cols] .
//            A_s[n][0:r8][cols]^T (tensor-pipe mma m16n8k16, bf16 in, fp32
//            accumulate).  The C partials meet in distributed shared memory
//            (st.async stores counted in bytes on the owner's mbarrier; the
//            owner adds them in rank order, so results are run-to-run
//            identical) and the owners write v = A x (fp32) for k < r_n.
//   expand   every block on its own takes an expand item = (unit, slice,
//            block of output columns): y[rows][cols] += (alpha_n / r_n) v .
//            B_s[n][cols][0:r8]^T, fp32 accumulation, y rounded once.
//
// In the fused mode v moves between the phases through a caller-provided
// workspace: the shrink owners write it, and an expand item of unit u starts
// its v copy once u's C blocks have signalled (a per-unit counter, release /
// acquire at GPU scope).  Its bytes stay in L2 (about 2 KB per row); the
// adapters and the rows cross HBM once.  Shrink units are taken by clusters
// and expand items by blocks from atomic tickets, so a block only ever waits
// for units that a running cluster already holds: the launch makes progress
// whatever number of its blocks is resident (and beside other kernels).  The
// tickets, the per-unit counters and an exit counter live at the head of the
// workspace; the last block to leave puts them back to zero.  The shrink-only
// and expand-only modes (v from / to the caller) assign work statically and
// need no workspace.
//
// Block layout (288 threads, one block per SM):
//   warp 8        producer: walks the block's work and fills a ring of
//                 GB_STAGES x 32 KB stages through the TMA engine - A boxes
//                 of 8-64 ranks x 64 columns (128-byte swizzle), B boxes of 64
//                 output columns x 8-64 ranks (swizzle matched to the box
//                 width), one 1-D bulk copy per gathered x / y / v row piece.
//                 Each stage carries a header (what the chunk is, its rows)
//                 written before the stage's arrival; a full/empty mbarrier
//                 pair guards each stage.
//   warps 0-7     consumers: follow the headers; shrink chunks -> mma into
//                 registers, the last chunk of a pass -> exchange; expand
//                 chunks -> mma with s v as a bf16 hi + lo pair (about 16
//                 mantissa bits), y updated in shared memory and written back
//                 with 16-byte stores.
// Box sizes follow the adapter's own rank (r8 = r_n rounded up to 8), not the
// slot size r_max: rank rows / columns r8..r_max are never loaded; ranks
// r_n..r8 are loaded and masked out of every product.
//
// Every wait is bounded (a suspend-time hint per try, and a try limit): a wait
// that runs out sets LORA_DEV_TIMEOUT in the status word and the block stops
// taking work; consumer threads agree on every outcome through a barrier
// reduction, so no named barrier is left unpaired.
#include "kernels.cuh"
#include "ptx.cuh"

#include <cstdlib>
#include <mutex>

namespace lora {

constexpr int GB_CONSUMERS = 8;                      // consumer warps
constexpr int GB_THREADS = (GB_CONSUMERS + 1) * 32;  // + 1 producer warp
constexpr int GB_ROWS = LORA_MAX_TILE_ROWS;          // rows of one unit
constexpr int GB_MAX_STAGES = 6;
constexpr int GB_STAGES_DEFAULT = 4;
constexpr int GB_SB = 32768;                         // bytes of one ring stage
constexpr int GB_HDR = 384;                          // bytes of one stage header
constexpr int GB_XCAP = 8192;                        // partial elements of one exchange
constexpr int GB_XBUF = GB_XCAP + 64;                // floats of one exchange buffer
constexpr int GB_PART = 1024;                        // floats of the k-group staging
constexpr int GB_TK = 8;                             // shrink tickets in flight per cluster

enum { GB_SHRINK = 0, GB_EXPAND = 1, GB_END = 2 };
enum { GB_FIRST = 1, GB_LAST = 2, GB_NODATA = 4, GB_UNIT_DONE = 8 };

// What one ring stage holds, written by the producer before the stage's arrival.
struct GbHdr {
    int kind, flags;
    int unit, n, r_n, r8, cnt;   // unit, adapter, rank, rank rounded to 8, rows
    int s0, sn;                  // shrink: slices [s0, s0+sn) of this chunk; expand: slice s0
    int c0, w;                   // shrink: first input column, width; expand: slice-local column, width
    int cw;                      // chunk width: rows sit at 2*cw+16 bytes
    int bofs;                    // byte offset of the adapter boxes (shrink: A, expand: B)
    int yofs;                    // expand: byte offset of the y rows (v rows sit at 0)
    float scale;                 // expand: alpha_n / r_n
    int pad;
    int rows[GB_ROWS];
};
static_assert(sizeof(GbHdr) <= GB_HDR, "stage header");

// Workspace head of the fused mode (ints): tickets and exit counter, then one
// counter per unit.
constexpr int GB_CTL_INTS = 64;
enum { GB_T_SHRINK = 0, GB_T_EXPAND = 1, GB_T_EXIT = 2 };

// ------------------------------------------------------------------ PTX helpers
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void consumer_sync() {
    asm volatile("bar.sync 1, %0;\n" ::"n"(GB_CONSUMERS * 32) : "memory");
}
// every consumer thread passes p; returns the AND over all of them
__device__ __forceinline__ bool consumers_all(bool p) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred q, o;\n\tsetp.ne.u32 q, %1, 0;\n\t"
        "bar.red.and.pred o, 1, %2, q;\n\tselp.u32 %0, 1, 0, o;\n\t}\n"
        : "=r"(r)
        : "r"((uint32_t)p), "n"(GB_CONSUMERS * 32)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ uint32_t cta_rank_in_cluster() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;\n" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_size() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_nctarank;\n" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_barrier() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n"
                 "barrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}
__device__ __forceinline__ uint4 zero_if(bool z, uint4 v) { return z ? make_uint4(0, 0, 0, 0) : v; }
// 8 bytes into the shared memory of a block of the cluster, completing 8
// transaction bytes on that block's mbarrier (no fence on either side)
__device__ __forceinline__ void st_async_v2(uint32_t addr, float a, float b, uint32_t bar) {
    asm volatile(
        "st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.f32 [%0], {%1,%2}, [%3];\n" ::"r"(addr),
        "f"(a), "f"(b), "r"(bar)
        : "memory");
}
__device__ __forceinline__ void st_async_u32(uint32_t addr, uint32_t v, uint32_t bar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.u32 [%0], %1, [%2];\n" ::"r"(addr),
                 "r"(v), "r"(bar)
                 : "memory");
}
// one arrival on an mbarrier of another block of the cluster
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t remote_bar) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];\n" ::"r"(remote_bar)
                 : "memory");
}
__device__ __forceinline__ void red_release_gpu(int *p, int v) {
    asm volatile("red.release.gpu.global.add.s32 [%0], %1;\n" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ int ld_acquire_gpu(const int *p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];\n" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ float4 lds128f(uint32_t a) {
    float4 r;
    asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];\n"
                 : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w)
                 : "r"(a));
    return r;
}
__device__ __forceinline__ float2 lds64f(uint32_t a) {
    float2 r;
    asm volatile("ld.shared.v2.f32 {%0,%1}, [%2];\n" : "=f"(r.x), "=f"(r.y) : "r"(a));
    return r;
}

__device__ __forceinline__ int align_up(int v, int a) { return (v + a - 1) & ~(a - 1); }

// Byte offset of (output column col, rank k) in the B boxes of an expand
// chunk.  Per 64 columns: 128*r8 bytes.  r8 a power of two: one box of 64 rows
// x r8 ranks, rows of 2*r8 bytes, swizzled in 16-byte units by the row bits
// above 128 bytes (the TMA 32/64/128-byte swizzle for 32/64/128-byte rows);
// otherwise r8/8 boxes of 64 rows x 8 ranks (16-byte rows, no swizzle).
__device__ __forceinline__ uint32_t b_off(int col, int k, int r8) {
    const uint32_t blk = (uint32_t)(col >> 6) * (uint32_t)(128 * r8);
    const int cr = col & 63;
    if (r8 & (r8 - 1))
        return blk + (uint32_t)((k >> 3) * 1024 + cr * 16 + (k & 7) * 2);
    uint32_t off = (uint32_t)(cr * 2 * r8 + 2 * k);
    off ^= ((off >> 7) & (uint32_t)((r8 >> 3) - 1)) << 4;
    return blk + off;
}

// ------------------------------------------------------------------ geometry (shared by host tests)
// Rows of one shrink pass.  Each consumer warp owns one m16 tile of the pass
// and a run of its S*r8/8 rank tiles: mtp warps-groups (1, 2 or 4) cover the
// m16 tiles, and a warp holds at most 8 (m16, n8) accumulators, so
// pow2(m16 tiles) * S*r8 <= 512; that also bounds the exchange (16 * 512
// partial elements = GB_XCAP).
__host__ __device__ inline int gb_pass_rows(int cnt, int S, int r8) {
    const int mt_max = 512 / (S * r8);
    const int pr = mt_max >= 4 ? 64 : (mt_max >= 2 ? 32 : 16);
    return cnt < pr ? cnt : pr;
}
// Slices per shrink chunk: as many as fit a stage beside 64 columns of x rows.
__host__ __device__ inline int gb_shrink_slices(int pcnt, int S, int r8) {
    const int xb = (pcnt * (128 + 16) + 1023) & ~1023;
    int sg = (GB_SB - xb) / (r8 * 128);
    return sg < 1 ? 1 : (sg > S ? S : sg);
}
// Columns per shrink chunk (multiple of 64, at most 1024) for pcnt rows and sn slices.
__host__ __device__ inline int gb_shrink_cols(int pcnt, int sn, int r8) {
    int jc = (GB_SB - 16 * pcnt - 1023) / (2 * pcnt + 2 * sn * r8);
    jc &= ~63;
    return jc < 64 ? 64 : (jc > 1024 ? 1024 : jc);
}
// Columns per expand chunk (multiple of 64, at most 2048) for cnt rows with
// vbytes of v rows in front; 0 when not even 64 columns fit beside the v rows.
__host__ __device__ inline int gb_expand_cols(int cnt, int r8, int vbytes) {
    int cc = (GB_SB - ((vbytes + 15) & ~15) - 16 * cnt - 1023) / (2 * cnt + 2 * r8);
    cc &= ~63;
    return cc > 2048 ? 2048 : (cc < 0 ? 0 : cc);
}

// Shared memory: ring | headers | exchange buffers [2] | k-group staging | pass rows | tickets | barriers
struct GbSmem {
    uint32_t ring, hdr, recv, part, xrows, tkslot;
    uint32_t full0, empty0, xready0, tkbar0, tkfree0;
    int *flag;   // generic pointer: "this block leaves last"
};

size_t bgmv_smem_bytes(int mode, int stages) {
    size_t b = 1024 + (size_t)stages * (GB_SB + GB_HDR);
    if (mode != MODE_EXPAND) b += (size_t)2 * GB_XBUF * 4 + GB_PART * 4;
    b += GB_ROWS * 4 + GB_TK * 4 + 16 + (size_t)(2 * GB_MAX_STAGES + 2 + 2 * GB_TK) * 8;
    return b;
}

struct UnitInfo {
    int n, cnt, r_n, r8;
    bool ok;
};

// Unit u's adapter, rank and rows (all lanes of the producer warp; lane l holds
// rows l and l + 32 in row0 / row1).
__device__ __forceinline__ UnitInfo fetch_unit(const GbArgs &a, int u, int &row0, int &row1) {
    const int lane = threadIdx.x & 31;
    const Unit un = resolve_live_unit(a.tiles, u);
    UnitInfo f;
    f.n = un.id;
    f.cnt = un.cnt;
    f.r_n = un.cnt > 0 ? a.ranks[un.id] : 0;
    f.ok = un.cnt > 0 && f.r_n >= 1 && f.r_n <= a.r_max;
    f.r8 = (f.r_n + 7) & ~7;
    row0 = lane < f.cnt ? un.row(a.tiles, lane) : -1;
    row1 = lane + 32 < f.cnt ? un.row(a.tiles, lane + 32) : -1;
    return f;
}

// Tile record of unit v (one dependent load): adapter, first row (contiguous) or
// first index into grow (gathered), rows.  ng = live gathered tiles.
struct URec {
    int id, base, cnt, gathered;
};
__device__ __forceinline__ URec unit_rec(const Tiles &t, int ng, int v) {
    URec r{0, 0, 0, 1};
    if (v < ng) {
        const int4 g = t.gather[v];
        r.id = g.x;
        r.base = g.y;
        r.cnt = g.z;
        return r;
    }
    v -= ng;
    const int tile = v / t.subs, sub = v - tile * t.subs;
    const int4 c = t.contig[tile];
    const int first = sub * t.rows_per_unit;
    if (first < c.z) {
        r.id = c.x;
        r.base = c.y + first;
        r.cnt = min(t.rows_per_unit, c.z - first);
        r.gathered = 0;
    }
    return r;
}
// What the producer needs beyond the record: rank, alpha, rows (lane l: rows l, l+32).
struct UMeta {
    int r_n;
    float alpha;
    int row0, row1;
};
__device__ __forceinline__ UMeta unit_meta(const GbArgs &a, const URec &r) {
    const int lane = threadIdx.x & 31;
    UMeta m;
    m.r_n = r.cnt > 0 ? a.ranks[r.id] : 0;
    m.alpha = r.cnt > 0 ? a.alphas[r.id] : 0.f;
    m.row0 = lane < r.cnt ? (r.gathered ? a.tiles.grow[r.base + lane] : r.base + lane) : -1;
    m.row1 = lane + 32 < r.cnt ? (r.gathered ? a.tiles.grow[r.base + lane + 32] : r.base + lane + 32) : -1;
    return m;
}

// ================================================================ producer warp
template <int MODE>
__device__ void gb_producer(const GbArgs &a, const GbSmem &sm, bool &failed) {
    const int lane = threadIdx.x & 31;
    const int S = a.sl.n, NS = a.stages;
    const uint32_t crank = cta_rank_in_cluster(), C = cluster_size();
    const int cid = blockIdx.x / (int)C, ncl = gridDim.x / (int)C;
    const int live = n_live_units(a.tiles);
    uint32_t gi = 0;   // stages filled so far

    // next free stage (bounded wait; the whole warp sees the outcome)
    auto acquire = [&](int &st, uint32_t &dst, GbHdr *&h) -> bool {
        st = (int)(gi % (uint32_t)NS);
        bool ok = !failed;
        if (ok && gi >= (uint32_t)NS && lane == 0)
            ok = mbar_wait(sm.empty0 + 8 * st, ((gi / NS) - 1) & 1, a.status, failed, a.wait_limit);
        ok = __shfl_sync(FULL, ok ? 1 : 0, 0) != 0;
        if (!ok) failed = true;
        dst = sm.ring + (uint32_t)st * GB_SB;
        h = reinterpret_cast<GbHdr *>(__cvta_shared_to_generic(sm.hdr + (uint32_t)st * GB_HDR));
        return ok;
    };
    // test hook (a.dbg_stall): the block's first stage expects 16 bytes more than arrive,
    // so its consumers' bounded wait runs out
    const unsigned stall = a.dbg_stall ? 16u : 0u;
    auto commit = [&](int st, unsigned bytes) {   // header written: arrive with the stage's bytes
        __syncwarp();
        if (lane == 0) mbar_expect_tx(sm.full0 + 8 * st, bytes + (gi == 0 ? stall : 0u));
        __syncwarp();
        ++gi;
    };

    // ------------------------------------------------------------ phase 1: shrink
    if (MODE != MODE_EXPAND) {
        // fused mode: cluster rank 0 draws unit tickets and hands them to every block
        // of the cluster through a ring of GB_TK slots with credits
        auto send_ticket = [&](uint32_t j) {   // lane 0 of rank 0 only
            const uint32_t slot = j % GB_TK;
            if (j >= GB_TK &&
                !mbar_wait<true>(sm.tkfree0 + 8 * slot, ((j / GB_TK) - 1) & 1, a.status, failed,
                                 a.wait_limit))
                return;
            const int tk = atomicAdd(a.ctl + GB_T_SHRINK, 1);
            for (uint32_t c = 0; c < C; ++c)
                st_async_u32(map_rank(sm.tkslot + 4 * slot, c), (uint32_t)tk,
                             map_rank(sm.tkbar0 + 8 * slot, c));
        };
        if (MODE == MODE_FUSED && crank == 0 && lane == 0) send_ticket(0);
        for (uint32_t k = 0;; ++k) {
            int u = 0;
            if (MODE == MODE_FUSED) {
                const uint32_t slot = k % GB_TK;
                int got = -1;
                if (lane == 0 && !failed) {
                    mbar_expect_tx(sm.tkbar0 + 8 * slot, 4);
                    if (mbar_wait<true>(sm.tkbar0 + 8 * slot, (k / GB_TK) & 1, a.status, failed,
                                       a.wait_limit)) {
                        got = *reinterpret_cast<volatile int *>(
                            __cvta_shared_to_generic(sm.tkslot + 4 * slot));
                        mbar_arrive_cluster(map_rank(sm.tkfree0 + 8 * slot, 0));
                        if (crank == 0 && got < live) send_ticket(k + 1);
                    }
                }
                got = __shfl_sync(FULL, got, 0);
                // a wait of lane 0 that ran out (here or in send_ticket) stops the whole warp
                failed = __any_sync(FULL, failed) != 0;
                if (got < 0 || failed) {
                    failed = true;
                    break;
                }
                u = got;
            } else {
                u = cid + (int)k * ncl;
            }
            if (u >= live || failed) break;
            int row0, row1;
            const UnitInfo f = fetch_unit(a, u, row0, row1);
            if (!f.ok) {
                if (f.cnt > 0 && crank == 0 && lane == 0) atomicOr(a.status, LORA_DEV_BAD_RANK);
                continue;
            }
            const int r8 = f.r8;
            const int n64 = (a.d_in + 63) >> 6;
            const int j_lo = (int)((int64_t)crank * n64 / C) * 64;
            const int j_hi = min((int)((int64_t)(crank + 1) * n64 / C) * 64, a.d_in);
            const int span = j_hi - j_lo;
            const int pr = gb_pass_rows(f.cnt, S, r8);
            for (int p0 = 0; p0 < f.cnt && !failed; p0 += pr) {
                const int pcnt = min(pr, f.cnt - p0);
                const bool last_pass = p0 + pcnt >= f.cnt;
                const int sg = gb_shrink_slices(pcnt, S, r8);
                const int JC = gb_shrink_cols(pcnt, sg, r8);
                const int RS = 2 * JC + 16;
                const int ncol = span > 0 ? (span + JC - 1) / JC : 1;
                const int nsg = (S + sg - 1) / sg;
                const int nch = ncol * nsg;
                for (int q = 0; q < nch; ++q) {
                    int st;
                    uint32_t dst;
                    GbHdr *h;
                    if (!acquire(st, dst, h)) break;
                    const int qc = q / nsg, qs = q - qc * nsg;
                    const int jc0 = j_lo + qc * JC;
                    const int width = span > 0 ? min(JC, j_hi - jc0) : 0;
                    const int s0 = qs * sg, sn = min(sg, S - s0);
                    const int bofs = align_up(pcnt * RS, 1024);
                    if (lane == 0) {
                        h->kind = GB_SHRINK;
                        h->flags = (q == 0 ? GB_FIRST : 0) | (q == nch - 1 ? GB_LAST : 0) |
                                   (width == 0 ? GB_NODATA : 0) |
                                   (last_pass && q == nch - 1 ? GB_UNIT_DONE : 0);
                        h->unit = u;
                        h->n = f.n;
                        h->r_n = f.r_n;
                        h->r8 = r8;
                        h->cnt = pcnt;
                        h->s0 = s0;
                        h->sn = sn;
                        h->c0 = jc0;
                        h->w = width;
                        h->cw = JC;
                        h->bofs = bofs;
                        h->yofs = 0;
                        h->scale = 0.f;
                    }
                    // rows p0 .. p0+pcnt-1 of the unit
                    if (lane >= p0 && lane < p0 + pcnt) h->rows[lane - p0] = row0;
                    if (lane + 32 >= p0 && lane + 32 < p0 + pcnt) h->rows[lane + 32 - p0] = row1;
                    __syncwarp();
                    const int nbox = (width + 63) >> 6, ncb = JC >> 6;
                    // rank boxes: r8 as a sum of 64/32/16/8-rank boxes
                    int parts[4], nparts = 0;
                    for (int R = 64, k0 = 0; R >= 8; R >>= 1)
                        if (r8 & R) {
                            parts[nparts++] = (k0 << 8) | R;
                            k0 += R;
                        }
                    const unsigned bytes =
                        width > 0 ? (unsigned)(pcnt * width * 2 + sn * nbox * r8 * 128) : 0u;
                    if (width > 0) {
                        for (int r = lane; r < pcnt; r += 32)
                            bulk_g2s(dst + r * RS, a.x + (int64_t)h->rows[r] * a.ld_x + jc0,
                                     (unsigned)width * 2, sm.full0 + 8 * st);
                        const int nb = sn * nbox * nparts;
                        for (int e = lane; e < nb; e += 32) {
                            const int ss = e / (nbox * nparts), rem = e - ss * (nbox * nparts);
                            const int cb = rem / nparts, pi = rem - cb * nparts;
                            const int k0 = parts[pi] >> 8, R = parts[pi] & 255;
                            const int mi = R == 64 ? 3 : (R == 32 ? 2 : (R == 16 ? 1 : 0));
                            tma_2d(dst + bofs + (uint32_t)(((ss * ncb + cb) * r8 + k0) * 128),
                                   &a.tmA[s0 + ss][mi], jc0 + 64 * cb, f.n * a.r_max + k0,
                                   sm.full0 + 8 * st);
                        }
                    }
                    commit(st, bytes);
                }
            }
        }
    }

    // ------------------------------------------------------------ phase 2: expand
    // Items are drawn two ahead and their metadata one ahead: at the start of item i
    // the ticket of item i+2 and the tile record of item i+1 are requested, and the
    // rank, alpha and rows of item i+1 right after item i's chunks are issued, so
    // the dependent global reads overlap the ring's drain instead of stalling it.
    if (MODE != MODE_SHRINK && !failed) {
        const int nb = a.blk_off[S];
        const int total = live * nb;
        const int ng = a.tiles.use_gather ? min(a.tiles.counts[1], a.tiles.max_gather) : 0;
        auto claim = [&](int prev) -> int {   // the next item (fused: lane 0's ticket)
            if (MODE == MODE_FUSED) return lane == 0 ? atomicAdd(a.ctl + GB_T_EXPAND, 1) : 0;
            return prev + (int)gridDim.x;
        };
        auto bcast = [&](int v) -> int { return MODE == MODE_FUSED ? __shfl_sync(FULL, v, 0) : v; };
        int e_cur = bcast(claim((int)blockIdx.x - (int)gridDim.x));
        int e_raw = claim(e_cur);   // item i+1, not yet broadcast
        URec rec = e_cur < total ? unit_rec(a.tiles, ng, e_cur / nb) : URec{0, 0, 0, 1};
        UMeta meta = unit_meta(a, rec);
        for (;;) {
            if (e_cur >= total || failed) break;
            const int e_nxt = bcast(e_raw);
            const URec rec_nxt = e_nxt < total ? unit_rec(a.tiles, ng, e_nxt / nb) : URec{0, 0, 0, 1};
            e_raw = claim(e_nxt);
            const int u = e_cur / nb, b = e_cur - u * nb;
            int s = 0;
            while (s + 1 < S && a.blk_off[s + 1] <= b) ++s;
            const int c_item = (b - a.blk_off[s]) * a.bc;
            const int w_item = min(a.bc, a.sl.d_out[s] - c_item);
            const int cnt = rec.cnt, r_n = meta.r_n;
            const bool ok_rank = cnt > 0 && r_n >= 1 && r_n <= a.r_max;
            if (!ok_rank) {
                if (cnt > 0 && b == 0 && lane == 0) atomicOr(a.status, LORA_DEV_BAD_RANK);
            } else {
                const int r8 = (r_n + 7) & ~7;
                const float scale = meta.alpha / (float)r_n;
                const int vbytes = cnt * r8 * 4;
                const int d_out = a.sl.d_out[s];
                const int mi = r8 == 64 ? 3 : (r8 == 32 ? 2 : (r8 == 16 ? 1 : 0));
                const bool wide = (r8 & (r8 - 1)) == 0;
                int c = c_item;
                bool first = true;
                while ((c < c_item + w_item || first) && !failed) {
                    const int vb = first ? vbytes : 0;
                    int CC = gb_expand_cols(cnt, r8, vb);
                    int w = min(CC, c_item + w_item - c);
                    if (CC == 0) w = 0;   // v rows alone in this stage
                    int st;
                    uint32_t dst;
                    GbHdr *h;
                    if (!acquire(st, dst, h)) break;
                    const int CCs = CC > 0 ? CC : 64;
                    const int YS = 2 * CCs + 16;
                    const int yofs = align_up(vb, 16);
                    const int bofs = align_up(yofs + cnt * YS, 1024);
                    const bool last = c + w >= c_item + w_item;
                    if (lane == 0) {
                        h->kind = GB_EXPAND;
                        h->flags = (first ? GB_FIRST : 0) | (last ? GB_LAST : 0);
                        h->unit = u;
                        h->n = rec.id;
                        h->r_n = r_n;
                        h->r8 = r8;
                        h->cnt = cnt;
                        h->s0 = s;
                        h->sn = 1;
                        h->c0 = c;
                        h->w = w;
                        h->cw = CCs;
                        h->bofs = bofs;
                        h->yofs = yofs;
                        h->scale = scale;
                    }
                    if (lane < cnt) h->rows[lane] = meta.row0;
                    if (lane + 32 < cnt) h->rows[lane + 32] = meta.row1;
                    __syncwarp();
                    const int nbox = (w + 63) >> 6;
                    const unsigned bytes = (unsigned)(vb + cnt * w * 2 + nbox * 128 * r8);
                    if (lane == 0) mbar_expect_tx(sm.full0 + 8 * st, bytes + (gi == 0 ? stall : 0u));
                    __syncwarp();
                    if (w > 0) {
                        const __nv_bfloat16 *ybase = a.y + a.sl.col_off[s] + c;
                        for (int r = lane; r < cnt; r += 32)
                            bulk_g2s(dst + yofs + r * YS, ybase + (int64_t)h->rows[r] * a.ld_y,
                                     (unsigned)w * 2, sm.full0 + 8 * st);
                        const int nbb = wide ? nbox : nbox * (r8 >> 3);
                        for (int e2 = lane; e2 < nbb; e2 += 32) {
                            const int cb = wide ? e2 : e2 / (r8 >> 3);
                            const int kb = wide ? 0 : e2 - cb * (r8 >> 3);
                            tma_2d(dst + bofs + (uint32_t)(cb * 128 * r8 + kb * 1024),
                                   &a.tmB[s][wide ? mi : 0], kb * 8, rec.id * d_out + c + 64 * cb,
                                   sm.full0 + 8 * st);
                        }
                    }
                    if (first) {
                        if (MODE == MODE_FUSED) {
                            // v of this unit is complete once its C shrink blocks have signalled
                            bool ok = true;
                            if (lane == 0) {
                                unsigned it = 0;
                                while (ld_acquire_gpu(a.done + u) < (int)C) {
                                    if (++it >= a.wait_limit * 64u) {
                                        atomicOr(a.status, LORA_DEV_TIMEOUT);
                                        ok = false;
                                        break;
                                    }
                                    __nanosleep(128);
                                }
                            }
                            ok = __shfl_sync(FULL, ok ? 1 : 0, 0) != 0;
                            if (!ok) failed = true;
                            // the v rows were written by other blocks' generic stores; order
                            // the copies below (async proxy) after the acquire above
                            asm volatile("fence.proxy.async.global;\n" ::: "memory");
                        }
                        if (!failed) {
                            for (int r = lane; r < cnt; r += 32)
                                bulk_g2s(dst + r * r8 * 4,
                                         a.v + ((int64_t)s * a.T + h->rows[r]) * a.r_max,
                                         (unsigned)r8 * 4, sm.full0 + 8 * st);
                        }
                    }
                    __syncwarp();
                    ++gi;
                    c += w;
                    first = false;
                    if (w == 0 && CC > 0) break;
                }
            }
            meta = unit_meta(a, rec_nxt);   // the next item's rank, alpha and rows
            rec = rec_nxt;
            e_cur = e_nxt;
        }
    }

    // ------------------------------------------------------------ end of the stream
    {
        int st;
        uint32_t dst;
        GbHdr *h;
        const bool was_failed = failed;
        bool ok = !was_failed;
        if (ok) ok = acquire(st, dst, h);
        if (ok) {
            if (lane == 0) h->kind = GB_END;
            commit(st, 0);
        }
    }
}

// ================================================================ consumer warps
// Wait for stage gi to be full; every consumer thread sees the same outcome.
__device__ __forceinline__ bool gb_stage_wait(const GbArgs &a, const GbSmem &sm, uint32_t gi,
                                              bool &failed) {
    const int st = (int)(gi % (uint32_t)a.stages);
    bool ok = !failed && mbar_wait(sm.full0 + 8 * st, (gi / a.stages) & 1, a.status, failed,
                                  a.wait_limit);
    ok = consumers_all(ok);
    if (!ok) failed = true;
    return ok;
}
__device__ __forceinline__ const GbHdr *gb_hdr(const GbSmem &sm, int st) {
    return reinterpret_cast<const GbHdr *>(__cvta_shared_to_generic(sm.hdr + (uint32_t)st * GB_HDR));
}
// This warp is done with stage st (its shared memory may be refilled by TMA).
__device__ __forceinline__ void gb_release(const GbSmem &sm, int st) {
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(sm.empty0 + 8 * st);
}

// One warp's MMAs for one 64-column box of a shrink chunk: NPW pairs (this warp's
// m16 tile x NPW rank tiles), compile-time so that no branch surrounds the
// warp-synchronous MMAs; a pair whose slice is not in this chunk gets zero A
// fragments (loaded from a safe address).  One pair: two accumulators take
// alternate k-steps.
template <int NPW>
__device__ __forceinline__ void shrink_box(float (&acc)[8][4], const int (&pinfo)[8], uint32_t xrow,
                                           int RS, uint32_t abase, int ncb, int sp, int r8, int s0,
                                           int sn, int width, int g, int t) {
    const int col = sp * 64 + t * 16;
    const bool z0 = col >= width, z1 = col + 8 >= width;
    const uint32_t c0s = (uint32_t)(((2 * t) ^ g) << 4), c1s = (uint32_t)(((2 * t + 1) ^ g) << 4);
    const uint32_t xg = xrow + (uint32_t)(col * 2), xh = xg + 8 * RS;
    const uint4 xa0 = zero_if(z0, lds128(xg)), xa1 = zero_if(z1, lds128(xg + 16));
    const uint4 xb0 = zero_if(z0, lds128(xh)), xb1 = zero_if(z1, lds128(xh + 16));
    uint32_t arow[NPW];
    bool on[NPW];
#pragma unroll
    for (int i = 0; i < NPW; ++i) {
        const int s = pinfo[i] >> 8;
        on[i] = s >= s0 && s < s0 + sn;
        arow[i] = on[i] ? abase + (uint32_t)((((s - s0) * ncb + sp) * r8 + (pinfo[i] & 255)) * 128) : abase;
    }
    const uint32_t f0[4] = {xa0.x, xb0.x, xa0.y, xb0.y}, f1[4] = {xa0.z, xb0.z, xa0.w, xb0.w};
    const uint32_t f2[4] = {xa1.x, xb1.x, xa1.y, xb1.y}, f3[4] = {xa1.z, xb1.z, xa1.w, xb1.w};
#pragma unroll
    for (int half = 0; half < 2; ++half) {   // k-steps 0-1, then 2-3: each half's loads first
        const bool zh = half ? z1 : z0;
        const uint32_t cs = half ? c1s : c0s;
        uint4 af[NPW];
#pragma unroll
        for (int i = 0; i < NPW; ++i) af[i] = zero_if(zh || !on[i], lds128(arow[i] + cs));
        const uint32_t(&fa)[4] = half ? f2 : f0;
        const uint32_t(&fb)[4] = half ? f3 : f1;
        if (NPW == 1) {
            mma16816(acc[0], fa, af[0].x, af[0].y);
            mma16816(acc[1], fb, af[0].z, af[0].w);
        } else {
#pragma unroll
            for (int i = 0; i < NPW; ++i) mma16816(acc[i], fa, af[i].x, af[i].y);
#pragma unroll
            for (int i = 0; i < NPW; ++i) mma16816(acc[i], fb, af[i].z, af[i].w);
        }
    }
}

// Phase 1: shrink chunks until the stream moves on; returns the position of
// the first stage that is not a shrink chunk.
template <int MODE>
__device__ uint32_t gb_consume_shrink(const GbArgs &a, const GbSmem &sm, bool &failed) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, t = lane & 3;
    const uint32_t crank = cta_rank_in_cluster(), C = cluster_size();
    const int S = a.sl.n;
    int *xrows = reinterpret_cast<int *>(__cvta_shared_to_generic(sm.xrows));
    float *part = reinterpret_cast<float *>(__cvta_shared_to_generic(sm.part));

    float acc[8][4];
    // this warp's pairs: m16 tile wm, rank tiles n_lo .. n_lo + npw - 1 (k-group kgi of jg
    // when the rank tiles are fewer than the tile's warps); per pair i: slice << 8 | A rank row
    int pinfo[8];
    int nt = 0, np = 0, jg = 1, npw = 0, n_lo = 0, kgi = 0, W = 0, wm = 0;
    uint32_t xc = 0;   // exchanges so far (buffer parity)
    uint32_t gi = 0;
    for (;; ++gi) {
        if (!gb_stage_wait(a, sm, gi, failed)) break;
        const int st = (int)(gi % (uint32_t)a.stages);
        const GbHdr *h = gb_hdr(sm, st);
        if (h->kind != GB_SHRINK) break;
        const uint32_t stg = sm.ring + (uint32_t)st * GB_SB;
        const int flags = h->flags;
        const int cnt = h->cnt, r_n = h->r_n, r8 = h->r8;
        if (flags & GB_FIRST) {   // a new pass
            W = S * r8;
            const int mt = (cnt + 15) >> 4;
            const int mtp = mt <= 1 ? 1 : (mt <= 2 ? 2 : 4);
            const int wpm = GB_CONSUMERS / mtp;   // warps per m16 tile
            nt = W >> 3;
            np = mt * nt;
            wm = warp % mtp;
            const int wj = warp / mtp;
            // jg is the same in every consumer warp (idle ones included): it decides
            // whether the exchange takes the shared-memory staging and its barrier
            jg = nt >= wpm ? 1 : wpm / nt;
            npw = 0;
            kgi = 0;
            n_lo = 0;
            if (wm < mt) {
                if (jg == 1) {
                    const int per = (nt + wpm - 1) / wpm;
                    n_lo = wj * per;
                    npw = max(0, min(nt, n_lo + per) - n_lo);
                } else {
                    n_lo = wj % nt;
                    kgi = wj / nt;
                    npw = kgi < jg ? 1 : 0;
                }
            }
            const int nkb8 = r8 >> 3;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int nn = n_lo + (i < npw ? i : 0);
                const int s = nn / nkb8;
                pinfo[i] = (s << 8) | ((nn - s * nkb8) * 8 + g);
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[i][e] = 0.f;
            }
            if (tid < cnt) xrows[tid] = h->rows[tid];
        }
        if (!(flags & GB_NODATA) && npw > 0) {
            const int width = h->w, JC = h->cw, RS = 2 * JC + 16, ncb = JC >> 6;
            const int s0 = h->s0, sn = h->sn;
            const uint32_t abase = stg + (uint32_t)h->bofs;
            const int nbox = (width + 63) >> 6;
            const uint32_t xrow = stg + (uint32_t)((16 * wm + g) * RS);
            for (int sp = kgi; sp < nbox; sp += jg) {
#define LORA_SHRINK(N) shrink_box<N>(acc, pinfo, xrow, RS, abase, ncb, sp, r8, s0, sn, width, g, t)
                switch (npw) {
                    case 1: LORA_SHRINK(1); break;
                    case 2: LORA_SHRINK(2); break;
                    case 3: LORA_SHRINK(3); break;
                    case 4: LORA_SHRINK(4); break;
                    case 5: LORA_SHRINK(5); break;
                    case 6: LORA_SHRINK(6); break;
                    case 7: LORA_SHRINK(7); break;
                    default: LORA_SHRINK(8); break;
                }
#undef LORA_SHRINK
            }
        }
        const int unit = h->unit;
        gb_release(sm, st);   // the exchange below reads only registers and its own buffers
        if (!(flags & GB_LAST)) continue;

        // -------------------------------------------------------- exchange of the pass
        const uint32_t par = xc & 1u;
        const uint32_t xr = sm.xready0 + 8 * par;
        const uint32_t rbuf = sm.recv + par * (uint32_t)GB_XBUF * 4u;
        const int total_pairs = cnt * W / 2;
        const int spc = (total_pairs + (int)C - 1) / (int)C;
        const int mine = total_pairs > (int)crank ? (total_pairs - (int)crank + (int)C - 1) / (int)C : 0;
        if (tid == 0) mbar_expect_tx(xr, (unsigned)(mine * (int)C * 8));
        auto send = [&](int row, int col, float v0, float v1) {
            if (row >= cnt) return;
            const int P = (row * W + col) >> 1;
            const uint32_t o = (uint32_t)P % C, slot = (uint32_t)P / C;
            st_async_v2(map_rank(rbuf + ((crank * (uint32_t)spc + slot) * 2u) * 4u, o), v0, v1,
                        map_rank(xr, o));
        };
        if (npw == 1) {   // the two alternating accumulators of a single pair
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                acc[0][e] += acc[1][e];
                acc[1][e] = 0.f;
            }
        }
        if (jg > 1) {   // k-groups of one pair: add them in shared memory first
            if (npw > 0) {
                float *pp = part + (kgi * np + wm * nt + n_lo) * 128;
                pp[g * 8 + 2 * t] = acc[0][0];
                pp[g * 8 + 2 * t + 1] = acc[0][1];
                pp[(g + 8) * 8 + 2 * t] = acc[0][2];
                pp[(g + 8) * 8 + 2 * t + 1] = acc[0][3];
            }
            consumer_sync();
            for (int idx = tid; idx < np * 64; idx += GB_CONSUMERS * 32) {
                const int p = idx >> 6, r = (idx & 63) >> 2, c2 = (idx & 3) * 2;
                float v0 = 0.f, v1 = 0.f;
                for (int kg = 0; kg < jg; ++kg) {
                    v0 += part[(kg * np + p) * 128 + r * 8 + c2];
                    v1 += part[(kg * np + p) * 128 + r * 8 + c2 + 1];
                }
                const int m = p / nt, nn = p - m * nt;
                send(16 * m + r, nn * 8 + c2, v0, v1);
            }
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                if (i >= npw) break;
                const int col = (n_lo + i) * 8 + 2 * t;
                send(16 * wm + g, col, acc[i][0], acc[i][1]);
                send(16 * wm + g + 8, col, acc[i][2], acc[i][3]);
            }
        }
        bool xok = mbar_wait<true>(xr, (xc >> 1) & 1u, a.status, failed, a.wait_limit);
        xok = consumers_all(xok);
        ++xc;
        if (!xok) {
            failed = true;
            break;
        }
        // owned pairs: the C partials in rank order, v for k < r_n
        for (int j = tid; j < mine; j += GB_CONSUMERS * 32) {
            const int P = (int)crank + j * (int)C;
            float v0 = 0.f, v1 = 0.f;
            for (uint32_t c = 0; c < C; ++c) {
                const float2 pv = lds64f(rbuf + ((c * (uint32_t)spc + (uint32_t)j) * 2u) * 4u);
                v0 += pv.x;
                v1 += pv.y;
            }
            const int e = 2 * P, row = e / W, col = e - row * W;
            const int s = col / r8, k = col - s * r8;
            float *vr = a.v + ((int64_t)s * a.T + xrows[row]) * a.r_max;
            if (k < r_n) vr[k] = v0;
            if (k + 1 < r_n) vr[k + 1] = v1;
        }
        if (MODE == MODE_FUSED && (flags & GB_UNIT_DONE)) {
            // every consumer's v stores are ordered before thread 0's release by the barrier
            consumer_sync();
            if (tid == 0) red_release_gpu(a.done + unit, 1);
        } else {
            consumer_sync();   // xrows and the exchange buffer are reused by the next pass
        }
    }
    return gi;
}

// One warp's share of an expand chunk: y[rows of its m16 tile][its 8-column blocks]
// += (s v) B^T.  RB: ranks of one B box (8, 16, 32 or 64: one box per 64 columns,
// rows of 2*RB bytes swizzled in 16-byte units by the row bits above 128 bytes),
// or 0 for stacked 8-rank boxes (r8 / 8 boxes of 1 KB per 64 columns); NKB: 16-rank
// steps.  Both are compile-time so that the loop has no branch around the
// warp-synchronous MMAs and computes every shared-memory address without one.
// Loads are unconditional (out-of-chunk addresses stay inside the block's shared
// memory and their values are masked or never stored).
template <int RB, int NKB>
__device__ __forceinline__ void expand_warp(uint32_t bbase, uint32_t yg_ad, uint32_t yh_ad, bool okg,
                                            bool okh, int nblk, int b_first, int b_step, int r8,
                                            const uint32_t (&vhi)[4][4], const uint32_t (&vlo)[4][4],
                                            const uint32_t (&bmx)[4], const uint32_t (&bmy)[4], int g,
                                            int t) {
    constexpr int NB = 4;
    constexpr int SWM = RB >= 16 ? RB / 8 - 1 : 0;              // swizzle mask of the box rows
    constexpr int SWS = RB == 64 ? 0 : (RB == 32 ? 1 : 2);      // row bits above 128 bytes
    const int blk_bytes = 128 * (RB ? RB : r8);                // B bytes per 64 columns
    uint32_t kterm[NKB];                                       // rank part of the address
#pragma unroll
    for (int kb = 0; kb < NKB; ++kb)
        kterm[kb] = RB ? (uint32_t)(2 * (kb * 16 + 4 * t))
                       : (uint32_t)((2 * kb + (t >> 1)) * 1024 + 8 * (t & 1));
    for (int b0 = b_first; b0 < nblk; b0 += b_step) {
        uint2 bv[NB][NKB];
        uint32_t y0[NB], y1[NB];
#pragma unroll
        for (int j = 0; j < NB; ++j) {
            const int col = (b0 + j) * 8 + g, cr = col & 63;
            const uint32_t cbase = bbase + (uint32_t)((col >> 6) * blk_bytes);
#pragma unroll
            for (int kb = 0; kb < NKB; ++kb) {
                uint32_t off;
                if (RB) {
                    const uint32_t sw = SWM ? (uint32_t)(((RB == 64 ? cr : (cr >> SWS)) & SWM) << 4) : 0u;
                    off = (uint32_t)(cr * 2 * RB) + (kterm[kb] ^ sw);
                } else {
                    off = (uint32_t)(cr * 16) + kterm[kb];
                }
                bv[j][kb] = lds64(cbase + off);
            }
            y0[j] = lds32(yg_ad + (uint32_t)((b0 + j) * 16));
            y1[j] = lds32(yh_ad + (uint32_t)((b0 + j) * 16));
        }
        float d[NB][4];
#pragma unroll
        for (int j = 0; j < NB; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) d[j][e] = 0.f;
#pragma unroll
        for (int kb = 0; kb < NKB; ++kb) {
#pragma unroll
            for (int j = 0; j < NB; ++j)
                mma16816(d[j], vhi[kb], bv[j][kb].x & bmx[kb], bv[j][kb].y & bmy[kb]);
#pragma unroll
            for (int j = 0; j < NB; ++j)
                mma16816(d[j], vlo[kb], bv[j][kb].x & bmx[kb], bv[j][kb].y & bmy[kb]);
        }
        // y += delta in shared memory (rows g, g+8 of the tile; columns 2t, 2t+1)
#pragma unroll
        for (int j = 0; j < NB; ++j) {
            const bool okb = b0 + j < nblk;
            if (okb && okg)
                sts32(yg_ad + (uint32_t)((b0 + j) * 16),
                      pack_bf16x2(bf16_lo(y0[j]) + d[j][0], bf16_hi(y0[j]) + d[j][1]));
            if (okb && okh)
                sts32(yh_ad + (uint32_t)((b0 + j) * 16),
                      pack_bf16x2(bf16_lo(y1[j]) + d[j][2], bf16_hi(y1[j]) + d[j][3]));
        }
    }
}

// Phase 2: expand chunks from stage gi until the end of the stream.
template <int MODE>
__device__ void gb_consume_expand(const GbArgs &a, const GbSmem &sm, uint32_t gi, bool &failed) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, t = lane & 3;
    uint32_t vhi[4][4], vlo[4][4];
    uint32_t bmx[4], bmy[4];   // per 16-rank step: B's ranks 4t..4t+3 that are below r_n
    int em = 0, ecg = 0, ewpm = 1, nkb = 0;
    bool eactive = false;
    for (;; ++gi) {
        if (!gb_stage_wait(a, sm, gi, failed)) break;
        const int st = (int)(gi % (uint32_t)a.stages);
        const GbHdr *h = gb_hdr(sm, st);
        if (h->kind != GB_EXPAND) break;   // the end of the stream
        const uint32_t stg = sm.ring + (uint32_t)st * GB_SB;
        const int flags = h->flags;
        const int cnt = h->cnt, r_n = h->r_n, r8 = h->r8;
        if (flags & GB_FIRST) {   // a new item: s v fragments of this warp's m16 tile
            const int mtt = (cnt + 15) >> 4;
            const int mtp = mtt <= 1 ? 1 : (mtt <= 2 ? 2 : 4);
            ewpm = GB_CONSUMERS / mtp;
            em = warp % mtp;
            ecg = warp / mtp;
            eactive = em < mtt;
            nkb = (r_n + 15) >> 4;
#pragma unroll
            for (int kb = 0; kb < 4; ++kb) {
                const int keep = r_n - (kb * 16 + 4 * t);   // ranks of this thread's 4 below r_n
                bmx[kb] = keep >= 2 ? 0xffffffffu : (keep == 1 ? 0xffffu : 0u);
                bmy[kb] = keep >= 4 ? 0xffffffffu : (keep == 3 ? 0xffffu : 0u);
            }
            const float scale = h->scale;
#pragma unroll
            for (int kb = 0; kb < 4; ++kb) {
                float p[4] = {0.f, 0.f, 0.f, 0.f}, q[4] = {0.f, 0.f, 0.f, 0.f};
                const int k = kb * 16 + 4 * t;
                const int rg = 16 * em + g, rh = rg + 8;
                if (kb < nkb && k < r8) {
                    if (rg < cnt) {
                        const float4 v = lds128f(stg + (uint32_t)((rg * r8 + k) * 4));
                        p[0] = v.x; p[1] = v.y; p[2] = v.z; p[3] = v.w;
                    }
                    if (rh < cnt) {
                        const float4 v = lds128f(stg + (uint32_t)((rh * r8 + k) * 4));
                        q[0] = v.x; q[1] = v.y; q[2] = v.z; q[3] = v.w;
                    }
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    p[i] = k + i < r_n ? scale * p[i] : 0.f;
                    q[i] = k + i < r_n ? scale * q[i] : 0.f;
                }
                vhi[kb][0] = pack_bf16x2(p[0], p[1]);
                vhi[kb][1] = pack_bf16x2(q[0], q[1]);
                vhi[kb][2] = pack_bf16x2(p[2], p[3]);
                vhi[kb][3] = pack_bf16x2(q[2], q[3]);
                vlo[kb][0] = pack_bf16x2(p[0] - bf16_lo(vhi[kb][0]), p[1] - bf16_hi(vhi[kb][0]));
                vlo[kb][1] = pack_bf16x2(q[0] - bf16_lo(vhi[kb][1]), q[1] - bf16_hi(vhi[kb][1]));
                vlo[kb][2] = pack_bf16x2(p[2] - bf16_lo(vhi[kb][2]), p[3] - bf16_hi(vhi[kb][2]));
                vlo[kb][3] = pack_bf16x2(q[2] - bf16_lo(vhi[kb][3]), q[3] - bf16_hi(vhi[kb][3]));
            }
        }
        const int w = h->w;
        if (w > 0) {
            const int YS = 2 * h->cw + 16;
            const uint32_t ybase = stg + (uint32_t)h->yofs, bbase = stg + (uint32_t)h->bofs;
            const int nblk = w >> 3;
            if (eactive) {
                const int rg = 16 * em + g;
                const uint32_t yg_ad = ybase + (uint32_t)(rg * YS) + (uint32_t)(4 * t);
                const uint32_t yh_ad = yg_ad + (uint32_t)(8 * YS);
                const bool okg = rg < cnt, okh = rg + 8 < cnt;
                const int bf = ecg * 4, bs = 4 * ewpm;
#define LORA_EXPAND(RB, NKB)                                                                      \
    expand_warp<RB, NKB>(bbase, yg_ad, yh_ad, okg, okh, nblk, bf, bs, r8, vhi, vlo, bmx, bmy, g, t)
                if ((r8 & (r8 - 1)) == 0) {   // one box per 64 columns
                    if (r8 == 8) LORA_EXPAND(8, 1);
                    else if (r8 == 16) LORA_EXPAND(16, 1);
                    else if (r8 == 32) LORA_EXPAND(32, 2);
                    else LORA_EXPAND(64, 4);
                } else {                      // stacked 8-rank boxes: r8 = 24, 40, 48, 56
                    if (nkb == 2) LORA_EXPAND(0, 2);
                    else if (nkb == 3) LORA_EXPAND(0, 3);
                    else LORA_EXPAND(0, 4);
                }
#undef LORA_EXPAND
            }
            consumer_sync();
            const int ypc = w >> 3;
            const int s = h->s0;
            __nv_bfloat16 *ydst = a.y + a.sl.col_off[s] + h->c0;
            const unsigned char *yg =
                reinterpret_cast<const unsigned char *>(__cvta_shared_to_generic(ybase));
            for (int idx = tid; idx < cnt * ypc; idx += GB_CONSUMERS * 32) {
                const int r = idx / ypc, pc = idx - r * ypc;
                *reinterpret_cast<uint4 *>(ydst + (int64_t)h->rows[r] * a.ld_y + pc * 8) =
                    *reinterpret_cast<const uint4 *>(yg + r * YS + pc * 16);
            }
        }
        gb_release(sm, st);
    }
}

template <int MODE>
__device__ void gb_consumers(const GbArgs &a, const GbSmem &sm, bool &failed) {
    uint32_t gi = 0;
    if (MODE != MODE_EXPAND) gi = gb_consume_shrink<MODE>(a, sm, failed);
    if (MODE != MODE_SHRINK && !failed) gb_consume_expand<MODE>(a, sm, gi, failed);
}

// Persistent launch: clusters of C blocks; every block runs both phases.
template <int MODE>
__global__ void __launch_bounds__(GB_THREADS, 1) bgmv_kernel(const __grid_constant__ GbArgs a) {
    extern __shared__ __align__(128) unsigned char gb_sm[];
    const int tid = threadIdx.x;
    const uint32_t base = (smem_u32(gb_sm) + 1023u) & ~1023u;
    GbSmem sm;
    const int NS = a.stages;
    sm.ring = base;
    sm.hdr = sm.ring + (uint32_t)NS * GB_SB;
    uint32_t p = sm.hdr + (uint32_t)NS * GB_HDR;
    sm.recv = p;
    if (MODE != MODE_EXPAND) p += 2u * GB_XBUF * 4u;
    sm.part = p;
    if (MODE != MODE_EXPAND) p += GB_PART * 4u;
    sm.xrows = p;
    p += GB_ROWS * 4u;
    sm.tkslot = p;
    p += GB_TK * 4u;
    const uint32_t flag_s = p;
    p += 16u;
    p = (p + 7u) & ~7u;
    sm.full0 = p;
    sm.empty0 = p + 8u * GB_MAX_STAGES;
    sm.xready0 = p + 16u * GB_MAX_STAGES;
    sm.tkbar0 = sm.xready0 + 16u;
    sm.tkfree0 = sm.tkbar0 + 8u * GB_TK;
    sm.flag = reinterpret_cast<int *>(__cvta_shared_to_generic(flag_s));

    const int S = a.sl.n;
    const uint32_t C = cluster_size();
    if (tid == 0) {
        for (int st = 0; st < NS; ++st) {
            mbar_init(sm.full0 + 8 * st, 1);
            mbar_init(sm.empty0 + 8 * st, GB_CONSUMERS);
        }
        mbar_init(sm.xready0, 1);   // per exchange: the expect_tx arrival, then the partials' bytes
        mbar_init(sm.xready0 + 8, 1);
        for (int j = 0; j < GB_TK; ++j) {
            mbar_init(sm.tkbar0 + 8 * j, 1);
            mbar_init(sm.tkfree0 + 8 * j, C);   // used on cluster rank 0: one arrival per block
        }
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    if (tid >= GB_CONSUMERS * 32 && tid - GB_CONSUMERS * 32 < S) {   // descriptors this mode uses
        const int s = tid - GB_CONSUMERS * 32;
        for (int i = 0; i < 4; ++i) {
            if (MODE != MODE_EXPAND && (8 << i) <= a.r_max) prefetch_tmap(&a.tmA[s][i]);
            if (MODE != MODE_SHRINK && (8 << i) <= a.r_max) prefetch_tmap(&a.tmB[s][i]);
        }
    }
    cluster_barrier();   // barriers of every block initialised before any remote arrival

    bool failed = false;
    if (tid >= GB_CONSUMERS * 32)
        gb_producer<MODE>(a, sm, failed);
    else
        gb_consumers<MODE>(a, sm, failed);

    cluster_barrier();   // no block leaves while a peer may still write to it
    if (MODE == MODE_FUSED) {
        // the last block out puts the tickets and the per-unit counters back to zero
        if (tid == 0) {
            __threadfence();
            const int old = atomicAdd(a.ctl + GB_T_EXIT, 1);
            *sm.flag = old == (int)gridDim.x - 1;
        }
        __syncthreads();
        if (*sm.flag) {
            __threadfence();
            const int live = n_live_units(a.tiles);
            for (int u = tid; u < live; u += GB_THREADS) a.done[u] = 0;
            if (tid == 0) {
                a.ctl[GB_T_SHRINK] = 0;
                a.ctl[GB_T_EXPAND] = 0;
                a.ctl[GB_T_EXIT] = 0;
            }
        }
    }
}

namespace {

const void *gb_fn(int mode) {
    return mode == MODE_FUSED    ? (const void *)bgmv_kernel<MODE_FUSED>
           : mode == MODE_SHRINK ? (const void *)bgmv_kernel<MODE_SHRINK>
                                 : (const void *)bgmv_kernel<MODE_EXPAND>;
}

// Clusters of `cluster` blocks with `smem` bytes each that fit the device at once
// (0 if the query fails); the shared-memory limit is set once per device and mode.
int gb_active_clusters(int mode, int cluster, size_t smem) {
    struct Key {
        int dev, mode, cluster;
        size_t smem;
        int n;
    };
    static std::mutex mu;
    static Key cache[64];
    static int used = 0;
    int dev = 0;
    cudaGetDevice(&dev);
    {
        std::lock_guard<std::mutex> lock(mu);
        for (int i = 0; i < used; ++i)
            if (cache[i].dev == dev && cache[i].mode == mode && cache[i].cluster == cluster &&
                cache[i].smem == smem)
                return cache[i].n;
    }
    const void *fn = gb_fn(mode);
    int n = 0;
    // the limit is a per-device attribute of the kernel: always the mode's largest
    // launch, so no query for a smaller size can lower it under another launch
    const size_t smem_max = bgmv_smem_bytes(mode, mode == MODE_EXPAND ? GB_MAX_STAGES : 4);
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_max) ==
        cudaSuccess) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(cluster, 1, 1);
        cfg.blockDim = dim3(GB_THREADS, 1, 1);
        cfg.dynamicSmemBytes = smem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = cluster;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) != cudaSuccess) n = 0;
    }
    cudaGetLastError();   // a failed query must not surface as a later launch error
    std::lock_guard<std::mutex> lock(mu);
    if (used < 64) cache[used++] = Key{dev, mode, cluster, smem, n};
    return n;
}

}  // namespace

// Workspace of the fused mode: the control words (GB_CTL_INTS ints), one
// counter per unit, then v [S][T][r_max] fp32; each part 256-byte aligned.
size_t bgmv_workspace_bytes(int units, int T, int n_slices, int r_max) {
    const size_t head = (size_t)GB_CTL_INTS * 4 + (((size_t)units * 4 + 255) & ~(size_t)255);
    return head + (size_t)n_slices * (size_t)T * (size_t)r_max * 4;
}

// Persistent launch: as many clusters as fit the device at once.
int launch_bgmv(int mode, const GbArgs &args, int cluster, cudaStream_t st) {
    GbArgs a = args;
    // the exchange buffers of the shrink modes leave room for 4 stages; expand-only takes 6
    const int max_stages = mode == MODE_EXPAND ? GB_MAX_STAGES : 4;
    if (a.stages < 2 || a.stages > max_stages) a.stages = GB_STAGES_DEFAULT;
    const size_t smem = bgmv_smem_bytes(mode, a.stages);
    int clusters = gb_active_clusters(mode, cluster, smem);
    if (clusters < 1) {
        int dev = 0, sms = 148;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        clusters = sms / cluster > 0 ? sms / cluster : 1;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(cluster * clusters, 1, 1);
    cfg.blockDim = dim3(GB_THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t err;
    if (mode == MODE_FUSED)
        err = cudaLaunchKernelEx(&cfg, bgmv_kernel<MODE_FUSED>, a);
    else if (mode == MODE_SHRINK)
        err = cudaLaunchKernelEx(&cfg, bgmv_kernel<MODE_SHRINK>, a);
    else
        err = cudaLaunchKernelEx(&cfg, bgmv_kernel<MODE_EXPAND>, a);
    return cuda_rc(err);
}

}  // namespace lora
