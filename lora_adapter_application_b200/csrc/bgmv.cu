// Fused decode BGMV (page "Multi-LoRA Serving", section 3.2: BGMV-style
// grouped products; section 3.4: add_shrink then add_expand, grouped per
// adapter) for bf16, ranks up to 64.
//
// One unit of work = up to 16 rows that share an adapter (a gathered tile, or
// 16 rows of a contiguous tile).  A cluster of C thread blocks takes a unit;
// block c owns 1/C of the input columns (shrink) and 1/C of the output
// columns (expand).  Clusters are persistent: cluster k walks the units k,
// k + #clusters, ... of those counted on the device.  Each block is
// warp-specialised:
//
//   producer warp   walks the block's chunk stream and fills a 72 KB
//                   shared-memory ring (3 or 2 stages) through the TMA engine: 2-D tensor
//                   copies of 1-2 KB boxes for the adapters (A: 8 or 16 ranks
//                   x 64 columns, 128-byte swizzle; B: 64 output columns x 8
//                   or 16 ranks) and one 1-D bulk copy per gathered x or y
//                   row piece.  (Measured on B200: TMA copies leave the
//                   load/store pipe to the consumers, where a cp.async
//                   producer competes with their shared-memory traffic; TMA
//                   pays per copy, so copies should be 1 KB or more.)  A
//                   full/empty mbarrier pair guards each stage.
//   8 consumer warps
//     shrink chunks  x rows [cnt][JC] and A rows [r_n][JC] -> partial v
//                    (tensor-core mma m16n8k16, bf16 in, fp32 accumulate)
//     exchange       through distributed shared memory, stores only: every
//                    block sends each partial element to the block that owns
//                    it; the owner adds the C partials in a fixed order
//                    (run-to-run identical), scales by alpha/r_n and stores the
//                    result into every block's copy of v; the stores are
//                    st.async, counted in bytes on the receiver's mbarrier, so
//                    neither side needs a cluster-scope fence
//     expand chunks  B rows [CC][r_n] and y rows [cnt][CC] -> y += (s v) B^T in
//                    fp32, rounded once, written back with 16-byte stores
//
// The producer runs a ring's worth of chunks ahead, across the exchange, so HBM stays
// busy; every byte of x, A, B and y crosses HBM once and v never leaves the
// chip.  s v enters the expand products as a bf16 hi + lo pair (about 16
// mantissa bits): a single bf16 copy (2^-9 relative) is not enough when the
// delta is large and cancels against y.  The multiply-adds (about 4 per byte)
// run on the tensor pipe.  Large batches are bounded by HBM bandwidth; a
// small decode batch is latency-bound: each unit is a chain of dependent
// loads, the exchange and the expand, a few microseconds each.
//
// Inside one 16-wide K step each thread assigns 4 consecutive elements of each
// operand row to its four k-slots of the mma fragment; both operands use the
// same assignment, so the sum is unchanged and shared-memory reads are vectors.
//
// Every wait is bounded (a suspend-time hint per try, and a try limit): a wait
// that runs out sets LORA_DEV_TIMEOUT in the status word and the block skips
// its remaining work instead of hanging.
#include "kernels.cuh"
#include "ptx.cuh"

#include <cooperative_groups.h>

#include <cstdlib>

#include <mutex>

namespace cg = cooperative_groups;

namespace lora {

constexpr int BG_CONSUMERS = 8;                      // consumer warps
constexpr int BG_THREADS = (BG_CONSUMERS + 1) * 32;  // + 1 producer warp
constexpr int BG_ROWS = 16;
constexpr int BG_RMAX = 64;
constexpr int BG_MAX_STAGES = 3;                    // mbarrier pairs reserved
constexpr int BG_RING_BYTES = 73728;                // 3 x 24 KB or 2 x 36 KB (1 KB multiples)
constexpr int BG_VF_STRIDE = 80;   // floats per row of the reduced v (bank spread)


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
    asm volatile("bar.sync 1, %0;\n" ::"n"(BG_CONSUMERS * 32) : "memory");
}

__device__ __forceinline__ uint4 zero_if(bool z, uint4 v) { return z ? make_uint4(0, 0, 0, 0) : v; }

// Shared memory: ring | recv [S*16*64] | vfull [S][16][80] | part [16][64] | barriers
//   recv[c*(S*1024/C) + e/C] holds block c's partial of element e = (s*16+row)*64+k,
//   for the elements e with e % C == this block's rank.
size_t bgmv_smem_bytes(int n_slices) {
    return 1024 /* alignment of the ring to the 128-byte swizzle atom */ +
           (size_t)BG_RING_BYTES + (size_t)n_slices * BG_ROWS * BG_RMAX * 4 +
           (size_t)n_slices * BG_ROWS * BG_VF_STRIDE * 4 + (size_t)BG_ROWS * BG_RMAX * 4 + 128;
}

struct Geo {          // chunk geometry of one block for one unit
    int r8, nb8, nkb16;
    int j_lo, j_hi, JC, RS, A0, n_sc;    // shrink: columns, chunk width, x row stride, A boxes offset, chunks/slice
    int c_lo, c_hi, CC, YS, B0;          // expand: concatenated column range, chunk width, y row stride, B boxes offset
    int n_shrink, n_chunks;
};

// Shared-memory bytes of a chunk `cols` columns wide: 16 bf16 rows of x or y
// (padded by 16 bytes, 1 KB aligned), then the adapter boxes, which hold per
// 64 columns one 1 KB box per 8 ranks, or one 2 KB box per 16 ranks (ab16).
__device__ __forceinline__ int chunk_bytes(int cols, int nb8, bool ab16) {
    const int box_kb = ab16 ? 2 * ((nb8 + 1) >> 1) : nb8;   // per 64 columns
    return ((BG_ROWS * (cols * 2 + 16) + 1023) & ~1023) + box_kb * (cols >> 6) * 1024;
}

// Position in a block's chunk stream, advanced without divisions: shrink
// chunks slice by slice, then expand chunks slice by slice.
struct ChunkIt {
    int i;                 // chunk index
    int s, q;              // shrink: slice, chunk in slice
    int es, c0, w;         // expand: slice, first slice-local column, width
};

// Shared-memory carve-up of a block (the same for every unit it takes).
struct BgSmem {
    unsigned char *ring;
    float *recv, *vfull, *part;
    int *rows;
    uint32_t ring_s, full0, empty0, xready, vready;
};

// One unit on one block of its cluster.  `base`: chunks this block streamed
// through the ring for earlier units (slot and phase of every chunk follow
// from base + its index); `uiter`: units this block took before (phase of the
// exchange barriers).  Returns the unit's chunk count.
template <int MODE>
__device__ __forceinline__ uint32_t bgmv_unit(const BgArgs &a, const BgSmem &sm, const Unit &u,
                                              int r_n, uint32_t base, uint32_t uiter,
                                              bool &failed) {
    const int S = a.sl.n;
    unsigned char *ring = sm.ring;
    float *recv = sm.recv, *vfull = sm.vfull, *part = sm.part;
    const int *rows_sm = sm.rows;
    const uint32_t ring_s = sm.ring_s, full0 = sm.full0, empty0 = sm.empty0;
    const uint32_t xready = sm.xready, vready = sm.vready;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int C = gridDim.x, crank = blockIdx.x;
    const int n = u.id;
    const int cnt = u.cnt;

    // ------------------------------------------------------------ geometry
    const int NS = a.stages == 2 ? 2 : 3;                   // ring stages
    const int SB = BG_RING_BYTES / NS;                      // bytes per stage
    Geo G;
    G.r8 = (r_n + 7) & ~7;
    G.nb8 = G.r8 >> 3;
    G.nkb16 = (r_n + 15) >> 4;
    if (MODE != MODE_EXPAND) {
        const int n64 = (a.d_in + 63) >> 6;
        G.j_lo = (int)((int64_t)crank * n64 / C) * 64;
        G.j_hi = min((int)((int64_t)(crank + 1) * n64 / C) * 64, a.d_in);
        // widest power-of-two chunk (>= 64 columns) whose x rows and A boxes fit a stage
        int jc = 64;
        while (chunk_bytes(jc * 2, G.nb8, a.ab16) <= SB) jc *= 2;
        const int span = max(0, G.j_hi - G.j_lo);
        while (jc > 64 && jc / 2 >= span) jc /= 2;
        G.JC = jc;
        G.RS = G.JC * 2 + 16;
        G.A0 = (BG_ROWS * G.RS + 1023) & ~1023;
        G.n_sc = (span + G.JC - 1) / G.JC;
    } else {
        G.j_lo = G.j_hi = 0;
        G.JC = 64;
        G.RS = 144;
        G.A0 = 0;
        G.n_sc = 0;
    }
    G.n_shrink = S * G.n_sc;
    G.n_chunks = G.n_shrink;
    if (MODE != MODE_SHRINK) {
        const int n8 = a.sl.cat_off[S] >> 3;
        G.c_lo = (int)((int64_t)crank * n8 / C) * 8;
        G.c_hi = (int)((int64_t)(crank + 1) * n8 / C) * 8;
        // widest power-of-two chunk (>= 64 columns) whose y rows and B boxes fit a stage
        int cc = 64;
        while (chunk_bytes(cc * 2, G.nb8, a.ab16) <= SB) cc *= 2;
        G.CC = cc;
        G.YS = G.CC * 2 + 16;   // 16 (mod 128) bytes: the 8 rows of an mma tile hit 8 bank groups
        G.B0 = (BG_ROWS * G.YS + 1023) & ~1023;
        for (int s = 0; s < S; ++s) {
            const int lo = max(G.c_lo, a.sl.cat_off[s]), hi = min(G.c_hi, a.sl.cat_off[s + 1]);
            if (hi > lo) G.n_chunks += (hi - lo + G.CC - 1) / G.CC;
        }
    } else {
        G.c_lo = G.c_hi = 0;
        G.CC = 64;
        G.YS = 144;
        G.B0 = 0;
    }

    // next position of the chunk stream
    auto advance = [&](ChunkIt &it) {
        ++it.i;
        if (it.i < G.n_shrink) {
            if (++it.q == G.n_sc) {
                it.q = 0;
                ++it.s;
            }
            return;
        }
        if (it.i >= G.n_chunks) return;
        if (it.es >= 0) {   // next block of columns in this slice?
            const int hi = min(G.c_hi, a.sl.cat_off[it.es + 1]) - a.sl.cat_off[it.es];
            if (it.c0 + G.CC < hi) {
                it.c0 += G.CC;
                it.w = min(G.CC, hi - it.c0);
                return;
            }
        }
        for (int s = it.es + 1; s < S; ++s) {   // first later slice with columns in this block
            const int lo = max(G.c_lo, a.sl.cat_off[s]), hi = min(G.c_hi, a.sl.cat_off[s + 1]);
            if (hi > lo) {
                it.es = s;
                it.c0 = lo - a.sl.cat_off[s];
                it.w = min(G.CC, hi - lo);
                return;
            }
        }
    };
    auto first = [&](ChunkIt &it) {
        it.i = 0;
        it.s = it.q = 0;
        it.es = -1;
        it.c0 = it.w = 0;
        if (G.n_shrink == 0 && G.n_chunks > 0) {   // the stream starts with expand chunks
            it.i = -1;
            advance(it);
        }
    };


    if (warp == BG_CONSUMERS) {
        // ============================================================ producer
        ChunkIt it;
        first(it);
        for (; it.i < G.n_chunks; advance(it)) {
            const uint32_t gi = base + (uint32_t)it.i;   // position in the block's ring stream
            const int st = (int)(gi % (uint32_t)NS);
            const uint32_t full = full0 + 8 * st, dst = ring_s + st * SB;
            if (gi >= (uint32_t)NS)
                mbar_wait(empty0 + 8 * st, ((gi / NS) - 1) & 1, a.status, failed);
            if (failed) break;
            if (it.i < G.n_shrink) {
                const int jc0 = G.j_lo + it.q * G.JC;
                const int width = min(G.JC, G.j_hi - jc0), nbox = (width + 63) >> 6;
                const int ncb = G.JC >> 6;
                const unsigned xbytes = (unsigned)width * 2;
                const int nkg = a.ab16 ? (G.nb8 + 1) >> 1 : G.nb8;   // rank boxes
                const unsigned abox = a.ab16 ? 2048u : 1024u;
                if (lane == 0) mbar_expect_tx(full, xbytes * cnt + (unsigned)(nkg * nbox) * abox);
                __syncwarp();
                for (int r = lane; r < cnt; r += 32)   // gathered x rows
                    bulk_g2s(dst + r * G.RS, a.x + (int64_t)rows_sm[r] * a.ld_x + jc0, xbytes, full);
                for (int e = lane; e < nkg * nbox; e += 32) {   // A: 8 or 16 ranks x 64 columns per box
                    const int kg = e / nbox, cb = e - kg * nbox;
                    tma_2d(dst + G.A0 + (kg * ncb + cb) * abox, &a.tmA[it.s], jc0 + 64 * cb,
                           n * a.r_max + (a.ab16 ? 16 : 8) * kg, full);
                }
            } else {
                const int s = it.es, d_out = a.sl.d_out[s];
                const int nbox = (it.w + 63) >> 6, nbx = G.CC >> 6;
                const unsigned ybytes = (unsigned)it.w * 2;
                const int nkg = a.ab16 ? (G.nb8 + 1) >> 1 : G.nb8;
                const unsigned bbox = a.ab16 ? 2048u : 1024u;
                if (lane == 0) mbar_expect_tx(full, ybytes * cnt + (unsigned)(nkg * nbox) * bbox);
                __syncwarp();
                for (int r = lane; r < cnt; r += 32)   // gathered y rows
                    bulk_g2s(dst + r * G.YS,
                             a.y + (int64_t)rows_sm[r] * a.ld_y + a.sl.col_off[s] + it.c0, ybytes, full);
                for (int e = lane; e < nkg * nbox; e += 32) {   // B: 64 columns x 8 or 16 ranks per box
                    const int kg = e / nbox, cb = e - kg * nbox;
                    tma_2d(dst + G.B0 + (kg * nbx + cb) * bbox, &a.tmB[s], (a.ab16 ? 16 : 8) * kg,
                           n * d_out + it.c0 + 64 * cb, full);
                }
            }
        }
        return (uint32_t)G.n_chunks;
    }

    // ================================================================ consumers
    const int jg = max(1, BG_CONSUMERS / G.nb8);   // warps per 8-rank block
    const bool shrink_warp = warp < G.nb8 * jg;
    const int nbw = warp / jg, jgi = warp - (warp / jg) * jg;
    float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
    const int ctid = tid;   // 0 .. 255
    const int per_src = (S * BG_ROWS * BG_RMAX) / C;
    const uint32_t recv_s = smem_u32(recv), vfull_s = smem_u32(vfull);
    // Exchange rounds: st.async stores that count their bytes on the receiver's
    // barrier (no fence on either side).  With C dividing 64, every block
    // receives S * cnt * r8 partials (4 bytes each) in either round: the
    // elements it owns from every block, then every owner's scaled sums.
    if (MODE != MODE_EXPAND && ctid == 0) {
        const unsigned bytes = (unsigned)(S * cnt * G.r8) * 4u;
        mbar_expect_tx(xready, bytes);
        if (MODE == MODE_FUSED) mbar_expect_tx(vready, bytes);
    }

    // block partial of slice s (from part, or zeros) -> recv of the owning block
    auto send_partials = [&](int s, bool from_part) {
        for (int idx = ctid; idx < cnt * G.r8; idx += BG_CONSUMERS * 32) {
            const int row = idx / G.r8, k = idx - row * G.r8;
            float sum = 0.f;
            if (from_part)
                for (int j = 0; j < jg; ++j) sum += part[(j * BG_ROWS + row) * G.r8 + k];
            const int e = (s * BG_ROWS + row) * BG_RMAX + k;
            const uint32_t owner = (uint32_t)(e % C);
            st_async_f32(map_rank(recv_s + (uint32_t)(crank * per_src + e / C) * 4u, owner), sum,
                         map_rank(xready, owner));
        }
    };

    auto shrink_chunk = [&](const ChunkIt &it, uint32_t st) {
        if (shrink_warp) {
            const int jc0 = G.j_lo + it.q * G.JC;
            const int width = min(G.JC, G.j_hi - jc0);
            const int nsteps = (width + 63) >> 6;
            const uint32_t xg = st + g * G.RS, xh = st + (g + 8) * G.RS;
            // A box (8 or 16 ranks x 64 columns, 128-byte swizzle): rank 8 nbw + g, 16-byte
            // chunks 2t and 2t+1 (the swizzle follows address bits 7-9, the same in either box)
            const uint32_t ak = a.ab16 ? st + G.A0 + (nbw >> 1) * (G.JC >> 6) * 2048 + (nbw & 1) * 1024 + g * 128
                                       : st + G.A0 + nbw * (G.JC >> 6) * 1024 + g * 128;
            const uint32_t astep = a.ab16 ? 2048u : 1024u;
            const uint32_t c0 = (uint32_t)(((2 * t) ^ g) << 4), c1 = (uint32_t)(((2 * t + 1) ^ g) << 4);
            for (int sp = jgi; sp < nsteps; sp += jg) {
                const int col = sp * 64 + t * 16;
                const bool z0 = col >= width, z1 = col + 8 >= width;   // beyond the chunk: zero
                const uint32_t off = (uint32_t)(col * 2);
                const uint4 xa0 = zero_if(z0, lds128(xg + off)), xa1 = zero_if(z1, lds128(xg + off + 16));
                const uint4 xb0 = zero_if(z0, lds128(xh + off)), xb1 = zero_if(z1, lds128(xh + off + 16));
                const uint32_t box = ak + sp * astep;
                const uint4 a0 = zero_if(z0, lds128(box + c0)), a1 = zero_if(z1, lds128(box + c1));
                {
                    const uint32_t f[4] = {xa0.x, xb0.x, xa0.y, xb0.y};
                    mma16816(acc0, f, a0.x, a0.y);
                }
                {
                    const uint32_t f[4] = {xa0.z, xb0.z, xa0.w, xb0.w};
                    mma16816(acc1, f, a0.z, a0.w);
                }
                {
                    const uint32_t f[4] = {xa1.x, xb1.x, xa1.y, xb1.y};
                    mma16816(acc0, f, a1.x, a1.y);
                }
                {
                    const uint32_t f[4] = {xa1.z, xb1.z, xa1.w, xb1.w};
                    mma16816(acc1, f, a1.z, a1.w);
                }
            }
        }
        if (it.q == G.n_sc - 1) {   // slice done: block partial -> owners
            consumer_sync();        // every warp is past its reads of part from the last slice
            if (shrink_warp) {
                const int k = nbw * 8 + 2 * t;
                part[(jgi * BG_ROWS + g) * G.r8 + k] = acc0[0] + acc1[0];
                part[(jgi * BG_ROWS + g) * G.r8 + k + 1] = acc0[1] + acc1[1];
                part[(jgi * BG_ROWS + g + 8) * G.r8 + k] = acc0[2] + acc1[2];
                part[(jgi * BG_ROWS + g + 8) * G.r8 + k + 1] = acc0[3] + acc1[3];
#pragma unroll
                for (int e = 0; e < 4; ++e) acc0[e] = acc1[e] = 0.f;
            }
            consumer_sync();
            send_partials(it.s, true);
        }
    };

    auto exchange = [&]() {
        if (MODE == MODE_EXPAND) {
            const float scale = a.scales[n];
            for (int e = ctid; e < S * BG_ROWS * BG_RMAX; e += BG_CONSUMERS * 32) {
                const int s = e >> 10, rem = e & 1023;
                const int row = rem >> 6, k = rem & 63;
                if (row < cnt && k < G.r8)
                    vfull[(s * BG_ROWS + row) * BG_VF_STRIDE + k] =
                        k < r_n ? scale * a.v[((int64_t)s * a.T + rows_sm[row]) * a.r_max + k] : 0.f;
            }
            consumer_sync();
            return;
        }
        if (G.n_sc == 0)   // no input columns here: the partials are zero
            for (int s = 0; s < S; ++s) send_partials(s, false);
        mbar_wait(xready, uiter & 1u, a.status, failed);   // every partial has reached its owner
        const float scale = MODE == MODE_FUSED ? a.scales[n] : 1.f;
        const int mine = (S * BG_ROWS * BG_RMAX - crank + C - 1) / C;   // elements e = crank + C*j
        for (int j = ctid; j < mine; j += BG_CONSUMERS * 32) {
            const int e = crank + C * j;
            const int s = e >> 10, rem = e & 1023;
            const int row = rem >> 6, k = rem & 63;
            if (row >= cnt || k >= G.r8) continue;
            float sum = 0.f;
            for (int c = 0; c < C; ++c) sum += recv[c * per_src + j];
            const float val = k < r_n ? scale * sum : 0.f;
            if (MODE == MODE_SHRINK) {
                if (k < r_n) a.v[((int64_t)s * a.T + rows_sm[row]) * a.r_max + k] = val;
            } else {
                const uint32_t f = vfull_s + (uint32_t)((s * BG_ROWS + row) * BG_VF_STRIDE + k) * 4u;
                for (int c = 0; c < C; ++c) st_async_f32(map_rank(f, (uint32_t)c), val, map_rank(vready, (uint32_t)c));
            }
        }
        if (MODE == MODE_FUSED)
            mbar_wait(vready, uiter & 1u, a.status, failed);   // every block holds the full s*v
    };

    int cur_s = -1;
    uint32_t ahi[4][4], alo[4][4];
    auto expand_chunk = [&](const ChunkIt &it, uint32_t st) {
        const int s = it.es;
        if (s != cur_s) {   // mma fragments of s*v (bf16 hi + lo) for this slice
            cur_s = s;
            const float *vf = vfull + s * BG_ROWS * BG_VF_STRIDE;
#pragma unroll
            for (int kb = 0; kb < 4; ++kb) {
                const float4 p = *reinterpret_cast<const float4 *>(&vf[g * BG_VF_STRIDE + kb * 16 + 4 * t]);
                const float4 q =
                    *reinterpret_cast<const float4 *>(&vf[(g + 8) * BG_VF_STRIDE + kb * 16 + 4 * t]);
                ahi[kb][0] = pack_bf16x2(p.x, p.y);
                ahi[kb][1] = pack_bf16x2(q.x, q.y);
                ahi[kb][2] = pack_bf16x2(p.z, p.w);
                ahi[kb][3] = pack_bf16x2(q.z, q.w);
                alo[kb][0] = pack_bf16x2(p.x - bf16_lo(ahi[kb][0]), p.y - bf16_hi(ahi[kb][0]));
                alo[kb][1] = pack_bf16x2(q.x - bf16_lo(ahi[kb][1]), q.y - bf16_hi(ahi[kb][1]));
                alo[kb][2] = pack_bf16x2(p.z - bf16_lo(ahi[kb][2]), p.w - bf16_hi(ahi[kb][2]));
                alo[kb][3] = pack_bf16x2(q.z - bf16_lo(ahi[kb][3]), q.w - bf16_hi(ahi[kb][3]));
            }
        }
        const int nblk = it.w >> 3;
        const uint32_t bbase = st + G.B0, nbx = G.CC >> 6;
        for (int nb0 = warp * 2; nb0 < nblk; nb0 += BG_CONSUMERS * 2) {
            float d[2][4];
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) d[j][e] = 0.f;
#pragma unroll
            for (int kb = 0; kb < 4; ++kb) {
                if (kb < G.nkb16) {
                    const int k = kb * 16 + 4 * t;
                    uint2 bv[2];
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        bv[j] = make_uint2(0, 0);
                        if (k < r_n && nb0 + j < nblk) {
                            const int col = (nb0 + j) * 8 + g;   // B box: 64 columns x 8 (16) ranks
                            bv[j] = a.ab16 ? lds64(bbase + ((k >> 4) * nbx + (col >> 6)) * 2048 +
                                                   (col & 63) * 32 + (k & 15) * 2)
                                           : lds64(bbase + ((k >> 3) * nbx + (col >> 6)) * 1024 +
                                                   (col & 63) * 16 + (k & 7) * 2);
                            if (k + 4 > r_n) {   // the rank ends inside this group of 4
                                const int keep = r_n - k;
                                if (keep < 2) bv[j].x &= 0xffffu;
                                if (keep < 3) bv[j].y = 0;
                                else bv[j].y &= 0xffffu;
                            }
                        }
                    }
#pragma unroll
                    for (int j = 0; j < 2; ++j) mma16816(d[j], ahi[kb], bv[j].x, bv[j].y);
#pragma unroll
                    for (int j = 0; j < 2; ++j) mma16816(d[j], alo[kb], bv[j].x, bv[j].y);
                }
            }
            // y += delta in shared memory (rows g and g+8, columns 2t, 2t+1 of each 8-column block)
            const uint32_t yg = st + g * G.YS + (nb0 * 8 + 2 * t) * 2;
            const uint32_t yh = yg + 8 * G.YS;
            uint32_t y0[2], y1[2];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const bool ok = nb0 + j < nblk;
                y0[j] = (ok && g < cnt) ? lds32(yg + j * 16) : 0u;
                y1[j] = (ok && g + 8 < cnt) ? lds32(yh + j * 16) : 0u;
            }
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                if (nb0 + j < nblk) {
                    if (g < cnt)
                        sts32(yg + j * 16, pack_bf16x2(bf16_lo(y0[j]) + d[j][0], bf16_hi(y0[j]) + d[j][1]));
                    if (g + 8 < cnt)
                        sts32(yh + j * 16, pack_bf16x2(bf16_lo(y1[j]) + d[j][2], bf16_hi(y1[j]) + d[j][3]));
                }
            }
        }
        consumer_sync();
        const int ypc = it.w >> 3;
        const unsigned char *stp = ring + (st - ring_s);
        for (int r = warp; r < cnt; r += BG_CONSUMERS) {
            __nv_bfloat16 *dst = a.y + (int64_t)rows_sm[r] * a.ld_y + a.sl.col_off[s] + it.c0;
            for (int pc = lane; pc < ypc; pc += 32)
                *reinterpret_cast<uint4 *>(dst + pc * 8) =
                    *reinterpret_cast<const uint4 *>(stp + r * G.YS + pc * 16);
        }
    };

    ChunkIt it;
    first(it);
    bool exchanged = false;
    for (; it.i < G.n_chunks; advance(it)) {
        const uint32_t gi = base + (uint32_t)it.i;
        const int st = (int)(gi % (uint32_t)NS);
        const uint32_t sta = ring_s + st * SB;
        if (!exchanged && it.i >= G.n_shrink) {
            exchange();
            exchanged = true;
        }
        const bool ready = mbar_wait(full0 + 8 * st, (gi / NS) & 1, a.status, failed);
        if (ready) {
            if (it.i < G.n_shrink)
                shrink_chunk(it, sta);
            else
                expand_chunk(it, sta);
        }
        asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(empty0 + 8 * st);
    }
    if (!exchanged) exchange();
    return (uint32_t)G.n_chunks;
}

// Persistent clusters: cluster k takes the live units k, k + #clusters, ...
template <int MODE>
__global__ void __launch_bounds__(BG_THREADS, 2) bgmv_kernel(const __grid_constant__ BgArgs a) {
    extern __shared__ __align__(128) unsigned char bg_sm[];
    __shared__ int rows_sm[BG_ROWS];

    const int S = a.sl.n;
    BgSmem sm;
    // ring on a 1 KB boundary: swizzled TMA boxes need their 1 KB atom aligned
    sm.ring = bg_sm + ((1024u - (smem_u32(bg_sm) & 1023u)) & 1023u);
    sm.recv = reinterpret_cast<float *>(sm.ring + BG_RING_BYTES);
    sm.vfull = sm.recv + S * BG_ROWS * BG_RMAX;
    sm.part = sm.vfull + S * BG_ROWS * BG_VF_STRIDE;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm.part + BG_ROWS * BG_RMAX);
    sm.rows = rows_sm;
    sm.ring_s = smem_u32(sm.ring);
    sm.full0 = smem_u32(bars);
    sm.empty0 = sm.full0 + 8 * BG_MAX_STAGES;
    sm.xready = sm.full0 + 16 * BG_MAX_STAGES;
    sm.vready = sm.xready + 8;

    const int tid = threadIdx.x;
    if (tid >= BG_CONSUMERS * 32 && tid - BG_CONSUMERS * 32 < S) {   // producer lanes: descriptors
        const int s = tid - BG_CONSUMERS * 32;
        if (MODE != MODE_EXPAND) prefetch_tmap(&a.tmA[s]);   // only the maps this mode built
        if (MODE != MODE_SHRINK) prefetch_tmap(&a.tmB[s]);
    }
    if (tid == 0) {
        for (int st = 0; st < BG_MAX_STAGES; ++st) {
            mbar_init(sm.full0 + 8 * st, 1);
            mbar_init(sm.empty0 + 8 * st, BG_CONSUMERS);
        }
        mbar_init(sm.xready, 1);   // per unit: the expect_tx arrival, then C x the owned partials' bytes
        mbar_init(sm.vready, 1);
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    cg::cluster_group cluster = cg::this_cluster();

    // Every block of a cluster walks the same units and takes the same branches,
    // so the cluster barriers below always pair up; a block whose wait ran out
    // keeps walking (its waits then return at once) instead of leaving early.
    bool failed = false;
    uint32_t base = 0, uiter = 0;
    const int live = n_live_units(a.tiles);
    for (int v = blockIdx.y; v < live; v += gridDim.y) {
        const Unit u = resolve_live_unit(a.tiles, v);
        if (u.cnt == 0) continue;
        const int r_n = a.ranks[u.id];
        if (r_n < 1 || r_n > a.r_max) {
            if (blockIdx.x == 0 && tid == 0) atomicOr(a.status, LORA_DEV_BAD_RANK);
            continue;
        }
        if (uiter > 0) cluster.sync();   // the previous unit is done in every block
        if (tid < BG_ROWS) rows_sm[tid] = tid < u.cnt ? u.row(a.tiles, tid) : -1;
        for (int e = tid; e < S * BG_ROWS * BG_VF_STRIDE; e += BG_THREADS) sm.vfull[e] = 0.f;
        cluster.sync();                  // barriers, rows and zeroed s*v ready in every block
        base += bgmv_unit<MODE>(a, sm, u, r_n, base, uiter, failed);
        ++uiter;
    }
    cluster.sync();   // no block leaves while a peer may still write to it
}

namespace {

const void *bg_fn(int mode) {
    return mode == MODE_FUSED    ? (const void *)bgmv_kernel<MODE_FUSED>
           : mode == MODE_SHRINK ? (const void *)bgmv_kernel<MODE_SHRINK>
                                 : (const void *)bgmv_kernel<MODE_EXPAND>;
}

// Clusters of `cluster` blocks with `smem` bytes each that fit the device at once
// (0 if the query fails).
int bg_active_clusters(int mode, int cluster, size_t smem) {
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
    const void *fn = bg_fn(mode);
    int n = 0;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)bgmv_smem_bytes(LORA_MAX_SLICES)) == cudaSuccess) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(cluster, 1, 1);
        cfg.blockDim = dim3(BG_THREADS, 1, 1);
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

// Persistent launch: as many clusters as fit the device at once (at most one
// per unit of the tile-list capacity); each walks the live units.
int launch_bgmv(int mode, const BgArgs &args, int n_units, int cluster, cudaStream_t st) {
    if (n_units <= 0) return LORA_OK;
    // Two 36 KB stages: chunks twice as wide as with three 24 KB stages up to rank
    // 48 (half the gathered-row copies), and the whole shrink stream of a decode
    // unit in flight at once.  Measured on B200 (graph-timed): decode q_proj
    // kernel 21.8 us against 24.8 with three stages; Llama-3-8B layer set at
    // decode 583 against 587 us.
    BgArgs a = args;
    a.stages = 2;
    if (const char *e = std::getenv("LORA_BG_STAGES"))   // tuning override: 2 or 3
        if (std::atoi(e) == 3) a.stages = 3;
    const size_t smem = bgmv_smem_bytes(a.sl.n);
    int clusters = bg_active_clusters(mode, cluster, smem);
    if (clusters < 1) {
        int dev = 0, sms = 148;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        clusters = sms / cluster > 0 ? sms / cluster : 1;
    }
    clusters = clusters < n_units ? clusters : n_units;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(cluster, clusters, 1);
    cfg.blockDim = dim3(BG_THREADS, 1, 1);
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
