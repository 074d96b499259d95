// Gathered-tile kernel on the 5th-generation tensor cores (sm_100a), fused
// shrink and expand of one linear layer: page "Multi-LoRA Serving", section
// 3.4 (add_shrink then add_expand, one batched call), with the rows of a
// batch grouped per adapter into units of at most 16 rows (section 3.2: the
// rows that share an adapter form a segment).
//
// For a unit of cnt <= 16 rows with adapter n and rank r_n, and a slice s:
//   shrink  D1[128 ranks][16 rows]  = A_s[n] . X^T          (K = d_in)
//   expand  D2[128 cols][16 rows]   = B_s[n][cols] . (s_n v)^T   (K = r_n)
// both as tcgen05.mma kind::f16 with M = 128, N = 16: the ranks (shrink) or
// 128 output columns (expand) run along M, the unit's rows along N, so a
// unit of one row costs the same operand bytes as one of sixteen, and the
// tensor core's unused lanes cost nothing that matters (the layer is bound
// by HBM).  s_n = alpha_n / r_n.
//
// Work items, taken from atomic tickets in the workspace by a persistent grid
// of BT_BLOCKS_PER_SM (2) blocks per SM:
//   shrink item  (unit, slice): streams A_s[n] (its r_n rank rows) and the
//                unit's x rows in 64-column chunks; writes s_n v as a bf16
//                hi + lo pair (about 16 mantissa bits) to the workspace and
//                counts the unit's done word up.
//   expand item  (unit, slice, `bc` output columns = bc/128 tiles): waits for
//                the unit's done word, adds D2 to the unit's y rows.
// Every block takes shrink tickets until they run out, then expand tickets:
// a shrink item is held only by a running block, whose pipeline finishes it
// without waiting on anything, so every wait on a done word ends.
//
// Warp roles (192 threads):
//   warp 0     producer: tickets, item records, and every copy.  By TMA tensor
//              copies: A, one box per 256-column stage (4 chunks of 64 columns x
//              the item's ranks rounded to 8, 128-byte swizzle; 64 x 8-rank boxes
//              when d_in is not a multiple of 64), B boxes (8 ranks x 128
//              columns) and y rows (four rows of 128 columns a copy,
//              tile::gather4).  x rows by cp.async into the swizzled layout (one
//              16-byte piece per lane); s_n v by a bulk copy once the unit is done.
//   warp 1     tensor-memory allocator and MMA issuer (one thread issues).
//   warps 2-5  epilogue: tensor memory -> registers (lane = rank or output
//              column), then v to the workspace, or y + D2 rounded once to
//              bf16 and written straight to the unit's rows (64 contiguous
//              bytes per warp and row).
//
// Shared memory holds two byte rings with in-order reuse, operands (A and x
// chunks, B tiles) and y tiles, and a few fixed slots for v pairs.  Allocations are variable in size,
// so small ranks and short units still keep ~100 KB in flight per SM.  Each
// allocation owns a full/empty mbarrier pair; a y tile goes back to the
// producer as soon as the epilogue has read it.
//
// Padding never reaches a sum: A rows past r_n only fill accumulator lanes
// that are not read, x rows past cnt only fill accumulator columns that are
// not read, B ranks past r_n are zeroed in shared memory (r_n % 8 != 0) or
// come from a zero buffer (the upper half of a k16 step when r_n rounds to an
// odd number of 8-rank groups), and v is written as zero there.
//
// Every wait is bounded (LORA_DEV_TIMEOUT in the status word when one runs
// out; an expand item whose unit never finishes is dropped, and its block
// takes no more tickets).
#include "kernels.cuh"
#include "tc.cuh"

#include <mutex>

namespace lora {
namespace {

#ifndef BT_BLOCKS_PER_SM
#define BT_BLOCKS_PER_SM 2
#endif
// Blocks per SM: each has its own producer warp, whose issue rate (about one
// shrink chunk or expand tile per 0.3-0.5 us) bounds its block; the rings shrink
// with the count so that the SM's bytes in flight stay about the same.
constexpr int BT_PER_SM = BT_BLOCKS_PER_SM;
static_assert(BT_PER_SM >= 1 && BT_PER_SM <= 2, "blocks per SM");
constexpr int BT_THREADS = 192;
constexpr uint32_t BT_RB = BT_PER_SM == 1 ? (128u << 10) : BT_PER_SM == 2 ? (64u << 10) : (32u << 10);   // operand ring
constexpr uint32_t BT_RY = BT_PER_SM == 1 ? (48u << 10) : (16u << 10);    // y ring
constexpr int BT_NV = BT_PER_SM == 1 ? 6 : BT_PER_SM == 2 ? 4 : 3;        // v pair slots (4 KB each: r_max <= 64)
constexpr uint32_t BT_VSLOT = 4096;
constexpr int BT_NSB = 64;               // operand allocations in flight at most
constexpr int BT_NYB = 64;               // y allocations in flight at most
constexpr int BT_NQ = 32;                // item records
constexpr uint32_t BT_TMEM_COLS = BT_PER_SM == 1 ? 256u : BT_PER_SM == 2 ? 256u : 128u;
constexpr int BT_NT = (int)BT_TMEM_COLS / 16;   // accumulators of 16 tensor-memory columns
constexpr int BT_ITEM_INTS = 32;
constexpr uint32_t BT_IDESC = idesc_bf16(128, 16);

// shared memory, from a 1 KB boundary
constexpr uint32_t OFF_RY = BT_RB;
constexpr uint32_t OFF_V = OFF_RY + BT_RY;               // v pair slots
constexpr uint32_t OFF_ZERO = OFF_V + BT_NV * BT_VSLOT;  // 2 KB of zeros (one 8-rank group of 128 rows)
constexpr uint32_t OFF_STG = OFF_ZERO + 2048;            // 4 KB: v pair being written out
constexpr uint32_t OFF_ITEM = OFF_STG + 4096;            // item records
constexpr uint32_t OFF_SADDR = OFF_ITEM + BT_NQ * BT_ITEM_INTS * 4;
constexpr uint32_t OFF_SEND = OFF_SADDR + BT_NSB * 4;
constexpr uint32_t OFF_YADDR = OFF_SEND + BT_NSB * 4;
constexpr uint32_t OFF_YEND = OFF_YADDR + BT_NYB * 4;
constexpr uint32_t OFF_BAR = OFF_YEND + BT_NYB * 4;
constexpr uint32_t BT_NBARS = 2 * BT_NSB + 2 * BT_NYB + 2 * BT_NQ + 2 * BT_NT + 2 * BT_NV;
constexpr uint32_t BT_SMEM = OFF_BAR + 8 * BT_NBARS + 1024;   // + room to align the base
static_assert(BT_PER_SM * (BT_SMEM + 1024) <= 228 * 1024, "shared memory");
// A shrink chunk's A rows are read as 128 rows (16 KB) from the chunk's start,
// which may reach up to 8 KB past its stage (r8 * 128 B per chunk, x after the
// last): the bytes past the operand ring that such a read may reach are the y ring's
static_assert(BT_RY >= 16384, "A over-read stays inside the allocation");
// the largest allocations (a 256-column shrink stage at r_max 64: 32 KB of A and
// 8 KB of x; 16 rows of y) fit their rings with room for the next
static_assert(BT_RB >= 40960 + 16384 && BT_RY >= 2 * 4096, "ring sizes");

// item record fields
enum { IT_KIND = 0, IT_U, IT_S, IT_ID, IT_CNT, IT_RN, IT_N, IT_CLO, IT_SCALE, IT_FAIL, IT_ROWS = 16 };
enum { KIND_SHRINK = 0, KIND_EXPAND = 1, KIND_END = 2 };

__device__ __forceinline__ void red_release_gpu(int *p, int v) {
    asm volatile("red.release.gpu.global.add.s32 [%0], %1;\n" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ int ld_acquire_gpu(const int *p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];\n" : "=r"(v) : "l"(p) : "memory");
    return v;
}
// 16 bytes global -> shared (L2 only), the first `bytes` of them read, the rest zero
__device__ __forceinline__ void cp16z(uint32_t dst, const void *src, int bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ uint32_t lds16(uint32_t a) {
    uint16_t r;
    asm volatile("ld.shared.u16 %0, [%1];\n" : "=h"(r) : "r"(a));
    return r;
}
__device__ __forceinline__ void sts16(uint32_t a, uint32_t v) {
    asm volatile("st.shared.u16 [%0], %1;\n" ::"r"(a), "h"((uint16_t)v) : "memory");
}
__device__ __forceinline__ uint32_t bf16_bits(float f) {
    const __nv_bfloat16 h = __float2bfloat16_rn(f);
    return *reinterpret_cast<const uint16_t *>(&h);
}
__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, 128;\n" ::: "memory"); }
// generic-proxy global writes (another block's v pair, seen through an acquire)
// before this thread's bulk copy reads them
__device__ __forceinline__ void proxy_fence_global() { asm volatile("fence.proxy.async.global;\n" ::: "memory"); }
// Four gathered rows of a 2-D tensor (box one row high) in one TMA copy, landing
// one after the other in shared memory
__device__ __forceinline__ void tma_gather4(uint32_t dst, const CUtensorMap *map, int x, int r0, int r1, int r2,
                                            int r3, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes [%0], [%1, "
        "{%2, %3, %4, %5, %6}], [%7];\n" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(r0), "r"(r1), "r"(r2), "r"(r3), "r"(bar)
        : "memory");
}
// K-major operand without swizzle: 8-row x 16-byte core matrices of 128
// contiguous bytes, the next 8 rows `sbo` bytes on, the next 8 K elements
// `lbo` bytes on (same field layout as desc_plain)
__device__ __forceinline__ uint64_t desc_kmaj(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}
// Bounded wait for a unit's done word (lane 0 polls; the warp agrees on the outcome)
__device__ __forceinline__ bool wait_done(const int *done, int need, unsigned limit, int32_t *status) {
    bool ready = true;
    if ((threadIdx.x & 31) == 0) {
        unsigned it = 0;
        while (ld_acquire_gpu(done) < need) {
            if (++it >= limit * 64u) {
                atomicOr(status, LORA_DEV_TIMEOUT);
                ready = false;
                break;
            }
            __nanosleep(64);
        }
    }
    return __shfl_sync(FULL, ready ? 1 : 0, 0) != 0;
}

__global__ void __launch_bounds__(BT_THREADS, BT_PER_SM) bgmv_tc_kernel(const __grid_constant__ BtArgs p) {
    const GbArgs &a = p.g;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    __shared__ uint32_t tmem_sm;
    __shared__ int exit_sm;
    __shared__ int epi_fail_sm;   // an epilogue warp's wait ran out
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char *sm = smem_raw + (base - raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t rb = base, ry = base + OFF_RY, zero = base + OFF_ZERO, stg = base + OFF_STG;
    int *items = reinterpret_cast<int *>(sm + OFF_ITEM);
    uint32_t *saddr = reinterpret_cast<uint32_t *>(sm + OFF_SADDR);
    uint32_t *send = reinterpret_cast<uint32_t *>(sm + OFF_SEND);
    uint32_t *yaddr = reinterpret_cast<uint32_t *>(sm + OFF_YADDR);
    uint32_t *yend = reinterpret_cast<uint32_t *>(sm + OFF_YEND);
    const uint32_t sfull = base + OFF_BAR, sempty = sfull + 8 * BT_NSB;
    const uint32_t yfull = sempty + 8 * BT_NSB, yempty = yfull + 8 * BT_NYB;
    const uint32_t qfull = yempty + 8 * BT_NYB, qempty = qfull + 8 * BT_NQ;
    const uint32_t afull = qempty + 8 * BT_NQ, aempty = afull + 8 * BT_NT;
    const uint32_t vfull = aempty + 8 * BT_NT, vempty = vfull + 8 * BT_NV;
    const uint32_t vbase = base + OFF_V;
    const int S = a.sl.n;
    const int live = n_live_units(a.tiles);
    // bytes of one (unit, slice) v pair in the workspace: hi and lo, rank groups of 8 x 16 rows x 16 B
    const int vstride = 2 * (((a.r_max + 15) >> 4) * 2) * 256;

    if (tid == 0) {
        for (int i = 0; i < BT_NSB; ++i) {
            mbar_init(sfull + 8 * i, 33);   // the producer's expect_tx + one cp.async arrival per lane
            mbar_init(sempty + 8 * i, 1);
        }
        for (int i = 0; i < BT_NYB; ++i) {
            mbar_init(yfull + 8 * i, 1);
            mbar_init(yempty + 8 * i, 4);   // one per epilogue warp
        }
        for (int i = 0; i < BT_NQ; ++i) {
            mbar_init(qfull + 8 * i, 1);
            mbar_init(qempty + 8 * i, 2);   // MMA warp and epilogue
        }
        for (int i = 0; i < BT_NT; ++i) {
            mbar_init(afull + 8 * i, 1);
            mbar_init(aempty + 8 * i, 4);   // one per epilogue warp
        }
        for (int i = 0; i < BT_NV; ++i) {
            mbar_init(vfull + 8 * i, 1);
            mbar_init(vempty + 8 * i, 1);
        }
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
        epi_fail_sm = 0;
    }
    for (int i = tid; i < 2048 / 16; i += BT_THREADS) sts128(zero + 16 * i, make_uint4(0u, 0u, 0u, 0u));
    fence_proxy_async();   // the zero buffer is read by the tensor cores
    if (warp == 0 && lane < S) {
        prefetch_tmap(&p.tmA[lane]);
        prefetch_tmap(&p.tmB[lane]);
        prefetch_tmap(&p.tmY[lane]);
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(
                         smem_u32(&tmem_sm)),
                     "r"(BT_TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_sm;

    if (warp == 0) {
        // ======================================================== producer
        uint32_t bhead = 0, btail = 0, yhead = 0, ytail = 0;
        int sbh = 0, sbt = 0, ybh = 0, ybt = 0, qc = 0, vc = 0;
        bool failed = false;
        // n bytes (a multiple of 1 KB) of the operand ring; its allocation index in *idx.
        // Allocations never wrap: one that would run past the end starts at the
        // beginning, the skipped tail counted with it; an empty ring restarts there.
        auto alloc_b = [&](uint32_t n, int *idx) -> uint32_t {
            for (;;) {
                const uint32_t off = bhead & (BT_RB - 1);
                const uint32_t pad = off + n > BT_RB ? BT_RB - off : 0u;
                if (pad && sbh == sbt) {   // nothing live: move to the beginning
                    bhead += pad;
                    btail = bhead;
                    continue;
                }
                if (bhead + pad + n - btail <= BT_RB && sbh - sbt < BT_NSB) {
                    bhead += pad;
                    const uint32_t addr = rb + (bhead & (BT_RB - 1));
                    bhead += n;
                    *idx = sbh % BT_NSB;
                    if (lane == 0) {
                        send[*idx] = bhead;
                        saddr[*idx] = addr;
                    }
                    ++sbh;
                    return addr;
                }
                const int i = sbt % BT_NSB;   // the oldest live allocation comes back
                if (!warp_wait(sempty + 8 * i, (unsigned)(sbt / BT_NSB) & 1u, a.status, failed)) return 0u;
                btail = send[i];
                ++sbt;
            }
        };
        // n bytes (a multiple of 256) of the y ring, the same way
        auto alloc_y = [&](uint32_t n, int *idx) -> uint32_t {
            for (;;) {
                const uint32_t off = yhead % BT_RY;
                const uint32_t pad = off + n > BT_RY ? BT_RY - off : 0u;
                if (pad && ybh == ybt) {
                    yhead += pad;
                    ytail = yhead;
                    continue;
                }
                if (yhead + pad + n - ytail <= BT_RY && ybh - ybt < BT_NYB) {
                    yhead += pad;
                    const uint32_t addr = ry + yhead % BT_RY;
                    yhead += n;
                    *idx = ybh % BT_NYB;
                    if (lane == 0) {
                        yend[*idx] = yhead;
                        yaddr[*idx] = addr;
                    }
                    ++ybh;
                    return addr;
                }
                const int i = ybt % BT_NYB;
                if (!warp_wait(yempty + 8 * i, (unsigned)(ybt / BT_NYB) & 1u, a.status, failed)) return 0u;
                ytail = yend[i];
                ++ybt;
            }
        };
        // the next item record (waits until both consumers are done with its slot)
        auto take_record = [&]() -> int * {
            const int q = qc % BT_NQ;
            if (!warp_wait(qempty + 8 * q, ((unsigned)(qc / BT_NQ) & 1u) ^ 1u, a.status, failed)) return nullptr;
            return items + q * BT_ITEM_INTS;
        };
        auto publish = [&]() {
            __syncwarp();
            if (lane == 0) mbar_arrive(qfull + 8 * (qc % BT_NQ));
            ++qc;
        };
        auto ticket = [&](int which) -> int {
            const int t = lane == 0 ? atomicAdd(a.ctl + which, 1) : 0;
            return __shfl_sync(FULL, t, 0);
        };

        // ------------------------------------------------ shrink items
        const int total1 = live * S;
        const int ks = p.ks;                       // 64-column chunks per stage
        const int nch = (a.d_in + 63) >> 6;
        const int nst = (nch + ks - 1) / ks;
        int cur = ticket(GB_T_SHRINK);
        while (cur < total1 && !failed) {
            const int nxt = ticket(GB_T_SHRINK);   // in flight during this item
            const int u = cur / S, s = cur - u * S;
            const Unit un = resolve_live_unit(a.tiles, u);
            const int r_n = un.cnt > 0 ? a.ranks[un.id] : 0;
            const bool ok = un.cnt > 0 && un.cnt <= 16 && r_n >= 1 && r_n <= a.r_max;
            if (!ok) {
                // nothing to compute: the unit's expand items skip it too, but may wait on it
                if (lane == 0) {
                    if (un.cnt > 0 && s == 0) atomicOr(a.status, un.cnt > 16 ? LORA_DEV_TILE_OVERFLOW : LORA_DEV_BAD_RANK);
                    red_release_gpu(a.done + u, 1);
                }
                cur = nxt;
                continue;
            }
            const int row_l = lane < un.cnt ? un.row(a.tiles, lane) : 0;
            // lane's x pieces: rows (lane >> 3) + 4m, 16-byte piece lane & 7 of each 64-column chunk
            const __nv_bfloat16 *xr[4];
            bool xv[4];
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int j = (lane >> 3) + 4 * m;
                const int row = __shfl_sync(FULL, row_l, j);
                xv[m] = j < un.cnt;
                xr[m] = a.x + (int64_t)row * a.ld_x;
            }
            const int g8 = (r_n + 7) >> 3;
            int *it = take_record();
            if (!it) break;
            if (lane == 0) {
                it[IT_KIND] = KIND_SHRINK;
                it[IT_U] = u;
                it[IT_S] = s;
                it[IT_ID] = un.id;
                it[IT_CNT] = un.cnt;
                it[IT_RN] = r_n;
                it[IT_N] = nst;
                it[IT_SCALE] = __float_as_int(a.alphas[un.id] / (float)r_n);
                it[IT_FAIL] = 0;
            }
            publish();
            const int arow = un.id * a.r_max;
            const uint32_t pc = (uint32_t)(lane & 7);
            for (int st = 0; st < nst; ++st) {
                const int c0 = st * ks, nsub = min(ks, nch - c0);
                int si = 0;
                // A: the item's r8 rank rows of ks chunks (one box), then x: ks chunks of 16 rows x 128 B
                const uint32_t sa = alloc_b((uint32_t)(g8 * ks) * 1024u + (uint32_t)ks * 2048u, &si);
                if (failed) break;
                const uint32_t xa = sa + (uint32_t)(g8 * ks) * 1024u;
                if (lane == 0) mbar_expect_tx(sfull + 8 * si, (uint32_t)(g8 * ks) * 1024u);
                __syncwarp();
                if (ks == 4) {
                    if (lane == 0) tma_3d(sa, &p.tmA4[g8 - 1][s], 0, arow, c0, sfull + 8 * si);
                } else if (lane < g8) {
                    tma_2d(sa + (uint32_t)lane * 1024u, &p.tmA[s], c0 * 64, arow + 8 * lane, sfull + 8 * si);
                }
                for (int c = 0; c < nsub; ++c) {
                    const int col = (c0 + c) * 64 + (int)pc * 8;
                    const int sz = min(max(2 * (a.d_in - col), 0), 16);
                    const uint32_t xc = xa + (uint32_t)c * 2048u;
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        const uint32_t j = (uint32_t)((lane >> 3) + 4 * m);
                        if (xv[m])
                            cp16z(xc + j * 128u + ((pc ^ (j & 7u)) << 4),
                                  sz ? (const void *)(xr[m] + col) : (const void *)xr[m], sz);
                    }
                }
                cp_async_arrive(sfull + 8 * si);   // once this lane's x pieces have landed
            }
            cur = nxt;
        }

        // ------------------------------------------------ expand items
        const int nb = a.blk_off[S];
        const int total2 = live * nb;
        const int need = S + (a.dbg_stall ? 1 : 0);   // the stall test hook waits for one more
        cur = failed ? total2 : ticket(GB_T_EXPAND);
        while (cur < total2 && !failed) {
            const int nxt = ticket(GB_T_EXPAND);
            const int u = cur / nb, b = cur - u * nb;
            int s = 0;
            while (s + 1 < S && a.blk_off[s + 1] <= b) ++s;
            const int c_lo = (b - a.blk_off[s]) * a.bc;
            const int c_hi = min(c_lo + a.bc, (int)a.sl.d_out[s]);
            const int nt = (c_hi - c_lo + 127) >> 7;
            const Unit un = resolve_live_unit(a.tiles, u);
            const int r_n = un.cnt > 0 ? a.ranks[un.id] : 0;
            if (!(un.cnt > 0 && un.cnt <= 16 && r_n >= 1 && r_n <= a.r_max)) {
                cur = nxt;
                continue;
            }
            const int row_l = lane < un.cnt ? un.row(a.tiles, lane) : 0;
            const int g8 = (r_n + 7) >> 3, g16 = ((r_n + 15) >> 4) * 2;
            const int brow = un.id * a.sl.d_out[s] + c_lo;
            // the item's v slot (its own ring: the B tiles go back one by one as their MMAs finish)
            const int vi = vc % BT_NV;
            if (!warp_wait(vempty + 8 * vi, ((unsigned)(vc / BT_NV) & 1u) ^ 1u, a.status, failed)) break;
            ++vc;
            // tile t's y rows and B boxes; the first tile flies while the unit's shrink may
            // still run, the others follow the v copy (the MMA warp starts on v, so the
            // item's tiles go back one by one and never need the ring all at once)
            // y rows in groups of four (one gather copy each; a group past the unit's last
            // row repeats that row, whose copy lands in bytes the epilogue does not read)
            const int nq = (un.cnt + 3) >> 2;
            int yr[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) yr[i] = __shfl_sync(FULL, row_l, min(4 * (lane & 3) + i, un.cnt - 1));
            auto issue_tile = [&](int t) {
                int yi = 0, bi = 0;
                const uint32_t ya = alloc_y((uint32_t)nq * 1024u, &yi);
                if (failed) return;
                if (lane == 0) mbar_expect_tx(yfull + 8 * yi, (uint32_t)nq * 1024u);
                __syncwarp();
                if (lane < nq)
                    tma_gather4(ya + (uint32_t)lane * 1024u, &p.tmY[s], c_lo + 128 * t, yr[0], yr[1], yr[2], yr[3],
                                yfull + 8 * yi);
                const uint32_t ba = alloc_b((uint32_t)g8 * 2048u, &bi);
                if (failed) return;
                if (lane == 0) mbar_expect_tx(sfull + 8 * bi, (uint32_t)g8 * 2048u);
                __syncwarp();
                if (lane < g8) tma_2d(ba + (uint32_t)lane * 2048u, &p.tmB[s], 8 * lane, brow + 128 * t, sfull + 8 * bi);
                cp_async_arrive(sfull + 8 * bi);   // no x here: the lanes' arrivals are immediate
            };
            issue_tile(0);
            if (failed) break;
            const uint32_t vbytes = (uint32_t)g16 * 512u;
            // the record goes out once the unit's v is known to be written (or its wait ran out)
            const bool ready = wait_done(a.done + u, need, a.wait_limit, a.status);
            int *it = take_record();
            if (!it) break;
            if (lane == 0) {
                it[IT_KIND] = KIND_EXPAND;
                it[IT_U] = u;
                it[IT_S] = s;
                it[IT_ID] = un.id;
                it[IT_CNT] = un.cnt;
                it[IT_RN] = r_n;
                it[IT_N] = nt;
                it[IT_CLO] = c_lo;
                it[IT_FAIL] = ready ? 0 : 1;
            }
            if (lane < 16) it[IT_ROWS + lane] = row_l;
            publish();
            if (lane == 0) {
                mbar_expect_tx(vfull + 8 * vi, vbytes);
                proxy_fence_global();   // v was written through the generic proxy by another block
                bulk_g2s(vbase + (uint32_t)vi * BT_VSLOT, p.vws + (size_t)(u * S + s) * (size_t)vstride, vbytes,
                         vfull + 8 * vi);
            }
            for (int t = 1; t < nt && !failed; ++t) issue_tile(t);
            if (failed) break;
            if (!ready) break;   // a unit that never finished: this block takes no more tickets
            cur = nxt;
        }
        int *it = take_record();
        if (it) {
            if (lane == 0) it[IT_KIND] = KIND_END;
            publish();
        }
    } else if (warp == 1) {
        // ======================================================== MMA issuer
        int qc = 0, sc = 0, ts = 0, vc = 0;
        bool failed = false;
        for (;;) {
            const int q = qc % BT_NQ;
            if (!warp_wait(qfull + 8 * q, (unsigned)(qc / BT_NQ) & 1u, a.status, failed)) break;
            const int *it = items + q * BT_ITEM_INTS;
            const int kind = it[IT_KIND];
            if (kind == KIND_END) break;
            const int r_n = it[IT_RN], n = it[IT_N];
            const int g8 = (r_n + 7) >> 3;
            if (kind == KIND_SHRINK) {
                const int slot = ts % BT_NT;
                if (!warp_wait(aempty + 8 * slot, ((unsigned)(ts / BT_NT) & 1u) ^ 1u, a.status, failed)) break;
                tc_fence_after();
                const uint32_t d = tmem + (uint32_t)slot * 16u;
                const int ks = p.ks, nch = (a.d_in + 63) >> 6;
                for (int st = 0; st < n; ++st) {
                    const int i = sc % BT_NSB;
                    if (!warp_wait(sfull + 8 * i, (unsigned)(sc / BT_NSB) & 1u, a.status, failed)) break;
                    tc_fence_after();
                    const int nsub = min(ks, nch - st * ks);
                    const uint32_t sa = saddr[i], xa = sa + (uint32_t)(g8 * ks) * 1024u;
                    if (lane == 0) {
                        fence_proxy_async();   // x arrived by cp.async (generic proxy); the MMA reads it as an operand
                        for (int c = 0; c < nsub; ++c) {
                            // chunk c: its r8 rank rows are contiguous (8-row atoms 1 KB apart)
                            const uint32_t ac = sa + (uint32_t)(c * g8) * 1024u, xc = xa + (uint32_t)c * 2048u;
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                tc_mma(d, desc_sw128(ac + 32u * kk), desc_sw128(xc + 32u * kk), BT_IDESC,
                                       (st | c | kk) ? 1u : 0u);
                        }
                        tc_commit(sempty + 8 * i);
                    }
                    __syncwarp();
                    ++sc;
                }
                if (failed) break;
                if (lane == 0) tc_commit(afull + 8 * slot);
                __syncwarp();
                ++ts;
            } else {
                const int g16 = ((r_n + 15) >> 4) * 2;
                const int vi = vc % BT_NV;
                if (!warp_wait(vfull + 8 * vi, (unsigned)(vc / BT_NV) & 1u, a.status, failed)) break;
                const uint32_t va = vbase + (uint32_t)vi * BT_VSLOT;
                for (int t = 0; t < n; ++t) {
                    const int slot = ts % BT_NT;
                    if (!warp_wait(aempty + 8 * slot, ((unsigned)(ts / BT_NT) & 1u) ^ 1u, a.status, failed)) break;
                    const int i = (sc + t) % BT_NSB;
                    if (!warp_wait(sfull + 8 * i, (unsigned)((sc + t) / BT_NSB) & 1u, a.status, failed)) break;
                    tc_fence_after();
                    const uint32_t ba = saddr[i];
                    if (r_n & 7) {
                        // ranks r_n .. 8*g8-1 of the last group are the slot's padding: zero them
                        const uint32_t g = ba + (uint32_t)(g8 - 1) * 2048u;
                        for (int c = lane; c < 128; c += 32)
                            for (int e = r_n & 7; e < 8; ++e) sts16(g + (uint32_t)c * 16u + 2u * e, 0u);
                        fence_proxy_async();
                        __syncwarp();
                    }
                    if (lane == 0) {
                        const uint32_t d = tmem + (uint32_t)slot * 16u;
                        for (int kk = 0; 2 * kk < g8; ++kk) {
                            const uint32_t a0 = ba + (uint32_t)kk * 4096u;
                            // an odd last group pairs with the zero buffer
                            const uint32_t lbo = 2 * kk + 1 < g8 ? 2048u : zero - a0;
                            const uint64_t ad = desc_kmaj(a0, lbo, 128u);
                            tc_mma(d, ad, desc_kmaj(va + (uint32_t)kk * 512u, 256u, 128u), BT_IDESC, kk ? 1u : 0u);
                            tc_mma(d, ad, desc_kmaj(va + (uint32_t)(g16 * 256 + kk * 512), 256u, 128u), BT_IDESC, 1u);
                        }
                        tc_commit(sempty + 8 * i);
                        tc_commit(afull + 8 * slot);
                    }
                    __syncwarp();
                    ++ts;
                }
                if (failed) break;
                if (lane == 0) tc_commit(vempty + 8 * vi);
                __syncwarp();
                sc += n;
                ++vc;
            }
            if (lane == 0) mbar_arrive(qempty + 8 * q);
            ++qc;
        }
    } else {
        // ======================================================== epilogue (warps 2-5)
        // The four warps meet at named barriers; a warp whose wait runs out still
        // reaches them, and all four leave together at the end of that item.
        const int et = tid - 64, q4 = warp & 3, L = 32 * q4 + lane;
        const uint32_t lane_base = tmem + ((uint32_t)(32 * q4) << 16);
        int qc = 0, ts = 0, yc = 0;
        bool failed = false;
        for (;;) {
            const int q = qc % BT_NQ;
            if (!warp_wait(qfull + 8 * q, (unsigned)(qc / BT_NQ) & 1u, a.status, failed)) break;
            const int *it = items + q * BT_ITEM_INTS;
            const int kind = it[IT_KIND];
            if (kind == KIND_END) break;
            const int u = it[IT_U], s = it[IT_S], cnt = it[IT_CNT], r_n = it[IT_RN], n = it[IT_N];
            if (kind == KIND_SHRINK) {
                const float scale = __int_as_float(it[IT_SCALE]);
                const int g16 = ((r_n + 15) >> 4) * 2;
                const int slot = ts % BT_NT;
                if (warp_wait(afull + 8 * slot, (unsigned)(ts / BT_NT) & 1u, a.status, failed)) {
                    tc_fence_after();
                    float f[16];
                    tc_ld16(lane_base + (uint32_t)slot * 16u, f);
                    tc_wait_ld();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(aempty + 8 * slot);
                    // s_n v as hi + lo bf16, [hi | lo][rank group][16 rows][8 ranks]; zero past r_n
                    if (L < 8 * g16) {
                        const bool live_rank = L < r_n;   // lanes past r_n hold padding or stale rows' sums
                        const uint32_t o = stg + (uint32_t)(L >> 3) * 256u + (uint32_t)(L & 7) * 2u;
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const float v = live_rank ? scale * f[j] : 0.f;
                            const uint32_t h = bf16_bits(v);
                            const uint32_t l = bf16_bits(v - __uint_as_float(h << 16));
                            sts16(o + (uint32_t)j * 16u, h);
                            sts16(o + (uint32_t)(g16 * 256 + j * 16), l);
                        }
                    }
                } else if (lane == 0) {
                    epi_fail_sm = 1;
                }
                ++ts;
                epi_sync();
                const bool go = *reinterpret_cast<volatile int *>(&epi_fail_sm) == 0;
                if (go) {
                    uint4 *dst = reinterpret_cast<uint4 *>(p.vws + (size_t)(u * S + s) * (size_t)vstride);
                    for (int o = et; o < g16 * 32; o += 128) dst[o] = lds128(stg + (uint32_t)o * 16u);
                    __threadfence();
                }
                epi_sync();
                if (go && et == 0) red_release_gpu(a.done + u, 1);
            } else {
                const bool fail = it[IT_FAIL] != 0;
                const int c_lo = it[IT_CLO];
                const int dout = a.sl.d_out[s];
                __nv_bfloat16 *ys = a.y + a.sl.col_off[s];
                for (int t = 0; t < n; ++t) {
                    const int slot = ts % BT_NT;
                    if (!warp_wait(afull + 8 * slot, (unsigned)(ts / BT_NT) & 1u, a.status, failed)) break;
                    tc_fence_after();
                    float f[16];
                    tc_ld16(lane_base + (uint32_t)slot * 16u, f);
                    tc_wait_ld();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(aempty + 8 * slot);
                    ++ts;
                    const int yi = yc % BT_NYB;
                    if (!warp_wait(yfull + 8 * yi, (unsigned)(yc / BT_NYB) & 1u, a.status, failed)) break;
                    const uint32_t ya = yaddr[yi];
                    // y + D2, one rounding, straight to the rows: thread L owns output
                    // column c_lo + 128t + L (a warp writes 64 contiguous bytes per row)
                    const int col = c_lo + 128 * t + L;
                    uint32_t out[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        out[j] = j < cnt ? bf16_bits(__uint_as_float(lds16(ya + (uint32_t)j * 256u + (uint32_t)L * 2u) << 16) + f[j])
                                         : 0u;
                    __syncwarp();
                    if (lane == 0) mbar_arrive(yempty + 8 * yi);   // the tile's y is read: its bytes go back
                    ++yc;
                    if (!fail && col < dout) {
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            if (j < cnt)
                                *reinterpret_cast<uint16_t *>(ys + (int64_t)it[IT_ROWS + j] * a.ld_y + col) =
                                    (uint16_t)out[j];
                    }
                }
                if (failed && lane == 0) epi_fail_sm = 1;
                epi_sync();   // every thread is done with the record's rows
            }
            if (et == 0) mbar_arrive(qempty + 8 * q);
            ++qc;
            if (*reinterpret_cast<volatile int *>(&epi_fail_sm)) break;   // all four warps leave together
        }
    }

    // ------------------------------------------------------------ leave
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(BT_TMEM_COLS)
                     : "memory");
    }
    if (tid == 0) {
        __threadfence();
        exit_sm = atomicAdd(a.ctl + GB_T_EXIT, 1) == (int)gridDim.x - 1;
        __threadfence();
    }
    __syncthreads();
    if (exit_sm) {   // every other block has left: the control words go back to zero
        for (int i = tid; i < live; i += BT_THREADS) a.done[i] = 0;
        if (tid == 0) {
            a.ctl[GB_T_SHRINK] = 0;
            a.ctl[GB_T_EXPAND] = 0;
            a.ctl[GB_T_EXIT] = 0;
        }
    }
}

}  // namespace

size_t bgmv_tc_smem_bytes() { return BT_SMEM; }

// Widest expand item (columns): four 128-column tiles behind one v pair.
int bgmv_tc_max_item_cols() { return 512; }

size_t bgmv_tc_v_bytes(int units, int n_slices, int r_max) {
    return (size_t)units * (size_t)n_slices * (size_t)(2 * (((r_max + 15) >> 4) * 2) * 256);
}

// Persistent launch: BT_PER_SM blocks per SM (or `blocks` when positive).
int launch_bgmv_tc(const BtArgs &args, int blocks, cudaStream_t st) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    {
        static std::mutex mu;
        static bool set[64] = {};
        std::lock_guard<std::mutex> lock(mu);
        const int d = dev & 63;
        if (!set[d]) {
            const cudaError_t e = cudaFuncSetAttribute(bgmv_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                       (int)BT_SMEM);
            if (e != cudaSuccess) return cuda_rc(e);
            set[d] = true;
        }
    }
    const int grid = blocks > 0 ? blocks : BT_PER_SM * sms;
    bgmv_tc_kernel<<<grid, BT_THREADS, BT_SMEM, st>>>(args);
    return cuda_rc(cudaGetLastError());
}

}  // namespace lora
