// Fused multi-LoRA BGMV over gathered rows, bf16, ranks up to 64 (page
// "Multi-LoRA Serving", section 3.2: rows grouped per adapter, BGMV-style
// grouped products; section 3.4: add_shrink then add_expand in one call).
//
// Unit of work = up to 64 rows that share an adapter (a gathered tile, or a
// piece of a contiguous tile).  One persistent launch runs two phases:
//
//   shrink   block item = (unit, slice s, group of 32 ranks): the block's 8
//            warps split the input columns, each computes
//            v^T[ranks][rows] over its columns with mma m16n8k16 (bf16 in, fp32
//            accumulate; ranks on the m side, so a unit of 1-8 rows costs one
//            n8 tile), and the 8 partials meet in shared memory, added in warp
//            order (run-to-run identical).  v = A x (fp32) is written for k < r_n.
//   expand   warp item = (unit, slice s, block of output columns): the warp
//            holds (alpha_n / r_n) v of up to 32 rows as a bf16 hi + lo pair
//            (about 16 mantissa bits) and streams B_s[n][cols][0:r8] and the y
//            rows through the tensor pipe, 32 columns per step:
//            y[rows][cols] += scale * v . B^T, fp32 accumulation, y rounded once.
//
// Every operand is streamed by the warp that uses it: each lane moves 16 bytes
// per operand row per step with cp.async, straight into the order the mma
// fragments want (lane (g, t) of an 8-row operand reads columns 8t..8t+7 of row
// g; both operands of a product use the same permutation of the 32 columns of
// a step, so the sum over k is unchanged).  Each warp keeps a private 24 KB
// ring of steps in flight (2 to 16 of them, by step size), so loads issue from
// all warps of the SM and no thread walks the work for the others; an 8-row x 64-byte load
// keeps whole 32-byte sectors, and a warp's stream runs along its rows for its
// whole column range.  Output columns of an expand step are permuted the same
// way (lane t's accumulators are columns 8t..8t+7 of its rows), so y moves in
// 16-byte pieces per lane, read and written once.
//
// In the fused mode v moves between the phases through a caller-provided
// workspace: an expand item of unit u starts once all of u's shrink items have
// signalled (S slices x rank groups x pieces; a per-unit counter, release /
// acquire at GPU scope).  A small batch runs a second instantiation whose
// shrink items are two pieces along d_in, each writing its own partial v, which
// the expand adds in piece order.  Shrink items are taken by blocks and expand items by warps from
// atomic tickets, and a block turns to expand items only once every shrink
// item has been taken, so a warp only ever waits for units that a running
// block holds: the launch makes progress whatever number of its blocks is
// resident (and beside other kernels).  The tickets, the per-unit counters and
// an exit counter live at the head of the workspace; the last block to leave
// puts them back to zero.  The shrink-only and expand-only modes (v from / to
// the caller) assign work statically and need no workspace.
//
// Ranks r_n..r8 (r8 = r_n rounded up to 8) of A and B are loaded and masked
// out of every product; ranks r8..r_max are never loaded.  The one wait (an
// expand item for its unit) is bounded: when it runs out, LORA_DEV_TIMEOUT is
// set in the status word and the warp stops taking work.
#include "kernels.cuh"
#include "ptx.cuh"

#include <mutex>

namespace lora {
namespace {

constexpr int BG_WARPS = 8;
constexpr int BG_THREADS = BG_WARPS * 32;
constexpr int BG_ROWS = LORA_MAX_TILE_ROWS;      // rows of one unit
constexpr int BG_RING = 24576;                   // bytes of one warp's ring of steps
// Ranks of one shrink item: 32 (units of up to 64 rows), or all of the slot's 64 when
// units have at most 16 rows (the accumulators of 4 x 2 tiles fit a warp)
constexpr int BG_RG = 32;
constexpr int BG_RG_SMALL = 64;
constexpr int BG_SMALL_ROWS = 16;
// floats per row of the shrink reduction: the item's ranks + 4 (bank spread)
__host__ __device__ constexpr int red_ld(int rg) { return rg + 4; }
constexpr int BG_RED_BYTES = BG_WARPS * BG_ROWS * (BG_RG + 4) * 4;
static_assert(BG_WARPS * BG_SMALL_ROWS * (BG_RG_SMALL + 4) * 4 <= BG_RED_BYTES, "small-unit reduction");
static_assert(BG_RED_BYTES <= BG_WARPS * BG_RING, "the reduction overlays the rings");

// Steps of nld 16-byte loads per lane (nld * 512 bytes per warp) that a ring holds.
__host__ __device__ constexpr int ring_depth(int nld) {
    return BG_RING / (nld * 512) > 16 ? 16 : BG_RING / (nld * 512);
}

// Workspace head of the fused mode (ints): tickets and exit counter, then one
// counter per unit.

constexpr unsigned FULL = 0xffffffffu;

// ------------------------------------------------------------------ PTX helpers
// (not volatile: the compiler may interleave independent products)
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// 16 bytes global -> shared through L2, of which the first `bytes` are read and the
// rest zero-filled (0: nothing read)
__device__ __forceinline__ void cp16(uint32_t dst, const void *src, int bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(bytes)
                 : "memory");
}
// The same for B rows: their ranks past r8 are padding, so L2 fetches 64 bytes for
// them instead of its default line (a rank-8..32 adapter in a 64-rank slot then moves
// 64 bytes per output column through HBM, not 128)
__device__ __forceinline__ void cp16_64(uint32_t dst, const void *src, int bytes) {
    asm volatile("cp.async.cg.shared.global.L2::64B [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
// wait until at most N of this thread's copy groups are still in flight
template <int N>
__device__ __forceinline__ void cp_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}
__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 r;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "r"(a));
    return r;
}
__device__ __forceinline__ void red_release_gpu(int *p, int v) {
    asm volatile("red.release.gpu.global.add.s32 [%0], %1;\n" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ int ld_acquire_gpu(const int *p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];\n" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
// bf16 hi + lo split of two fp32 values (hi = round(v), lo = round(v - hi))
__device__ __forceinline__ void split2(float v0, float v1, uint32_t &hi, uint32_t &lo) {
    hi = pack_bf16x2(v0, v1);
    lo = pack_bf16x2(v0 - bf_lo(hi), v1 - bf_hi(hi));
}
__device__ __forceinline__ int clampi(int v, int lo, int hi) { return v < lo ? lo : (v > hi ? hi : v); }

// ------------------------------------------------------------------ shrink
// One warp's part of a shrink item: rank rows [0, rv) of the item's 32 (A_rows,
// lda bytes apart), the unit's rows (rows_s, -1 past the unit), k-steps
// [k_lo, k_hi) of 32 columns.  m = ranks (MG m16 tiles), n = rows (NTR n8
// tiles).  Ends with a block barrier and the warp's partial in red
// [warp][row][rank] (8*NTR rows of ld floats per warp).
template <int MG, int NTR>
__device__ __forceinline__ void shrink_warp(const char *A_rows, int64_t lda, int rv, const char *x,
                                            int64_t ldx, const int *rows_s, int d_in, int k_lo,
                                            int k_hi, uint32_t ring, float *red, int ld) {
    constexpr int NLD = 2 * MG + NTR;
    constexpr int NSL = ring_depth(NLD);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    // row starts (a row past the item reads nothing: its start stands in)
    const char *p[NLD];
    int sz[NLD];
#pragma unroll
    for (int mi = 0; mi < MG; ++mi)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int rr = 16 * mi + 8 * h + g;
            const bool ok = rr < rv;
            p[2 * mi + h] = A_rows + (ok ? rr : 0) * lda;
            sz[2 * mi + h] = ok ? 16 : 0;
        }
#pragma unroll
    for (int i = 0; i < NTR; ++i) {
        const int r = rows_s[8 * i + g];
        const bool ok = r >= 0;
        p[2 * MG + i] = x + (int64_t)(ok ? r : 0) * ldx;
        sz[2 * MG + i] = ok ? 16 : 0;
    }
    const int nst = k_hi - k_lo;
    const int nfull = clampi((d_in >> 5) - k_lo, 0, nst);   // steps inside d_in for every lane
    const int jv = max(0, (d_in - 8 * t - 32 * k_lo + 31) >> 5);   // steps inside d_in for this lane
    const uint32_t lbase = ring + (uint32_t)lane * 16u;
    auto issue = [&](int j, int slot) {
        const uint32_t b = lbase + (uint32_t)(slot * NLD * 512);
        if (j < nfull) {
            const int off = 64 * (k_lo + j) + 16 * t;
#pragma unroll
            for (int l = 0; l < NLD; ++l) cp16(b + l * 512, p[l] + off, sz[l]);
        } else {
            const bool cv = j < jv;
            const int off = cv ? 64 * (k_lo + j) + 16 * t : 0;
#pragma unroll
            for (int l = 0; l < NLD; ++l) cp16(b + l * 512, p[l] + off, cv ? sz[l] : 0);
        }
    };
    float acc[MG][NTR][4];
#pragma unroll
    for (int mi = 0; mi < MG; ++mi)
#pragma unroll
        for (int i = 0; i < NTR; ++i)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[mi][i][e] = 0.f;

#pragma unroll 1   // one copy of the issue code (the instruction cache is a first-order cost)
    for (int j = 0; j < NSL - 1; ++j) {
        if (j < nst) issue(j, j);
        cp_commit();
    }
    int si = NSL - 1, sc = 0;   // slots of the next issue and of the next step consumed
    for (int j = 0; j < nst; ++j) {
        if (j + NSL - 1 < nst) issue(j + NSL - 1, si);
        si = si + 1 == NSL ? 0 : si + 1;
        cp_commit();
        cp_wait<NSL - 1>();
        const uint32_t b = lbase + (uint32_t)(sc * NLD * 512);
        sc = sc + 1 == NSL ? 0 : sc + 1;
        uint4 q[NLD];
#pragma unroll
        for (int l = 0; l < NLD; ++l) q[l] = lds128(b + l * 512);
#pragma unroll
        for (int kb = 0; kb < 2; ++kb)
#pragma unroll
            for (int mi = 0; mi < MG; ++mi) {
                const uint32_t a[4] = {kb ? q[2 * mi].z : q[2 * mi].x, kb ? q[2 * mi + 1].z : q[2 * mi + 1].x,
                                       kb ? q[2 * mi].w : q[2 * mi].y, kb ? q[2 * mi + 1].w : q[2 * mi + 1].y};
#pragma unroll
                for (int i = 0; i < NTR; ++i)
                    mma16816(acc[mi][i], a, kb ? q[2 * MG + i].z : q[2 * MG + i].x,
                             kb ? q[2 * MG + i].w : q[2 * MG + i].y);
            }
    }
    cp_wait<0>();
    __syncthreads();   // every warp is done with its ring: the reduction buffer overlays them
    float *rw = red + warp * 8 * NTR * ld;
#pragma unroll
    for (int mi = 0; mi < MG; ++mi)
#pragma unroll
        for (int i = 0; i < NTR; ++i) {
            const int r0 = 8 * i + 2 * t, k0 = 16 * mi + g;
            rw[r0 * ld + k0] = acc[mi][i][0];
            rw[(r0 + 1) * ld + k0] = acc[mi][i][1];
            rw[r0 * ld + k0 + 8] = acc[mi][i][2];
            rw[(r0 + 1) * ld + k0 + 8] = acc[mi][i][3];
        }
}

// n8 row tiles of the item: 2, 4 or 8 (the loaded rows past the unit are zero-filled; a
// unit of up to 8 rows takes the 2-tile form, one variant fewer in the instruction cache);
// returns the tile count used (the reduction buffer's rows per warp / 8)
template <int MG>
__device__ __forceinline__ int shrink_dispatch(int ntr, const char *A_rows, int64_t lda, int rv,
                                               const char *x, int64_t ldx, const int *rows_s, int d_in,
                                               int k_lo, int k_hi, uint32_t ring, float *red, int ld) {
    if (ntr <= 2) {
        shrink_warp<MG, 2>(A_rows, lda, rv, x, ldx, rows_s, d_in, k_lo, k_hi, ring, red, ld);
        return 2;
    }
    if (MG <= 2 && ntr <= 4) {
        shrink_warp<MG, 4>(A_rows, lda, rv, x, ldx, rows_s, d_in, k_lo, k_hi, ring, red, ld);
        return 4;
    }
    shrink_warp<(MG <= 2 ? MG : 2), 8>(A_rows, lda, rv, x, ldx, rows_s, d_in, k_lo, k_hi, ring, red, ld);
    return 8;
}

// ------------------------------------------------------------------ expand
// L2 policy for the y rows: read once and written once, they go first, so the
// repeats of A, B and x stay longer.
__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;\n" : "=l"(p));
    return p;
}
__device__ __forceinline__ void cp16_hint(uint32_t dst, const void *src, int bytes, uint64_t pol) {
    asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2, %3;\n" ::"r"(dst), "l"(src),
                 "r"(bytes), "l"(pol)
                 : "memory");
}
__device__ __forceinline__ void stg128_hint(void *p, uint4 v, uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.v4.u32 [%0], {%1,%2,%3,%4}, %5;\n" ::"l"(p), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w), "l"(pol)
                 : "memory");
}

// The fused mode's wait of an expand item for its unit's v: until *done reaches
// need (bounded; nullptr = nothing to wait for).  Every lane then acquires the
// count itself, ordering its v reads after the shrink's writes.
struct EWait {
    const int *done;
    int need;
    unsigned limit;
    int32_t *status;
};
__device__ __forceinline__ bool e_wait(const EWait &w) {
    if (!w.done) return true;
    bool ready = true;
    if ((threadIdx.x & 31) == 0) {
        unsigned it = 0;
        while (ld_acquire_gpu(w.done) < w.need) {
            if (++it >= w.limit * 64u) {
                atomicOr(w.status, LORA_DEV_TIMEOUT);
                ready = false;
                break;
            }
            __nanosleep(128);
        }
    }
    if (__shfl_sync(FULL, ready ? 1 : 0, 0) == 0) return false;
    (void)ld_acquire_gpu(w.done);
    return true;
}

// One warp's expand pass over output columns [c_lo, c_hi) of one slice for up
// to 32 rows of a unit (row_l: this lane's row, -1 past the unit; rows 16*mi+g
// and 16*mi+g+8 of the pass are m16 tile mi).  RK: ranks loaded per row, 32 or
// 64 (16-byte loads of ranks 32c+8t..32c+8t+7; a rank-8 or rank-16 adapter takes
// the 32-rank form with its upper lanes reading nothing: one variant fewer keeps
// the hot code inside the instruction cache, which measured faster); bytes past
// rank r_n are zero-filled, not read.  m = rows, n = output columns: n-tile j's column for n-index q is
// c0 + 8*(q>>1) + 2*j + (q&1), so lane t ends with columns c0+8t .. c0+8t+7.
// The accumulators start from the y values, so y + scale * v . B^T is rounded
// to bf16 once.
template <int MR, int RK>
__device__ __forceinline__ bool expand_warp(int row_l, const char *Bn, int r_max, int r_n,
                                            float scale, int c_lo, int c_hi,
                                            __nv_bfloat16 *ys, int64_t ld_y, const float *vs, int64_t vpiece,
                                            uint32_t ring, const EWait &wt) {
    constexpr int H = 2;                            // row halves (g, g+8) of an m16 tile
    constexpr int CH = RK == 64 ? 2 : 1;            // rank chunks per step
    constexpr int NB = 4 * CH;                      // B loads per step
    constexpr int NLD = NB + MR * H;
    constexpr int NSL = ring_depth(NLD);
    constexpr int KB = 2;                           // k16 products per chunk
    constexpr int LB = 16;                          // bytes of one B load
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const int r8 = (r_n + 7) & ~7;
    const uint64_t pol = policy_evict_first();
    // rows of this lane's y pieces and v fragments
    int yrow[MR][2];
#pragma unroll
    for (int mi = 0; mi < MR; ++mi)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int r = __shfl_sync(FULL, row_l, 16 * mi + 8 * h + g);
            yrow[mi][h] = h < H ? r : -1;
        }
    const int rk0 = 8 * t;
    int szb[CH];   // bytes of chunk c below rank r_n
#pragma unroll
    for (int c = 0; c < CH; ++c) szb[c] = clampi(2 * (r_n - 32 * c - rk0), 0, LB);
    // B column of n-tile j at step ks: cb + 2j + 32ks (B rows are r_max ranks long); a
    // chunk that this lane reads nothing of points at Bn and does not move
    const int cb = c_lo + 8 * (g >> 1) + (g & 1);
    const char *pbc[CH];
    int bs[CH], bj[CH];
#pragma unroll
    for (int c = 0; c < CH; ++c) {
        const bool any = szb[c] > 0 && cb < c_hi;
        pbc[c] = any ? Bn + ((int64_t)cb * r_max + rk0 + 32 * c) * 2 : Bn;
        bs[c] = any ? 64 * r_max : 0;
        bj[c] = any ? 4 * r_max : 0;
    }
    // y piece of row (mi, h) at step ks: columns c_lo + 32ks + 8t .. +7 (the row's
    // first column of the item stands in for a piece that is not read)
    const char *py[MR][H];
    int sy[MR][H];
#pragma unroll
    for (int mi = 0; mi < MR; ++mi)
#pragma unroll
        for (int h = 0; h < H; ++h) {
            const bool ok = yrow[mi][h] >= 0;
            py[mi][h] = reinterpret_cast<const char *>(ys + (int64_t)(ok ? yrow[mi][h] : 0) * ld_y + c_lo);
            sy[mi][h] = ok ? 16 : 0;
        }
    const int nst = (c_hi - c_lo + 31) >> 5;
    const int nfull = (c_hi - c_lo) >> 5;   // steps whose 32 columns are all inside
    const uint32_t lbase = ring + (uint32_t)lane * 16u;
    auto issue = [&](int ks, int slot) {
        const uint32_t b = lbase + (uint32_t)(slot * NLD * 512);
        if (ks < nfull) {
#pragma unroll
            for (int c = 0; c < CH; ++c)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const char *src = pbc[c] + (ks * bs[c] + j * bj[c]);
                    cp16_64(b + (4 * c + j) * 512, src, szb[c]);
                }
#pragma unroll
            for (int mi = 0; mi < MR; ++mi)
#pragma unroll
                for (int h = 0; h < H; ++h)
                    cp16_hint(b + (NB + H * mi + h) * 512, py[mi][h] + (sy[mi][h] ? 64 * ks + 16 * t : 0),
                              sy[mi][h], pol);
        } else {
#pragma unroll
            for (int c = 0; c < CH; ++c)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const bool ok = cb + 2 * j + 32 * ks < c_hi;
                    const char *src = ok ? pbc[c] + (ks * bs[c] + j * bj[c]) : Bn;
                    cp16_64(b + (4 * c + j) * 512, src, ok ? szb[c] : 0);
                }
            const bool cv = c_lo + 8 * t + 32 * ks < c_hi;
#pragma unroll
            for (int mi = 0; mi < MR; ++mi)
#pragma unroll
                for (int h = 0; h < H; ++h) {
                    const bool ok = cv && sy[mi][h];
                    cp16_hint(b + (NB + H * mi + h) * 512, py[mi][h] + (ok ? 64 * ks + 16 * t : 0), ok ? 16 : 0,
                              pol);
                }
        }
    };
    // the first steps fly while the unit's shrink finishes and v is read
    constexpr int PRO = NSL - 1;
#pragma unroll 1   // one copy of the issue code (the instruction cache is a first-order cost)
    for (int j = 0; j < PRO; ++j) {
        if (j < nst) issue(j, j);
        cp_commit();
    }
    // B and y do not depend on v: the first steps fly while the unit's shrink finishes
    if (!e_wait(wt)) {
        cp_wait<0>();
        return false;
    }
    // scale * v as bf16 hi / lo pairs: vh[mi][c][h][p] = ranks 32c + rk0 + 2p, +1 of row (mi, h)
    uint32_t vh[MR][CH][2][4], vl[MR][CH][2][4];
#pragma unroll
    for (int mi = 0; mi < MR; ++mi)
#pragma unroll
        for (int c = 0; c < CH; ++c)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int row = yrow[mi][h];
                const int k = 32 * c + rk0;
                float f[8];
                if (row >= 0 && k < r8) {
                    const float4 *pv = reinterpret_cast<const float4 *>(vs + (int64_t)row * r_max + k);
                    float4 lo4 = pv[0], hi4 = pv[1];
                    if (vpiece) {   // a split shrink: the second piece's partial, added in piece order
                        const float4 *pw = pv + vpiece / 4;
                        const float4 lo2 = pw[0], hi2 = pw[1];
                        lo4 = make_float4(lo4.x + lo2.x, lo4.y + lo2.y, lo4.z + lo2.z, lo4.w + lo2.w);
                        hi4 = make_float4(hi4.x + hi2.x, hi4.y + hi2.y, hi4.z + hi2.z, hi4.w + hi2.w);
                    }
                    f[0] = lo4.x; f[1] = lo4.y; f[2] = lo4.z; f[3] = lo4.w;
                    f[4] = hi4.x; f[5] = hi4.y; f[6] = hi4.z; f[7] = hi4.w;
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e) f[e] = 0.f;
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) f[e] = k + e < r_n ? scale * f[e] : 0.f;
#pragma unroll
                for (int p = 0; p < 4; ++p) split2(f[2 * p], f[2 * p + 1], vh[mi][c][h][p], vl[mi][c][h][p]);
            }

    // one step from ring slot b: accumulators from the y pieces, products, y rounded and stored
    auto step = [&](uint32_t b, int ks) {
        float acc[MR][4][4];
#pragma unroll
        for (int mi = 0; mi < MR; ++mi)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                if (h < H) {
                    const uint4 w = lds128(b + (NB + H * mi + h) * 512);
                    const uint32_t win[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        acc[mi][j][2 * h] = bf_lo(win[j]);
                        acc[mi][j][2 * h + 1] = bf_hi(win[j]);
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[mi][j][2 * h] = acc[mi][j][2 * h + 1] = 0.f;
                }
            }
#pragma unroll
        for (int c = 0; c < CH; ++c)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint4 w = lds128(b + (4 * c + j) * 512);
                const uint32_t q[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int kb = 0; kb < KB; ++kb)
#pragma unroll
                    for (int hl = 0; hl < 2; ++hl)
#pragma unroll
                        for (int mi = 0; mi < MR; ++mi) {
                            const uint32_t(&vv)[2][4] = hl ? vl[mi][c] : vh[mi][c];
                            const uint32_t av[4] = {vv[0][2 * kb], vv[1][2 * kb], vv[0][2 * kb + 1],
                                                    vv[1][2 * kb + 1]};
                            mma16816(acc[mi][j], av, q[2 * kb], q[2 * kb + 1]);
                        }
            }
        const int c0 = c_lo + 32 * ks;
        const bool cv = c0 + 8 * t < c_hi;
#pragma unroll
        for (int mi = 0; mi < MR; ++mi)
#pragma unroll
            for (int h = 0; h < H; ++h)
                if (cv && yrow[mi][h] >= 0)
                    stg128_hint(ys + (int64_t)yrow[mi][h] * ld_y + c0 + 8 * t,
                                make_uint4(pack_bf16x2(acc[mi][0][2 * h], acc[mi][0][2 * h + 1]),
                                           pack_bf16x2(acc[mi][1][2 * h], acc[mi][1][2 * h + 1]),
                                           pack_bf16x2(acc[mi][2][2 * h], acc[mi][2][2 * h + 1]),
                                           pack_bf16x2(acc[mi][3][2 * h], acc[mi][3][2 * h + 1])),
                                pol);
    };

    int si = PRO, sc = 0;
    for (int ks = 0; ks < nst; ++ks) {
        if (ks + NSL - 1 < nst) issue(ks + NSL - 1, si);
        si = si + 1 == NSL ? 0 : si + 1;
        cp_commit();
        cp_wait<NSL - 1>();
        const uint32_t b = lbase + (uint32_t)(sc * NLD * 512);
        sc = sc + 1 == NSL ? 0 : sc + 1;
        step(b, ks);
    }
    cp_wait<0>();
    return true;
}

template <int MR>
__device__ __forceinline__ bool expand_dispatch(int r8, int row_l, const char *Bn, int r_max, int r_n,
                                                float scale, int c_lo, int c_hi, __nv_bfloat16 *ys,
                                                int64_t ld_y, const float *vs, int64_t vpiece, uint32_t ring,
                                                const EWait &wt) {
    if (r8 <= 32)
        return expand_warp<MR, 32>(row_l, Bn, r_max, r_n, scale, c_lo, c_hi, ys, ld_y, vs, vpiece, ring, wt);
    return expand_warp<MR, 64>(row_l, Bn, r_max, r_n, scale, c_lo, c_hi, ys, ld_y, vs, vpiece, ring, wt);
}

// What an expand warp needs of one item before it starts: unit, rank, this
// lane's row among the first 32 (loaded one item ahead).
struct ERec {
    Unit un;
    int r_n;
    int row_l;
};
__device__ __forceinline__ ERec erec_load(const GbArgs &a, int e, int total, int nb) {
    ERec r{};
    r.un = Unit{0, 0, 0, true};
    r.r_n = 0;
    r.row_l = -1;
    if (e < total) {
        r.un = resolve_live_unit(a.tiles, e / nb);
        if (r.un.cnt > 0) r.r_n = a.ranks[r.un.id];
        const int lane = threadIdx.x & 31;
        r.row_l = lane < r.un.cnt ? r.un.row(a.tiles, lane) : -1;
    }
    return r;
}

// ------------------------------------------------------------------ kernel
// SPLIT (fused mode): every shrink item is two pieces along d_in, each writing
// its own partial v; the expand adds them.  A separate instantiation, so that the
// unsplit kernel's hot code is unchanged.
template <int MODE, bool SPLIT = false>
__global__ void __launch_bounds__(BG_THREADS, 1) bgmv_kernel(const GbArgs a) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ int rows_s[BG_ROWS];
    __shared__ int info_s[4];   // current shrink ticket, next ticket, "this block leaves last"
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t ring = smem_u32(smem) + (uint32_t)(warp * BG_RING);
    float *red = reinterpret_cast<float *>(smem);
    const int S = a.sl.n;
    const int live = n_live_units(a.tiles);
    // shrink items per unit and slice: one for units of up to 16 rows, else one per 32 ranks
    const bool small = a.tiles.rows_per_unit <= BG_SMALL_ROWS;
    const int RGW = small ? BG_RG_SMALL : BG_RG;
    const int GM = (a.r_max + RGW - 1) / RGW;
    const int rld = red_ld(RGW);

    // ------------------------------------------------------------ phase 1: shrink
    if (MODE != MODE_EXPAND) {
        constexpr int KS = MODE == MODE_FUSED && SPLIT ? 2 : 1;   // pieces of an item along d_in
        const int total = live * S * GM * KS;
        if (tid == 0) info_s[0] = MODE == MODE_FUSED ? atomicAdd(a.ctl + GB_T_SHRINK, 1) : (int)blockIdx.x;
        __syncthreads();
        const int nsteps = (a.d_in + 31) >> 5;
        for (;;) {
            const int item = info_s[0];
            if (item >= total) break;
            if (tid == 0)   // the next ticket flies during this item
                info_s[1] = MODE == MODE_FUSED ? atomicAdd(a.ctl + GB_T_SHRINK, 1) : item + (int)gridDim.x;
            const int piece = item % KS, ig = item / KS;
            const int u = ig / (S * GM), rem = ig - u * S * GM;
            const int s = rem / GM, grp = rem - s * GM;
            // the piece's 32-column steps, split over the block's warps
            const int p_lo = piece * nsteps / KS, p_n = (piece + 1) * nsteps / KS - p_lo;
            const int k_lo = p_lo + warp * p_n / BG_WARPS, k_hi = p_lo + (warp + 1) * p_n / BG_WARPS;
            const Unit un = resolve_live_unit(a.tiles, u);
            if (tid < BG_ROWS) rows_s[tid] = tid < un.cnt ? un.row(a.tiles, tid) : -1;
            const int r_n = un.cnt > 0 ? a.ranks[un.id] : 0;
            const bool ok = un.cnt > 0 && r_n >= 1 && r_n <= a.r_max;
            if (!ok && un.cnt > 0 && s == 0 && grp == 0 && tid == 0) atomicOr(a.status, LORA_DEV_BAD_RANK);
            const int rv = ok ? min(RGW, ((r_n + 7) & ~7) - RGW * grp) : 0;
            __syncthreads();
            if (rv > 0) {
                const char *A_rows = static_cast<const char *>(a.sl.A[s]) +
                                     ((int64_t)un.id * a.r_max + RGW * grp) * a.d_in * 2;
                const char *x = reinterpret_cast<const char *>(a.x);
                const int64_t lda = (int64_t)a.d_in * 2;
                float *vb = a.v + piece * a.vpiece + (int64_t)s * a.T * a.r_max;
                const int ntr = (un.cnt + 7) >> 3;
                int nt;
                if (rv > 32)
                    nt = shrink_dispatch<4>(ntr, A_rows, lda, rv, x, a.ld_x * 2, rows_s, a.d_in, k_lo, k_hi, ring,
                                            red, rld);
                else if (rv > 16)
                    nt = shrink_dispatch<2>(ntr, A_rows, lda, rv, x, a.ld_x * 2, rows_s, a.d_in, k_lo, k_hi, ring,
                                            red, rld);
                else
                    nt = shrink_dispatch<1>(ntr, A_rows, lda, rv, x, a.ld_x * 2, rows_s, a.d_in, k_lo, k_hi, ring,
                                            red, rld);
                __syncthreads();
                // the 8 partials in warp order; v rows of the unit, ranks of the group below r_n
                const int wst = 8 * nt * rld;   // floats of one warp's partial
                for (int p = tid; p < un.cnt * RGW; p += BG_THREADS) {
                    const int row = p / RGW, rl = p - row * RGW, k = RGW * grp + rl;
                    if (rl < rv && k < r_n) {
                        float sum = 0.f;
#pragma unroll
                        for (int w = 0; w < BG_WARPS; ++w) sum += red[w * wst + row * rld + rl];
                        vb[(int64_t)rows_s[row] * a.r_max + k] = sum;
                    }
                }
                if (MODE == MODE_FUSED) __threadfence();
            }
            __syncthreads();
            if (tid == 0) {
                if (MODE == MODE_FUSED) red_release_gpu(a.done + u, 1);   // this item's v rows are written
                info_s[0] = info_s[1];
            }
            __syncthreads();
        }
    }

    // ------------------------------------------------------------ phase 2: expand
    // Items are drawn two ahead and their records one ahead: while item i runs,
    // the ticket of item i+2 and the unit, rank, alpha and first rows of item i+1
    // are on their way.
    if (MODE != MODE_SHRINK) {
        const int nb = a.blk_off[S];
        const int total = live * nb;
        const int need = S * GM * (MODE == MODE_FUSED && SPLIT ? 2 : 1) + (a.dbg_stall ? 1 : 0);   // the stall test hook waits for one more
        auto claim = [&](int prev) -> int {
            if (MODE == MODE_FUSED) {
                const int v = lane == 0 ? atomicAdd(a.ctl + GB_T_EXPAND, 1) : 0;
                return __shfl_sync(FULL, v, 0);
            }
            return prev + (int)gridDim.x * BG_WARPS;
        };
        int cur = claim((int)blockIdx.x * BG_WARPS + warp - (int)gridDim.x * BG_WARPS);
        ERec rc = erec_load(a, cur, total, nb);
        int nxt = claim(cur);
        while (cur < total) {
            const ERec rn = erec_load(a, nxt, total, nb);
            const int nxt2 = nxt < total ? claim(nxt) : nxt;
            const int u = cur / nb, b = cur - u * nb;
            int s = 0;
            while (s + 1 < S && a.blk_off[s + 1] <= b) ++s;
            const int c_lo = (b - a.blk_off[s]) * a.bc;
            const int c_hi = min(c_lo + a.bc, (int)a.sl.d_out[s]);
            const Unit &un = rc.un;
            const int r_n = rc.r_n;
            const bool ok = un.cnt > 0 && r_n >= 1 && r_n <= a.r_max;
            if (!ok && un.cnt > 0 && b == 0 && lane == 0 && MODE == MODE_EXPAND)
                atomicOr(a.status, LORA_DEV_BAD_RANK);
            if (ok) {
                const float scale = a.alphas[un.id] / (float)r_n;
                const int r8 = (r_n + 7) & ~7;
                const char *Bn = static_cast<const char *>(a.sl.B[s]) +
                                 (int64_t)un.id * a.sl.d_out[s] * a.r_max * 2;
                __nv_bfloat16 *ys = a.y + a.sl.col_off[s];
                const float *vs = a.v + (int64_t)s * a.T * a.r_max;
                // the first pass waits (fused mode) for unit u's shrink items, after issuing
                // its first steps
                EWait wt{MODE == MODE_FUSED ? a.done + u : nullptr, need, a.wait_limit, a.status};
                bool ok_pass = true;
                for (int rg = 0; rg * 32 < un.cnt && ok_pass; ++rg) {
                    const int q = 32 * rg + lane;
                    const int row_l = rg == 0 ? rc.row_l : (q < un.cnt ? un.row(a.tiles, q) : -1);
                    const int rows = un.cnt - 32 * rg;
                    if (rows > 16)
                        ok_pass = expand_dispatch<2>(r8, row_l, Bn, a.r_max, r_n, scale, c_lo, c_hi, ys, a.ld_y,
                                                        vs, MODE == MODE_FUSED && SPLIT ? a.vpiece : 0, ring, wt);
                    else
                        ok_pass = expand_dispatch<1>(r8, row_l, Bn, a.r_max, r_n, scale, c_lo, c_hi, ys, a.ld_y,
                                                        vs, MODE == MODE_FUSED && SPLIT ? a.vpiece : 0, ring, wt);
                    wt.done = nullptr;
                }
                if (!ok_pass) break;   // the wait ran out: the warp takes no more work
            }
            cur = nxt;
            nxt = nxt2;
            rc = rn;
        }
    }

    // ------------------------------------------------------------ leave
    if (MODE == MODE_FUSED) {
        __syncthreads();
        if (tid == 0) {
            __threadfence();
            info_s[2] = atomicAdd(a.ctl + GB_T_EXIT, 1) == (int)gridDim.x - 1;
            __threadfence();
        }
        __syncthreads();
        if (info_s[2]) {   // every other block has left: the control words go back to zero
            for (int i = tid; i < live; i += BG_THREADS) a.done[i] = 0;
            if (tid == 0) {
                a.ctl[GB_T_SHRINK] = 0;
                a.ctl[GB_T_EXPAND] = 0;
                a.ctl[GB_T_EXIT] = 0;
            }
        }
    }
}

const void *bg_fn(int mode, bool split) {
    return mode == MODE_FUSED ? (split ? (const void *)bgmv_kernel<MODE_FUSED, true>
                                       : (const void *)bgmv_kernel<MODE_FUSED>)
                              : (mode == MODE_SHRINK ? (const void *)bgmv_kernel<MODE_SHRINK>
                                                     : (const void *)bgmv_kernel<MODE_EXPAND>);
}

}  // namespace

size_t bgmv_smem_bytes(int mode) {
    (void)mode;
    return (size_t)BG_WARPS * BG_RING;
}

size_t bgmv_workspace_head(int units) {
    return (size_t)GB_CTL_INTS * 4 + (((size_t)units * 4 + 255) & ~(size_t)255);
}

size_t bgmv_workspace_bytes(int units, int T, int n_slices, int r_max) {
    const size_t v32 = (size_t)BG_KSPLIT_MAX * n_slices * (size_t)T * (size_t)r_max * 4;   // this kernel's fp32 v
    const size_t vtc = bgmv_tc_v_bytes(units, n_slices, r_max);            // the tensor-core kernel's v pairs
    return bgmv_workspace_head(units) + (v32 > vtc ? v32 : vtc);
}

// Persistent launch: one block per SM (or `blocks` when positive).
int launch_bgmv(int mode, const GbArgs &args, int blocks, cudaStream_t st) {
    const GbArgs &a = args;
    const size_t smem = bgmv_smem_bytes(mode);
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    {
        // the limit is a per-device attribute of the kernel: set once, to the largest ring
        static std::mutex mu;
        static bool set[64][4] = {};
        const bool split = mode == MODE_FUSED && a.ks == 2;
        const int slot = split ? 3 : mode;
        std::lock_guard<std::mutex> lock(mu);
        const int d = dev & 63;
        if (!set[d][slot]) {
            const cudaError_t e =
                cudaFuncSetAttribute(bg_fn(mode, split), cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return cuda_rc(e);
            set[d][slot] = true;
        }
    }
    const int grid = blocks > 0 ? blocks : sms;
    if (mode == MODE_FUSED) {
        if (a.ks == 2)
            bgmv_kernel<MODE_FUSED, true><<<grid, BG_THREADS, smem, st>>>(a);
        else
            bgmv_kernel<MODE_FUSED><<<grid, BG_THREADS, smem, st>>>(a);
    } else if (mode == MODE_SHRINK)
        bgmv_kernel<MODE_SHRINK><<<grid, BG_THREADS, smem, st>>>(a);
    else
        bgmv_kernel<MODE_EXPAND><<<grid, BG_THREADS, smem, st>>>(a);
    return cuda_rc(cudaGetLastError());
}

}  // namespace lora
