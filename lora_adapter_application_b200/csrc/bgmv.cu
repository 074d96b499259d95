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
// a step, so the sum over k is unchanged).  Each warp keeps a private ring of
// `stages` steps in flight (6 KB per step), so loads issue from all warps of
// the SM and no thread walks the work for the others; an 8-row x 64-byte load
// keeps whole 32-byte sectors, and a warp's stream runs along its rows for its
// whole column range.  Output columns of an expand step are permuted the same
// way (lane t's accumulators are columns 8t..8t+7 of its rows), so y moves in
// 16-byte pieces per lane, read and written once.
//
// In the fused mode v moves between the phases through a caller-provided
// workspace: an expand item of unit u starts once u's S * ceil(r_max / 32)
// shrink items have signalled (a per-unit counter, release / acquire at GPU
// scope).  Shrink items are taken by blocks and expand items by warps from
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
constexpr int BG_LD = 12;                        // 16-byte loads per lane per ring step
constexpr int BG_STEP = BG_LD * 32 * 16;         // bytes of one step of a warp's ring
constexpr int BG_MAX_STAGES = 4;
constexpr int BG_RG = 32;                        // ranks of one shrink item
constexpr int BG_RED_LD = BG_RG + 4;             // floats per row of the shrink reduction
constexpr int BG_RED_BYTES = BG_WARPS * BG_ROWS * BG_RED_LD * 4;
static_assert(BG_RED_BYTES <= 2 * BG_WARPS * BG_STEP, "the reduction fits the smallest ring");

// Workspace head of the fused mode (ints): tickets and exit counter, then one
// counter per unit.
constexpr int GB_CTL_INTS = 64;
enum { GB_T_SHRINK = 0, GB_T_EXPAND = 1, GB_T_EXIT = 2 };

constexpr unsigned FULL = 0xffffffffu;

// ------------------------------------------------------------------ PTX helpers
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// 16 (8) bytes global -> shared through L2; zero-filled (nothing read) when !valid
__device__ __forceinline__ void cp16(uint32_t dst, const void *src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src),
                 "r"(valid ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp8(uint32_t dst, const void *src, bool valid) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;\n" ::"r"(dst), "l"(src),
                 "r"(valid ? 8 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
// wait until at most n of this thread's copy groups are still in flight
__device__ __forceinline__ void cp_wait(int n) {
    switch (n) {
        case 0: asm volatile("cp.async.wait_group 0;\n" ::: "memory"); break;
        case 1: asm volatile("cp.async.wait_group 1;\n" ::: "memory"); break;
        case 2: asm volatile("cp.async.wait_group 2;\n" ::: "memory"); break;
        default: asm volatile("cp.async.wait_group 3;\n" ::: "memory"); break;
    }
}
__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 r;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "r"(a));
    return r;
}
__device__ __forceinline__ uint2 lds64(uint32_t a) {
    uint2 r;
    asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];\n" : "=r"(r.x), "=r"(r.y) : "r"(a));
    return r;
}
__device__ __forceinline__ void stg128(void *p, uint4 v) {
    asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};\n" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w)
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
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
// bf16 hi + lo split of two fp32 values (hi = round(v), lo = round(v - hi))
__device__ __forceinline__ void split2(float v0, float v1, uint32_t &hi, uint32_t &lo) {
    hi = pack_bf16x2(v0, v1);
    lo = pack_bf16x2(v0 - bf_lo(hi), v1 - bf_hi(hi));
}
// halves of a bf16 pair word that hold ranks k, k+1: all ones where the rank is below r_n
__device__ __forceinline__ uint32_t rank_mask(int k, int r_n) {
    return (k < r_n ? 0x0000ffffu : 0u) | (k + 1 < r_n ? 0xffff0000u : 0u);
}

// ------------------------------------------------------------------ shrink
// One warp's part of a shrink item: rank rows [0, rv) of the item's 32 (A_rows,
// lda bytes apart), the unit's rows (rows_s, -1 past the unit), k-steps
// [k_lo, k_hi) of 32 columns.  m = ranks (MG m16 tiles), n = rows (NTR n8
// tiles).  Ends with a block barrier and the warp's partial in red
// [warp][row][rank].
template <int MG, int NTR>
__device__ __forceinline__ void shrink_warp(const char *A_rows, int64_t lda, int rv, const char *x,
                                            int64_t ldx, const int *rows_s, int d_in, int k_lo,
                                            int k_hi, uint32_t ring, int NS, float *red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const char *pa[MG][2];
    bool va[MG][2];
#pragma unroll
    for (int mi = 0; mi < MG; ++mi)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int rr = 16 * mi + 8 * h + g;
            va[mi][h] = rr < rv;
            pa[mi][h] = A_rows + (va[mi][h] ? rr : 0) * lda + 16 * t;
        }
    const char *px[NTR];
    bool vx[NTR];
#pragma unroll
    for (int i = 0; i < NTR; ++i) {
        const int r = rows_s[8 * i + g];
        vx[i] = r >= 0;
        px[i] = x + (int64_t)(vx[i] ? r : 0) * ldx + 16 * t;
    }
    const uint32_t lbase = ring + (uint32_t)lane * 16u;
    auto issue = [&](int ks, int slot) {
        const uint32_t b = lbase + (uint32_t)slot * BG_STEP;
        const bool cv = 32 * ks + 8 * t < d_in;
#pragma unroll
        for (int mi = 0; mi < MG; ++mi)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const bool ok = va[mi][h] && cv;
                cp16(b + (2 * mi + h) * 512, ok ? pa[mi][h] + 64 * ks : A_rows, ok);
            }
#pragma unroll
        for (int i = 0; i < NTR; ++i) {
            const bool ok = vx[i] && cv;
            cp16(b + (2 * MG + i) * 512, ok ? px[i] + 64 * ks : x, ok);
        }
    };
    float acc[MG][NTR][4];
#pragma unroll
    for (int mi = 0; mi < MG; ++mi)
#pragma unroll
        for (int i = 0; i < NTR; ++i)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[mi][i][e] = 0.f;

    const int nst = k_hi - k_lo;
    for (int j = 0; j < NS - 1; ++j) {
        if (j < nst) issue(k_lo + j, j);
        cp_commit();
    }
    for (int j = 0; j < nst; ++j) {
        const int jn = j + NS - 1;
        if (jn < nst) issue(k_lo + jn, jn % NS);
        cp_commit();
        cp_wait(NS - 1);
        const uint32_t b = lbase + (uint32_t)(j % NS) * BG_STEP;
        uint4 qa[MG][2], qx[NTR];
#pragma unroll
        for (int mi = 0; mi < MG; ++mi) {
            qa[mi][0] = lds128(b + (2 * mi) * 512);
            qa[mi][1] = lds128(b + (2 * mi + 1) * 512);
        }
#pragma unroll
        for (int i = 0; i < NTR; ++i) qx[i] = lds128(b + (2 * MG + i) * 512);
#pragma unroll
        for (int mi = 0; mi < MG; ++mi) {
            const uint32_t a0[4] = {qa[mi][0].x, qa[mi][1].x, qa[mi][0].y, qa[mi][1].y};
            const uint32_t a1[4] = {qa[mi][0].z, qa[mi][1].z, qa[mi][0].w, qa[mi][1].w};
#pragma unroll
            for (int i = 0; i < NTR; ++i) {
                mma16816(acc[mi][i], a0, qx[i].x, qx[i].y);
                mma16816(acc[mi][i], a1, qx[i].z, qx[i].w);
            }
        }
    }
    cp_wait(0);
    __syncthreads();   // every warp is done with its ring: the reduction buffer overlays them
    float *rw = red + warp * BG_ROWS * BG_RED_LD;
#pragma unroll
    for (int mi = 0; mi < MG; ++mi)
#pragma unroll
        for (int i = 0; i < NTR; ++i) {
            const int r0 = 8 * i + 2 * t, k0 = 16 * mi + g;
            rw[r0 * BG_RED_LD + k0] = acc[mi][i][0];
            rw[(r0 + 1) * BG_RED_LD + k0] = acc[mi][i][1];
            rw[r0 * BG_RED_LD + k0 + 8] = acc[mi][i][2];
            rw[(r0 + 1) * BG_RED_LD + k0 + 8] = acc[mi][i][3];
        }
}

template <int MG>
__device__ __forceinline__ void shrink_dispatch(int ntr, const char *A_rows, int64_t lda, int rv,
                                                const char *x, int64_t ldx, const int *rows_s, int d_in,
                                                int k_lo, int k_hi, uint32_t ring, int NS, float *red) {
    if (ntr <= 1)
        shrink_warp<MG, 1>(A_rows, lda, rv, x, ldx, rows_s, d_in, k_lo, k_hi, ring, NS, red);
    else if (ntr <= 2)
        shrink_warp<MG, 2>(A_rows, lda, rv, x, ldx, rows_s, d_in, k_lo, k_hi, ring, NS, red);
    else if (ntr <= 4)
        shrink_warp<MG, 4>(A_rows, lda, rv, x, ldx, rows_s, d_in, k_lo, k_hi, ring, NS, red);
    else
        shrink_warp<MG, 8>(A_rows, lda, rv, x, ldx, rows_s, d_in, k_lo, k_hi, ring, NS, red);
}

// ------------------------------------------------------------------ expand
// One warp's expand pass over output columns [c_lo, c_hi) of one slice for up
// to 32 rows of a unit (row_l: this lane's row, -1 past the unit; rows 16*mi+g
// and 16*mi+g+8 of the pass are m16 tile mi).  RK: ranks loaded per row,
// 16 (8-byte loads of ranks 4t..4t+3), 32 or 64 (16-byte loads of ranks
// 32c+8t..32c+8t+7).  m = rows, n = output columns: n-tile j's column for
// n-index q is c0 + 8*(q>>1) + 2*j + (q&1), so lane t ends with columns
// c0+8t .. c0+8t+7.
template <int MR, int RK>
__device__ __forceinline__ void expand_warp(int row_l, const char *Bn, int r_max, int r_n,
                                            float scale, int c_lo, int c_hi,
                                            __nv_bfloat16 *ys, int64_t ld_y, const float *vs,
                                            uint32_t ring, int NS) {
    constexpr int CH = RK == 64 ? 2 : 1;            // rank chunks per step
    constexpr int NB = 4 * CH;                      // B loads per step
    constexpr int KB = RK == 16 ? 1 : 2;            // k16 products per chunk
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const int r8 = (r_n + 7) & ~7;
    // rows of this lane's y pieces and v fragments
    int yrow[MR][2];
#pragma unroll
    for (int mi = 0; mi < MR; ++mi)
#pragma unroll
        for (int h = 0; h < 2; ++h) yrow[mi][h] = __shfl_sync(FULL, row_l, 16 * mi + 8 * h + g);
    // B rank offset of chunk c for this lane, and the masks of ranks r_n..r8
    const int rk0 = RK == 16 ? 4 * t : 8 * t;
    uint32_t bm[CH][4];
#pragma unroll
    for (int c = 0; c < CH; ++c)
#pragma unroll
        for (int p = 0; p < 4; ++p) bm[c][p] = rank_mask(32 * c + rk0 + 2 * p, r_n);
    const int bcol = 8 * (g >> 1) + (g & 1);
    const uint32_t lbase = ring + (uint32_t)lane * 16u;
    auto issue = [&](int ks, int slot) {
        const uint32_t b = lbase + (uint32_t)slot * BG_STEP;
        const int c0 = c_lo + 32 * ks;
#pragma unroll
        for (int c = 0; c < CH; ++c)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int col = c0 + bcol + 2 * j;
                const bool ok = col < c_hi && 32 * c + rk0 < r8;
                const char *src = Bn + ((int64_t)col * r_max + 32 * c + rk0) * 2;
                if (RK == 16)
                    cp8(b + (4 * c + j) * 512, ok ? src : Bn, ok);
                else
                    cp16(b + (4 * c + j) * 512, ok ? src : Bn, ok);
            }
        const bool cv = c0 + 8 * t < c_hi;
#pragma unroll
        for (int mi = 0; mi < MR; ++mi)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const bool ok = cv && yrow[mi][h] >= 0;
                const char *src = reinterpret_cast<const char *>(ys + (int64_t)(ok ? yrow[mi][h] : 0) * ld_y +
                                                                 (ok ? c0 + 8 * t : 0));
                cp16(b + (NB + 2 * mi + h) * 512, src, ok);
            }
    };
    const int nst = (c_hi - c_lo + 31) >> 5;
    for (int j = 0; j < NS - 1; ++j) {   // the first steps fly while v is read
        if (j < nst) issue(j, j);
        cp_commit();
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
                    const float4 *p = reinterpret_cast<const float4 *>(vs + (int64_t)row * r_max + k);
                    const float4 lo4 = p[0];
                    f[0] = lo4.x; f[1] = lo4.y; f[2] = lo4.z; f[3] = lo4.w;
                    if (RK != 16) {
                        const float4 hi4 = p[1];
                        f[4] = hi4.x; f[5] = hi4.y; f[6] = hi4.z; f[7] = hi4.w;
                    } else {
                        f[4] = f[5] = f[6] = f[7] = 0.f;
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e) f[e] = 0.f;
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) f[e] = k + e < r_n ? scale * f[e] : 0.f;
#pragma unroll
                for (int p = 0; p < 4; ++p) split2(f[2 * p], f[2 * p + 1], vh[mi][c][h][p], vl[mi][c][h][p]);
            }

    for (int ks = 0; ks < nst; ++ks) {
        const int jn = ks + NS - 1;
        if (jn < nst) issue(jn, jn % NS);
        cp_commit();
        cp_wait(NS - 1);
        const uint32_t b = lbase + (uint32_t)(ks % NS) * BG_STEP;
        float acc[MR][4][4];
#pragma unroll
        for (int mi = 0; mi < MR; ++mi)
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[mi][j][e] = 0.f;
#pragma unroll
        for (int c = 0; c < CH; ++c)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint32_t q[4];
                if (RK == 16) {
                    const uint2 w = lds64(b + (4 * c + j) * 512);
                    q[0] = w.x & bm[c][0];
                    q[1] = w.y & bm[c][1];
                    q[2] = q[3] = 0u;
                } else {
                    const uint4 w = lds128(b + (4 * c + j) * 512);
                    q[0] = w.x & bm[c][0];
                    q[1] = w.y & bm[c][1];
                    q[2] = w.z & bm[c][2];
                    q[3] = w.w & bm[c][3];
                }
#pragma unroll
                for (int mi = 0; mi < MR; ++mi) {
#pragma unroll
                    for (int kb = 0; kb < KB; ++kb) {
                        const uint32_t ah[4] = {vh[mi][c][0][2 * kb], vh[mi][c][1][2 * kb],
                                                vh[mi][c][0][2 * kb + 1], vh[mi][c][1][2 * kb + 1]};
                        const uint32_t al[4] = {vl[mi][c][0][2 * kb], vl[mi][c][1][2 * kb],
                                                vl[mi][c][0][2 * kb + 1], vl[mi][c][1][2 * kb + 1]};
                        mma16816(acc[mi][j], ah, q[2 * kb], q[2 * kb + 1]);
                        mma16816(acc[mi][j], al, q[2 * kb], q[2 * kb + 1]);
                    }
                }
            }
        // y rows: lane t's 8 columns, word j = columns 8t+2j, 8t+2j+1 = accumulators (j, 2h), (j, 2h+1)
        const int c0 = c_lo + 32 * ks;
        const bool cv = c0 + 8 * t < c_hi;
#pragma unroll
        for (int mi = 0; mi < MR; ++mi)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint4 w = lds128(b + (NB + 2 * mi + h) * 512);
                const uint32_t win[4] = {w.x, w.y, w.z, w.w};
                uint32_t o[4];
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    o[j] = pack_bf16x2(bf_lo(win[j]) + acc[mi][j][2 * h],
                                       bf_hi(win[j]) + acc[mi][j][2 * h + 1]);
                if (cv && yrow[mi][h] >= 0)
                    stg128(ys + (int64_t)yrow[mi][h] * ld_y + c0 + 8 * t, make_uint4(o[0], o[1], o[2], o[3]));
            }
    }
    cp_wait(0);
}

template <int MR>
__device__ __forceinline__ void expand_dispatch(int r8, int row_l, const char *Bn, int r_max, int r_n,
                                                float scale, int c_lo, int c_hi, __nv_bfloat16 *ys,
                                                int64_t ld_y, const float *vs, uint32_t ring, int NS) {
    if (r8 <= 16)
        expand_warp<MR, 16>(row_l, Bn, r_max, r_n, scale, c_lo, c_hi, ys, ld_y, vs, ring, NS);
    else if (r8 <= 32)
        expand_warp<MR, 32>(row_l, Bn, r_max, r_n, scale, c_lo, c_hi, ys, ld_y, vs, ring, NS);
    else
        expand_warp<MR, 64>(row_l, Bn, r_max, r_n, scale, c_lo, c_hi, ys, ld_y, vs, ring, NS);
}

// ------------------------------------------------------------------ kernel
template <int MODE>
__global__ void __launch_bounds__(BG_THREADS, 1) bgmv_kernel(const GbArgs a) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ int rows_s[BG_ROWS];
    __shared__ int info_s[4];   // current shrink ticket, next ticket, "this block leaves last"
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int NS = a.stages;
    const uint32_t ring = smem_u32(smem) + (uint32_t)(warp * NS * BG_STEP);
    float *red = reinterpret_cast<float *>(smem);
    const int S = a.sl.n;
    const int live = n_live_units(a.tiles);
    const int GM = (a.r_max + BG_RG - 1) / BG_RG;   // shrink items per unit and slice

    // ------------------------------------------------------------ phase 1: shrink
    if (MODE != MODE_EXPAND) {
        const int total = live * S * GM;
        if (tid == 0) info_s[0] = MODE == MODE_FUSED ? atomicAdd(a.ctl + GB_T_SHRINK, 1) : (int)blockIdx.x;
        __syncthreads();
        const int nsteps = (a.d_in + 31) >> 5;
        const int k_lo = warp * nsteps / BG_WARPS, k_hi = (warp + 1) * nsteps / BG_WARPS;
        for (;;) {
            const int item = info_s[0];
            if (item >= total) break;
            if (tid == 0)   // the next ticket flies during this item
                info_s[1] = MODE == MODE_FUSED ? atomicAdd(a.ctl + GB_T_SHRINK, 1) : item + (int)gridDim.x;
            const int u = item / (S * GM), rem = item - u * S * GM;
            const int s = rem / GM, grp = rem - s * GM;
            const Unit un = resolve_live_unit(a.tiles, u);
            if (tid < BG_ROWS) rows_s[tid] = tid < un.cnt ? un.row(a.tiles, tid) : -1;
            const int r_n = un.cnt > 0 ? a.ranks[un.id] : 0;
            const bool ok = un.cnt > 0 && r_n >= 1 && r_n <= a.r_max;
            if (!ok && un.cnt > 0 && s == 0 && grp == 0 && tid == 0) atomicOr(a.status, LORA_DEV_BAD_RANK);
            const int rv = ok ? min(BG_RG, ((r_n + 7) & ~7) - BG_RG * grp) : 0;
            __syncthreads();
            if (rv > 0) {
                const char *A_rows = static_cast<const char *>(a.sl.A[s]) +
                                     ((int64_t)un.id * a.r_max + BG_RG * grp) * a.d_in * 2;
                const char *x = reinterpret_cast<const char *>(a.x);
                const int ntr = (un.cnt + 7) >> 3;
                if (rv > 16)
                    shrink_dispatch<2>(ntr, A_rows, (int64_t)a.d_in * 2, rv, x, a.ld_x * 2, rows_s, a.d_in,
                                       k_lo, k_hi, ring, NS, red);
                else
                    shrink_dispatch<1>(ntr, A_rows, (int64_t)a.d_in * 2, rv, x, a.ld_x * 2, rows_s, a.d_in,
                                       k_lo, k_hi, ring, NS, red);
                __syncthreads();
                // the 8 partials in warp order; v rows of the unit, ranks of the group below r_n
                float *vb = a.v + (int64_t)s * a.T * a.r_max;
                for (int p = tid; p < un.cnt * BG_RG; p += BG_THREADS) {
                    const int row = p / BG_RG, rl = p - row * BG_RG, k = BG_RG * grp + rl;
                    if (rl < rv && k < r_n) {
                        float sum = 0.f;
#pragma unroll
                        for (int w = 0; w < BG_WARPS; ++w) sum += red[(w * BG_ROWS + row) * BG_RED_LD + rl];
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
    if (MODE != MODE_SHRINK) {
        const int nb = a.blk_off[S];
        const int total = live * nb;
        const int need = S * GM + (a.dbg_stall ? 1 : 0);   // the stall test hook waits for one more
        int cur;
        if (MODE == MODE_FUSED) {
            cur = lane == 0 ? atomicAdd(a.ctl + GB_T_EXPAND, 1) : 0;
            cur = __shfl_sync(FULL, cur, 0);
        } else {
            cur = (int)blockIdx.x * BG_WARPS + warp;
        }
        while (cur < total) {
            int nxt;
            if (MODE == MODE_FUSED)
                nxt = lane == 0 ? atomicAdd(a.ctl + GB_T_EXPAND, 1) : 0;
            else
                nxt = cur + (int)gridDim.x * BG_WARPS;
            const int u = cur / nb, b = cur - u * nb;
            int s = 0;
            while (s + 1 < S && a.blk_off[s + 1] <= b) ++s;
            const int c_lo = (b - a.blk_off[s]) * a.bc;
            const int c_hi = min(c_lo + a.bc, (int)a.sl.d_out[s]);
            const Unit un = resolve_live_unit(a.tiles, u);
            const int r_n = un.cnt > 0 ? a.ranks[un.id] : 0;
            const bool ok = un.cnt > 0 && r_n >= 1 && r_n <= a.r_max;
            if (!ok && un.cnt > 0 && b == 0 && lane == 0 && MODE == MODE_EXPAND)
                atomicOr(a.status, LORA_DEV_BAD_RANK);
            if (ok) {
                if (MODE == MODE_FUSED) {   // v of unit u: all its shrink items have signalled
                    bool ready = true;
                    if (lane == 0) {
                        unsigned it = 0;
                        while (ld_acquire_gpu(a.done + u) < need) {
                            if (++it >= a.wait_limit * 64u) {
                                atomicOr(a.status, LORA_DEV_TIMEOUT);
                                ready = false;
                                break;
                            }
                            __nanosleep(128);
                        }
                    }
                    if (__shfl_sync(FULL, ready ? 1 : 0, 0) == 0) break;   // the warp takes no more work
                    (void)ld_acquire_gpu(a.done + u);   // every lane orders its v reads after the count
                }
                const float scale = a.alphas[un.id] / (float)r_n;
                const int r8 = (r_n + 7) & ~7;
                const char *Bn = static_cast<const char *>(a.sl.B[s]) +
                                 (int64_t)un.id * a.sl.d_out[s] * a.r_max * 2;
                __nv_bfloat16 *ys = a.y + a.sl.col_off[s];
                const float *vs = a.v + (int64_t)s * a.T * a.r_max;
                for (int rg = 0; rg * 32 < un.cnt; ++rg) {
                    const int q = 32 * rg + lane;
                    const int row_l = q < un.cnt ? un.row(a.tiles, q) : -1;
                    if (un.cnt - 32 * rg > 16)
                        expand_dispatch<2>(r8, row_l, Bn, a.r_max, r_n, scale, c_lo, c_hi, ys, a.ld_y, vs,
                                           ring, NS);
                    else
                        expand_dispatch<1>(r8, row_l, Bn, a.r_max, r_n, scale, c_lo, c_hi, ys, a.ld_y, vs,
                                           ring, NS);
                }
            }
            cur = MODE == MODE_FUSED ? __shfl_sync(FULL, nxt, 0) : nxt;
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

const void *bg_fn(int mode) {
    return mode == MODE_FUSED ? (const void *)bgmv_kernel<MODE_FUSED>
                              : (mode == MODE_SHRINK ? (const void *)bgmv_kernel<MODE_SHRINK>
                                                     : (const void *)bgmv_kernel<MODE_EXPAND>);
}

}  // namespace

size_t bgmv_smem_bytes(int mode, int stages) {
    (void)mode;
    return (size_t)stages * BG_WARPS * BG_STEP;
}

size_t bgmv_workspace_bytes(int units, int T, int n_slices, int r_max) {
    const size_t head = (size_t)GB_CTL_INTS * 4 + (((size_t)units * 4 + 255) & ~(size_t)255);
    return head + (size_t)n_slices * (size_t)T * (size_t)r_max * 4;
}

// Persistent launch: one block per SM (or `blocks` when positive).
int launch_bgmv(int mode, const GbArgs &args, int blocks, cudaStream_t st) {
    GbArgs a = args;
    if (a.stages < 2 || a.stages > BG_MAX_STAGES) a.stages = BG_MAX_STAGES;
    const size_t smem = bgmv_smem_bytes(mode, a.stages);
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    {
        // the limit is a per-device attribute of the kernel: set once, to the largest ring
        static std::mutex mu;
        static bool set[64][3] = {};
        std::lock_guard<std::mutex> lock(mu);
        const int d = dev & 63;
        if (!set[d][mode]) {
            const cudaError_t e = cudaFuncSetAttribute(bg_fn(mode), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                       (int)bgmv_smem_bytes(mode, BG_MAX_STAGES));
            if (e != cudaSuccess) return cuda_rc(e);
            set[d][mode] = true;
        }
    }
    const int grid = blocks > 0 ? blocks : sms;
    if (mode == MODE_FUSED)
        bgmv_kernel<MODE_FUSED><<<grid, BG_THREADS, smem, st>>>(a);
    else if (mode == MODE_SHRINK)
        bgmv_kernel<MODE_SHRINK><<<grid, BG_THREADS, smem, st>>>(a);
    else
        bgmv_kernel<MODE_EXPAND><<<grid, BG_THREADS, smem, st>>>(a);
    return cuda_rc(cudaGetLastError());
}

}  // namespace lora
