// Tensor-core SGMV for contiguous tiles (prompt runs), bf16: page "Multi-LoRA
// Serving", section 3.2 (SGMV: rows that share an adapter form a segment and
// the per-segment products are dense) and section 3.4 (add_shrink, then
// add_expand, in one batched call).
//
// A contiguous tile is up to 128 consecutive rows with one adapter n, so both
// products are dense contractions with M = 128 rows:
//   shrink  D1[128][S*r_max] = X[128][d_in] . [A_0[n]; ...; A_{S-1}[n]]^T   (K = d_in)
//   expand  D2[128][128]     = (s_n v)[128][r_max] . B_s[n][cols]^T          (K = r_max)
// Both run on the 5th-generation tensor cores (tcgen05.mma kind::f16: bf16
// operands in shared memory, fp32 accumulators in tensor memory); every
// operand tile reaches shared memory through a TMA tensor copy.
//
// A cluster of C thread blocks takes a tile.  Block c reduces 1/C of the input
// columns and owns 1/C of the 128-column output chunks.  Every block sends its
// partial D1 to every block of the cluster through distributed shared memory;
// each block adds the C partials in rank order (run-to-run identical), keeps
// ranks k < r_n, scales by s_n = alpha_n/r_n and splits s_n v into a bf16 hi + lo
// pair (about 16 mantissa bits; one bf16 copy is not enough when the delta is
// large and cancels against y).  Clusters are persistent: cluster k takes
// tiles k, k + #clusters, ...; the TMA producer runs ahead across tiles, so
// HBM keeps streaming while a cluster exchanges its partials.
//
// Warp roles (352 threads, one block per SM):
//   warp 0     TMA producer: x and A boxes (shrink), y and B boxes (expand)
//              into a ring of `stages` slots; a full/empty mbarrier pair per
//              slot.  x and y move in boxes of lbr rows issued row group by row
//              group (both 64-column halves of a row group back to back), one
//              box per lane; a partial tile loads only the row groups it has.
//   warp 1     tensor-memory allocator and MMA issuer (one thread issues; when
//              r_n is not a multiple of 16 the warp first zeroes B's padded
//              ranks in the slot, so padding never reaches the sum)
//   warps 2-9  epilogue: D1 -> exchange -> s v in shared memory; D2 + y -> y
//              (fp32 add, rounded once to bf16) in place in the slot, or with
//              16-byte stores straight to the tile's rows for a partial tile
//              (a tensor store would write the neighbours' rows)
//   warp 10    store warp: TMA tensor stores of finished y boxes; it frees a
//              slot once its stores have read it.  (A store waits in the TMA
//              queue behind the loads issued before it, about 2 us under load;
//              on its own warp that wait no longer holds up the epilogue.)
//
// Tensor memory, 512 columns: D2 double buffer at columns 0 and 128, D1 at 256.
//
// Every wait is bounded: a wait that runs out sets LORA_DEV_TIMEOUT in the
// status word; the block then drains its copies and MMAs in flight and leaves.
#include "kernels.cuh"
#include "ptx.cuh"
#include "tc.cuh"

#include <cstdlib>
#include <mutex>

namespace lora {

constexpr int TC_THREADS = 352;
constexpr int TC_M = 128;                 // rows per tile = MMA M
constexpr uint32_t TC_XY = 32768;         // x or y part of a slot: two 64-column x 128-row boxes
constexpr uint32_t TC_BOX = 16384;        // one 64-column x 128-row bf16 box
constexpr uint32_t TC_D1_COL = 256;       // tensor-memory column of D1
constexpr uint32_t TC_TMEM_COLS = 512;
constexpr int TC_MAX_STAGES = 6;

// Shared memory (from a 1 KB boundary):
//   ring  stages x [x or y boxes: 32 KB | A or B boxes: SR*256 B]
//   V     SR*512 B   s v as bf16: [slice][hi, lo][rank / 8][128 rows][8]
//   XCH   2*C*SR*512 B partials (C > 1, shrink modes), one buffer per tile parity:
//         [parity][source block][SR/4][128 rows][4] fp32
//   mbarriers
// At least 120 KB, so that one block holds an SM: a block takes all 512
// tensor-memory columns, and two blocks of different clusters waiting for
// each other's columns could otherwise stall both clusters.
size_t sgmv_tc_smem_bytes(int mode, int stages, int SR, int C) {
    const size_t b = 1024 + (size_t)stages * (TC_XY + (size_t)SR * 256) + (size_t)SR * 512 +
                     ((mode != MODE_EXPAND && C > 1) ? (size_t)2 * C * SR * 512 : 0) + 512;
    return b < (size_t)120 * 1024 ? (size_t)120 * 1024 : b;
}

template <int MODE>
__global__ void __launch_bounds__(TC_THREADS, 1) sgmv_tc_kernel(const __grid_constant__ TcArgs a) {
    extern __shared__ __align__(1024) unsigned char tc_sm[];
    __shared__ uint32_t tmem_sm;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int S = a.sl.n, R = a.r_max, SR = S * R, C = a.C, STG = a.stages;
    const uint32_t crank = cluster_rank();
    const int cl = blockIdx.x / C, ncl = gridDim.x / C;
    const bool xchg = MODE != MODE_EXPAND && C > 1;
    // No tile for this cluster (a batch without prompt runs): leave before
    // touching tensor memory or the cluster barrier; the same for every block
    // of the cluster.
    const int n_tiles = min(a.counts[2], a.max_contig);
    if (cl >= n_tiles) return;

    const uint32_t ring = (smem_u32(tc_sm) + 1023u) & ~1023u;
    const uint32_t slot_bytes = TC_XY + (uint32_t)SR * 256u;
    const uint32_t vbuf = ring + (uint32_t)STG * slot_bytes;
    const uint32_t xch = vbuf + (uint32_t)SR * 512u;
    const uint32_t xch_bytes = (uint32_t)(C * SR) * 512u;   // one exchange buffer
    const uint32_t bars = xch + (xchg ? 2u * xch_bytes : 0u);
    // per slot: full, empty, and "the epilogue has written the slot's y"
    const uint32_t b_full = bars, b_empty = bars + 8u * STG, b_ystage = bars + 16u * STG;
    const uint32_t b_d1full = bars + 24u * STG, b_d1free = b_d1full + 8, b_vfull = b_d1full + 16;
    const uint32_t b_d2full = b_d1full + 24, b_d2empty = b_d1full + 40;   // [2] each
    const uint32_t b_xfull = b_d1full + 56, b_mma = b_d1full + 72;   // b_xfull[2]

    if (tid == 0) {
        for (int st = 0; st < STG; ++st) {
            mbar_init(b_full + 8 * st, 1);
            mbar_init(b_empty + 8 * st, 1);
            mbar_init(b_ystage + 8 * st, 8);
        }
        mbar_init(b_d1full, 1);
        mbar_init(b_d1free, 8);
        mbar_init(b_vfull, 8);
        mbar_init(b_d2full, 1);
        mbar_init(b_d2full + 8, 1);
        mbar_init(b_d2empty, 8);
        mbar_init(b_d2empty + 8, 8);
        mbar_init(b_xfull, 1);       // per phase: this block's expect_tx, then the partials' bytes
        mbar_init(b_xfull + 8, 1);
        mbar_init(b_mma, 1);
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    if (warp == 0) {   // descriptors of every map this block will copy with
        if (lane < S) {
            if (MODE != MODE_EXPAND) prefetch_tmap(&a.tmA[lane]);
            if (MODE != MODE_SHRINK) {
                prefetch_tmap(&a.tmB[lane]);
                prefetch_tmap(&a.tmY[lane]);
                prefetch_tmap(&a.tmYs[lane]);
            }
        }
        if (lane == 0 && MODE != MODE_EXPAND) prefetch_tmap(&a.tmX);
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(
                         smem_u32(&tmem_sm)),
                     "r"(TC_TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
    }
    tc_fence_before();
    cluster_sync_all();   // barriers initialised in every block of the cluster
    tc_fence_after();
    const uint32_t tmem = tmem_sm;

    // ------------------------------------------------------------ geometry
    const int nk = (a.d_in + 127) >> 7;   // 128-column chunks of the input
    const int k_lo = MODE == MODE_EXPAND ? 0 : (int)(((int64_t)crank * nk) / C);
    const int k_hi = MODE == MODE_EXPAND ? 0 : (int)(((int64_t)(crank + 1) * nk) / C);
    int NE = 0;
    for (int s = 0; s < S; ++s) NE += (a.sl.d_out[s] + 127) >> 7;
    const int e_lo = MODE == MODE_SHRINK ? 0 : (int)(((int64_t)crank * NE) / C);
    const int e_hi = MODE == MODE_SHRINK ? 0 : (int)(((int64_t)(crank + 1) * NE) / C);
    int es0 = 0, ec0 = 0;   // slice and first slice-local column of chunk e_lo
    {
        int e = e_lo;
        while (es0 < S - 1 && e >= ((a.sl.d_out[es0] + 127) >> 7)) {
            e -= (a.sl.d_out[es0] + 127) >> 7;
            ++es0;
        }
        ec0 = e * 128;
    }
    bool failed = false;

    if (warp == 0) {
        // ============================================================ producer
        uint32_t fills = 0;
        int st = 0;
        uint32_t ph = 0;
        for (int t = cl; t < n_tiles && !failed; t += ncl) {
            const int4 tile = a.contig[t];
            const int id = tile.x, row0 = tile.y;
            const int r_n = a.ranks[id];
            if (r_n < 1 || r_n > R) {
                if (crank == 0 && lane == 0) atomicOr(a.status, LORA_DEV_BAD_RANK);
                continue;
            }
            const int lbr = a.lbr, nrg = (tile.z + lbr - 1) / lbr;   // load boxes down the tile
            const uint32_t lbox = (uint32_t)lbr * 128u;                  // bytes of one load box
            for (int kc = k_lo; kc < k_hi; ++kc) {
                if (!warp_wait(b_empty + 8 * st, ph ^ 1u, a.status, failed)) break;
                const uint32_t slot = ring + (uint32_t)st * slot_bytes, full = b_full + 8 * st;
                const int k0 = kc * 128, nb = min(2, (a.d_in - k0 + 63) >> 6);
                if (lane == 0)
                    mbar_expect_tx(full, (uint32_t)(nb * nrg) * lbox + (uint32_t)(nb * SR) * 128u);
                __syncwarp();
                for (int i = lane; i < nrg * nb; i += 32) {   // x: row group major
                    const int rg = i / nb, b = i - rg * nb;
                    tma_2d(slot + b * TC_BOX + rg * lbox, &a.tmX, k0 + 64 * b, row0 + lbr * rg, full);
                }
                for (int i = lane; i < nb * S; i += 32) {     // A of every slice
                    const int b = i / S, s = i - b * S;
                    tma_2d(slot + TC_XY + (uint32_t)((b * S + s) * R) * 128u, &a.tmA[s], k0 + 64 * b,
                           id * R, full);
                }
                __syncwarp();
                ++fills;
                if (++st == STG) {
                    st = 0;
                    ph ^= 1u;
                }
            }
            if (failed) break;
            int s = es0, c0 = ec0;
            for (int e = e_lo; e < e_hi; ++e) {
                if (!warp_wait(b_empty + 8 * st, ph ^ 1u, a.status, failed)) break;
                const int d_out = a.sl.d_out[s];
                const uint32_t slot = ring + (uint32_t)st * slot_bytes, full = b_full + 8 * st;
                const int ny = d_out - c0 > 64 ? 2 : 1;
                if (lane == 0)
                    mbar_expect_tx(full, (uint32_t)(ny * nrg) * lbox + (uint32_t)(R >> 3) * 2048u);
                __syncwarp();
                for (int i = lane; i < nrg * ny; i += 32) {   // y: row group major
                    const int rg = i / ny, h = i - rg * ny;
                    tma_2d(slot + h * TC_BOX + rg * lbox, &a.tmY[s], c0 + 64 * h, row0 + lbr * rg, full);
                }
                for (int g = lane; g < (R >> 3); g += 32)    // B: 8 ranks x 128 output columns
                    tma_2d(slot + TC_XY + g * 2048u, &a.tmB[s], 8 * g, id * d_out + c0, full);
                __syncwarp();
                ++fills;
                if (++st == STG) {
                    st = 0;
                    ph ^= 1u;
                }
                c0 += 128;
                if (c0 >= d_out) {
                    ++s;
                    c0 = 0;
                }
            }
        }
        // drain: the copies of the last fill of every slot have landed
        bool f2 = false;
        for (int i = 0; i < STG; ++i) {
            if ((uint32_t)i >= fills) break;
            const uint32_t f = (uint32_t)i + (uint32_t)STG * ((fills - 1u - (uint32_t)i) / (uint32_t)STG);
            mbar_wait(b_full + 8 * i, (f / (uint32_t)STG) & 1u, a.status, f2);
        }
    } else if (warp == 1) {
        // ============================================================ MMA issuer
        int st = 0;
        uint32_t ph = 0, it = 0, ech = 0;
        const uint32_t id1 = idesc_bf16(TC_M, SR), id2 = idesc_bf16(TC_M, 128);
        for (int t = cl; t < n_tiles && !failed; t += ncl) {
            const int4 tile = a.contig[t];
            const int id = tile.x;
            const int r_n = a.ranks[id];
            if (r_n < 1 || r_n > R) continue;
            if (MODE != MODE_EXPAND) {
                if (!warp_wait(b_d1free, (it & 1u) ^ 1u, a.status, failed)) break;
                tc_fence_after();
                for (int kc = k_lo; kc < k_hi; ++kc) {
                    if (!warp_wait(b_full + 8 * st, ph, a.status, failed)) break;
                    tc_fence_after();
                    if (lane == 0) {
                        const uint32_t slot = ring + (uint32_t)st * slot_bytes;
                        const int nb = min(2, (a.d_in - kc * 128 + 63) >> 6);
                        for (int b = 0; b < nb; ++b)
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                tc_mma(tmem + TC_D1_COL, desc_sw128(slot + b * TC_BOX + kk * 32),
                                       desc_sw128(slot + TC_XY + (uint32_t)(b * SR) * 128u + kk * 32),
                                       id1, (kc > k_lo || b > 0 || kk > 0) ? 1u : 0u);
                        tc_commit(b_empty + 8 * st);
                    }
                    __syncwarp();
                    if (++st == STG) {
                        st = 0;
                        ph ^= 1u;
                    }
                }
                if (failed) break;
                if (lane == 0) tc_commit(b_d1full);
                __syncwarp();
            }
            if (MODE != MODE_SHRINK) {
                if (!warp_wait(b_vfull, it & 1u, a.status, failed)) break;
                tc_fence_after();
                const int ksteps = (r_n + 15) >> 4;
                int s = es0, c0 = ec0;
                for (int e = e_lo; e < e_hi; ++e) {
                    const uint32_t buf = ech & 1u;
                    if (!warp_wait(b_d2empty + 8 * buf, ((ech >> 1) & 1u) ^ 1u, a.status, failed))
                        break;
                    if (!warp_wait(b_full + 8 * st, ph, a.status, failed)) break;
                    tc_fence_after();
                    const uint32_t slot = ring + (uint32_t)st * slot_bytes;
                    if (r_n & 15) {   // zero B's ranks r_n .. 16*ksteps-1 (padding)
                        for (int g = r_n >> 3; g < 2 * ksteps; ++g) {
                            const int keep = max(0, r_n - 8 * g);
                            for (int nrow = lane; nrow < 128; nrow += 32) {
                                const uint32_t ad = slot + TC_XY + g * 2048u + nrow * 16u;
                                sts128(ad, keep8(lds128(ad), keep));
                            }
                        }
                        fence_proxy_async();
                        __syncwarp();
                    }
                    if (lane == 0) {
                        const uint32_t vh = vbuf + (uint32_t)(2 * s * R) * 256u, vl = vh + (uint32_t)R * 256u;
                        const uint32_t d = tmem + buf * 128u;
                        for (int kk = 0; kk < ksteps; ++kk) {
                            const uint64_t db = desc_plain(slot + TC_XY + kk * 4096u);
                            tc_mma(d, desc_plain(vh + kk * 4096u), db, id2, kk > 0 ? 1u : 0u);
                            tc_mma(d, desc_plain(vl + kk * 4096u), db, id2, 1u);
                        }
                        tc_commit(b_d2full + 8 * buf);
                    }
                    __syncwarp();
                    ++ech;
                    if (++st == STG) {
                        st = 0;
                        ph ^= 1u;
                    }
                    c0 += 128;
                    if (c0 >= a.sl.d_out[s]) {
                        ++s;
                        c0 = 0;
                    }
                }
                if (failed) break;
            }
            ++it;
        }
        // drain: every MMA this warp issued has completed
        if (lane == 0) tc_commit(b_mma);
        __syncwarp();
        bool f2 = false;
        warp_wait(b_mma, 0, a.status, f2);
    } else if (warp < 10) {
        // ============================================================ epilogue
        const int q = warp & 3, h = (warp - 2) >> 2, m = 32 * q + lane;
        const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
        const int half = SR >> 1, n8 = half >> 3;   // D1 columns of this thread's half
        int st = 0;
        uint32_t ph = 0, it = 0, ech = 0;
        for (int t = cl; t < n_tiles && !failed; t += ncl) {
            const int4 tile = a.contig[t];
            const int id = tile.x, row0 = tile.y, cnt = tile.z;
            const int r_n = a.ranks[id];
            if (r_n < 1 || r_n > R) continue;
            float p[64];
            if (MODE != MODE_EXPAND) {
                for (int kc = k_lo; kc < k_hi; ++kc)   // slots the MMA warp consumes
                    if (++st == STG) {
                        st = 0;
                        ph ^= 1u;
                    }
                if (!warp_wait(b_d1full, it & 1u, a.status, failed)) break;
                tc_fence_after();
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    if (j < n8) tc_ld8(lane_base + TC_D1_COL + (uint32_t)(h * half + 8 * j), &p[8 * j]);
                tc_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(b_d1free);
                if (xchg) {
                    // All-to-all of the partials through distributed shared memory: st.async
                    // stores that count their bytes on the receiver's barrier.  A buffer per
                    // tile parity: a block writes tile i+2 into a peer only after it received
                    // every peer's tile i+1 partials, which each peer sent after reading tile i.
                    const int NQ = SR >> 2, qh = half >> 2, q0 = h * qh;
                    const uint32_t xb = it & 1u, xbuf = xch + xb * xch_bytes, xbar = b_xfull + 8u * xb;
                    if (warp == 2 && lane == 0) mbar_expect_tx(xbar, xch_bytes);
                    const uint32_t off = (uint32_t)(((int)crank * NQ + q0) * 128 + m) * 16u;
                    for (int k = 0; k < C; ++k) {
                        const uint32_t rb = map_rank(xbuf, (uint32_t)k) + off;
                        const uint32_t rbar = map_rank(xbar, (uint32_t)k);
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            if (j < qh)
                                st_async_f4(rb + j * 2048u, p[4 * j], p[4 * j + 1], p[4 * j + 2],
                                            p[4 * j + 3], rbar);
                    }
                    if (!warp_wait(xbar, (it >> 1) & 1u, a.status, failed)) break;
#pragma unroll
                    for (int j = 0; j < 64; ++j) p[j] = 0.f;
                    for (int src = 0; src < C; ++src) {
                        const uint32_t lb = xbuf + (uint32_t)((src * NQ + q0) * 128 + m) * 16u;
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            if (j < qh) {
                                const float4 v = lds128f(lb + j * 2048u);
                                p[4 * j] += v.x;
                                p[4 * j + 1] += v.y;
                                p[4 * j + 2] += v.z;
                                p[4 * j + 3] += v.w;
                            }
                    }
                }
                if (MODE == MODE_SHRINK) {
                    // v rows of the tile; with a cluster, block c writes the rows m = c (mod C)
                    if (m < cnt && (m % C) == (int)crank) {
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            if (j < n8) {
                                const int col = h * half + 8 * j, s = col / R, kl = col - s * R;
                                float *dst = a.v + ((int64_t)s * a.T + row0 + m) * R + kl;
#pragma unroll
                                for (int e = 0; e < 8; ++e)
                                    if (kl + e < r_n) dst[e] = p[8 * j + e];
                            }
                    }
                    ++it;
                    continue;
                }
            } else {
                // s v from the caller's v (rows of the tile; zero beyond it)
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    if (j < n8) {
                        const int col = h * half + 8 * j, s = col / R, kl = col - s * R;
                        const float *src = a.v + ((int64_t)s * a.T + row0 + min(m, cnt - 1)) * R + kl;
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            p[8 * j + e] = (m < cnt && kl + e < r_n) ? src[e] : 0.f;
                    }
            }
            if (MODE != MODE_SHRINK) {
                // s v -> bf16 hi + lo in the no-swizzle K-major layout of the expand MMA
                const float scale = a.alphas[id] / (float)r_n;
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    if (j < n8) {
                        const int col = h * half + 8 * j, s = col / R, kl = col - s * R;
                        uint4 hi, lo;
                        uint32_t *hw = &hi.x, *lw = &lo.x;
#pragma unroll
                        for (int w = 0; w < 4; ++w) {
                            const float v0 = kl + 2 * w < r_n ? scale * p[8 * j + 2 * w] : 0.f;
                            const float v1 = kl + 2 * w + 1 < r_n ? scale * p[8 * j + 2 * w + 1] : 0.f;
                            hw[w] = pack_bf16x2(v0, v1);
                            lw[w] = pack_bf16x2(v0 - bf16_lo(hw[w]), v1 - bf16_hi(hw[w]));
                        }
                        const uint32_t va =
                            vbuf + (uint32_t)((2 * s) * (R >> 3) + (kl >> 3)) * 2048u + (uint32_t)m * 16u;
                        sts128(va, hi);
                        sts128(va + (uint32_t)R * 256u, lo);
                    }
                fence_proxy_async();
                __syncwarp();
                if (lane == 0) mbar_arrive(b_vfull);

                const bool fulltile = cnt == TC_M;
                int s = es0, c0 = ec0;
                for (int e = e_lo; e < e_hi; ++e) {
                    const uint32_t buf = ech & 1u;
                    if (!warp_wait(b_d2full + 8 * buf, (ech >> 1) & 1u, a.status, failed)) break;
                    if (!warp_wait(b_full + 8 * st, ph, a.status, failed)) break;
                    tc_fence_after();
                    float d[64];
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        tc_ld16(lane_base + buf * 128u + (uint32_t)(64 * h + 16 * j), &d[16 * j]);
                    tc_wait_ld();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(b_d2empty + 8 * buf);

                    const int d_out = a.sl.d_out[s];
                    const int cb = c0 + 64 * h;   // first slice-local column of this half's box
                    const uint32_t ybox = ring + (uint32_t)st * slot_bytes + (uint32_t)h * TC_BOX;
                    if (cb < d_out) {
                        const uint32_t rowa = ybox + (uint32_t)(m >> 3) * 1024u + (uint32_t)(m & 7) * 128u;
                        __nv_bfloat16 *yrow =
                            a.y + (int64_t)(row0 + min(m, cnt - 1)) * a.ld_y + a.sl.col_off[s] + cb;
#pragma unroll
                        for (int c = 0; c < 8; ++c)
                            if (cb + 8 * c < d_out) {
                                const uint32_t ad = rowa + (uint32_t)((c ^ (m & 7)) << 4);
                                const uint4 o = add8(lds128(ad), &d[8 * c]);
                                if (fulltile) sts128(ad, o);
                                else if (m < cnt) *reinterpret_cast<uint4 *>(yrow + 8 * c) = o;
                            }
                    }
                    if (fulltile) fence_proxy_async();   // generic writes -> the TMA store
                    __syncwarp();
                    if (lane == 0) mbar_arrive(b_ystage + 8 * st);   // this warp's rows are done
                    ++ech;
                    if (++st == STG) {
                        st = 0;
                        ph ^= 1u;
                    }
                    c0 += 128;
                    if (c0 >= d_out) {
                        ++s;
                        c0 = 0;
                    }
                }
                if (failed) break;
            }
            ++it;
        }
    } else if (MODE != MODE_SHRINK && warp == 10) {
        // ============================================================ store warp
        // Full tiles: TMA stores of the finished boxes (8-row boxes, one per lane),
        // the slot freed once they have read it (one chunk later, so that a store
        // stays in flight meanwhile).  Partial tiles: the epilogue stored the rows
        // itself; the slot is freed at once.
        int st = 0;
        uint32_t ph = 0;
        uint32_t yph = 0;   // bit st: phase parity of slot st's y barrier (expand uses only)
        int pend = -1;      // slot whose stores may still be reading it
        for (int t = cl; t < n_tiles && !failed; t += ncl) {
            const int4 tile = a.contig[t];
            const int id = tile.x, row0 = tile.y, cnt = tile.z;
            const int r_n = a.ranks[id];
            if (r_n < 1 || r_n > R) continue;
            for (int kc = k_lo; kc < k_hi; ++kc)
                if (++st == STG) {
                    st = 0;
                    ph ^= 1u;
                }
            const bool fulltile = cnt == TC_M;
            int s = es0, c0 = ec0;
            for (int e = e_lo; e < e_hi; ++e) {
                if (!warp_wait(b_ystage + 8 * st, (yph >> st) & 1u, a.status, failed)) break;
                const int d_out = a.sl.d_out[s];
                const int ny = d_out - c0 > 64 ? 2 : 1;
                const uint32_t slot = ring + (uint32_t)st * slot_bytes;
                if (fulltile) {
                    const int sbr = a.sbr, nsg = TC_M / sbr;
                    for (int i = lane; i < nsg * ny; i += 32) {
                        const int rg = i / ny, h = i - rg * ny;
                        tma_store_2d(&a.tmYs[s], c0 + 64 * h, row0 + sbr * rg,
                                     slot + h * TC_BOX + rg * (uint32_t)sbr * 128u);
                    }
                    bulk_commit();
                }
                if (pend >= 0) {
                    if (fulltile) bulk_wait_read_but1();
                    else bulk_wait_read();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(b_empty + 8 * pend);
                    pend = -1;
                }
                if (fulltile) {
                    pend = st;
                } else {
                    __syncwarp();
                    if (lane == 0) mbar_arrive(b_empty + 8 * st);
                }
                yph ^= 1u << st;
                if (++st == STG) {
                    st = 0;
                    ph ^= 1u;
                }
                c0 += 128;
                if (c0 >= d_out) {
                    ++s;
                    c0 = 0;
                }
            }
            if (pend >= 0) {   // no slot stays held into the next tile
                bulk_wait_read();
                __syncwarp();
                if (lane == 0) mbar_arrive(b_empty + 8 * pend);
                pend = -1;
            }
        }
        bulk_wait_all();
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem),
                     "r"(TC_TMEM_COLS)
                     : "memory");
    }
    cluster_sync_all();   // no block leaves while a peer may still write to it
}

// ------------------------------------------------------------------ host side
namespace {

const void *tc_fn(int mode) {
    return mode == MODE_FUSED    ? (const void *)sgmv_tc_kernel<MODE_FUSED>
           : mode == MODE_SHRINK ? (const void *)sgmv_tc_kernel<MODE_SHRINK>
                                 : (const void *)sgmv_tc_kernel<MODE_EXPAND>;
}

int env_int(const char *name, int dflt) {
    const char *s = std::getenv(name);
    return s && *s ? std::atoi(s) : dflt;
}

// Largest dynamic shared memory a block of fn may request (the opt-in limit
// less the kernel's static shared memory), set once as fn's attribute.  A
// failing runtime call leaves its error as the thread's last error: cleared
// here so that no later launch check reports it.
int tc_max_dynamic_smem(const void *fn, int dev) {
    int optin = 0;
    cudaFuncAttributes fa{};
    if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
        cudaFuncGetAttributes(&fa, fn) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    const int max_dyn = optin - (int)fa.sharedSizeBytes;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, max_dyn) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return max_dyn;
}

// Clusters of size C with `smem` bytes per block that fit the device at once.
int active_clusters(int mode, int C, size_t smem) {
    struct Key {
        int dev, mode, C;
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
            if (cache[i].dev == dev && cache[i].mode == mode && cache[i].C == C && cache[i].smem == smem)
                return cache[i].n;
    }
    const void *fn = tc_fn(mode);
    const int max_dyn = tc_max_dynamic_smem(fn, dev);
    if (max_dyn <= 0 || smem > (size_t)max_dyn) return 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(C, 1, 1);
    cfg.blockDim = dim3(TC_THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) != cudaSuccess) {
        cudaGetLastError();
        n = 0;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (used < 64) cache[used++] = Key{dev, mode, C, smem, n};
    return n;
}

}  // namespace

int launch_sgmv_tc(int mode, TcArgs &a, cudaStream_t st, int *idle_sms) {
    if (idle_sms) *idle_sms = 0;
    if (a.max_contig <= 0 || a.T <= 0) return LORA_OK;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int optin = tc_max_dynamic_smem(tc_fn(mode), dev);
    if (optin <= 0) return LORA_ERR_SHAPE;
    const int SR = a.sl.n * a.r_max;
    const int nk = (a.d_in + 127) / 128;
    int NE = 0;
    for (int s = 0; s < a.sl.n; ++s) NE += (a.sl.d_out[s] + 127) / 128;
    // Tiles to expect: every row in a full tile (the tile list on the device may be longer).
    const int est = std::max(1, std::min(a.max_contig, (a.T + TC_M - 1) / TC_M));
    const int forced_c = env_int("LORA_TC_CLUSTER", 0), forced_s = env_int("LORA_TC_STAGES", 0);

    int best_c = 0, best_stages = 0, best_ncl = 0;
    int cand_stages[9] = {}, cand_ncl[9] = {};
    double best = -1.0;
    for (int C = 1; C <= 8; C <<= 1) {
        if (forced_c && C != forced_c) continue;
        if (mode != MODE_EXPAND && nk < C) continue;
        if (mode != MODE_SHRINK && NE < C) continue;
        int stages = 0;
        for (int s = TC_MAX_STAGES; s >= 2; --s)
            if (sgmv_tc_smem_bytes(mode, s, SR, C) <= (size_t)optin) {
                stages = s;
                break;
            }
        if (forced_s >= 2 && forced_s <= stages) stages = forced_s;
        if (stages < 2) continue;
        const size_t smem = sgmv_tc_smem_bytes(mode, stages, SR, C);
        const int ncl = active_clusters(mode, C, smem);
        if (ncl < 1) continue;
        cand_stages[C] = stages;
        cand_ncl[C] = ncl;
        // fraction of the SMs busy over the whole launch, with whole rounds of tiles
        const int rounds = (est + ncl - 1) / ncl;
        const double score = (double)est / ((double)rounds * ncl) * ((double)ncl * C / sms);
        if (score > best * 1.03) {
            best = score;
            best_c = C;
            best_stages = stages;
            best_ncl = ncl;
        }
    }
    if (best_c == 0) return LORA_ERR_SHAPE;
    // Output much wider than the input, and fewer tiles than clusters: twice the
    // blocks per tile spread each tile's long expand over more SMs.  Measured on
    // B200 (8192 -> 28672, 60 tiles): 246 us with 4 blocks against 264 with 2; for
    // 28672 -> 8192 the 2-block choice stays (157 against 189).
    if (!forced_c && mode != MODE_SHRINK && (int64_t)NE * 128 >= 2LL * a.d_in && est < best_ncl &&
        best_c == 2 && cand_ncl[4] > 0) {
        best_c *= 2;
        best_stages = cand_stages[best_c];
        best_ncl = cand_ncl[best_c];
    }
    a.C = best_c;
    a.stages = best_stages;
    const size_t smem = sgmv_tc_smem_bytes(mode, best_stages, SR, best_c);
    const int clusters = std::min(best_ncl, a.max_contig);
    if (idle_sms) *idle_sms = std::max(0, clusters - est) * best_c;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(best_c * clusters, 1, 1);
    cfg.blockDim = dim3(TC_THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = best_c;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t err;
    if (mode == MODE_FUSED)
        err = cudaLaunchKernelEx(&cfg, sgmv_tc_kernel<MODE_FUSED>, a);
    else if (mode == MODE_SHRINK)
        err = cudaLaunchKernelEx(&cfg, sgmv_tc_kernel<MODE_SHRINK>, a);
    else
        err = cudaLaunchKernelEx(&cfg, sgmv_tc_kernel<MODE_EXPAND>, a);
    return cuda_rc(err);
}

}  // namespace lora
