// Fused decode BGMV (page "Multi-LoRA Serving", section 3.2: BGMV-style
// grouped products; section 3.4: add_shrink then add_expand, grouped per
// adapter) for bf16, ranks up to 64.
//
// One unit of work = up to 16 rows that share an adapter (a gathered tile, or
// 16 rows of a contiguous tile).  A cluster of C thread blocks takes a unit:
//
//   shrink   block c reduces its 1/C share of d_in:  v_c[row][k] = sum_j x A^T
//            (warp-level bf16 tensor-core mma m16n8k16: M = 16 rows,
//            N = 8 ranks, K = 16 inputs; fp32 accumulation)
//   reduce   each block sums the C partials through distributed shared memory
//            (fixed order, so results are run-to-run identical)
//   expand   block c writes its 1/C share of the output columns: delta =
//            (s v) B^T with M = 16 rows, N = 8 columns, K = 16 ranks; s v is
//            split into bf16 hi + lo parts so the product keeps ~16 mantissa
//            bits; y is read, added in fp32 and rounded once.
//
// x, A, B and y cross HBM once; the rank-r intermediate never leaves the chip.
// The arithmetic intensity (about 4 multiply-adds per byte) would keep the
// fp32 pipe busier than HBM at the power-capped clock, so the multiply-adds
// run on the tensor pipe; the kernel is bounded by HBM bandwidth.
//
// Inside one 16-wide K step every thread loads 4 consecutive elements of each
// operand row and assigns them to its four k-slots of the mma fragment; the
// same assignment is used for both operands, so the sum is unchanged and all
// loads are plain contiguous vectors.
#include "kernels.cuh"

#include <cooperative_groups.h>

namespace cg = cooperative_groups;

namespace lora {

constexpr int BG_THREADS = 256;
constexpr int BG_WARPS = 8;
constexpr int BG_ROWS = 16;
constexpr int BG_RMAX = 64;
constexpr int BG_PART_STRIDE = 72;    // floats per row of the per-warp partial / staging tile
constexpr int BG_VF_STRIDE = 80;      // floats per row of the reduced v
constexpr int BG_COLS = 64;           // output columns per warp block




__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint4 ldg16(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ uint2 ldg8(const void *p) {
    uint2 r;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];\n"
                 : "=r"(r.x), "=r"(r.y)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ uint32_t u4_get(const uint4 &v, int i) {
    return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// Dynamic shared memory:
//   part   [8 warps][16][72] fp32   shrink partials, later the expand staging tiles
//   vcta   [S][16][64]       fp32   this block's partial v, read by the peers
//   vfull  [S][16][80]       fp32   reduced (and scaled) v
size_t bgmv_smem_bytes(int n_slices) {
    return (size_t)BG_WARPS * BG_ROWS * BG_PART_STRIDE * 4 +
           (size_t)n_slices * BG_ROWS * BG_RMAX * 4 + (size_t)n_slices * BG_ROWS * BG_VF_STRIDE * 4;
}

template <int MODE>
__global__ void __launch_bounds__(BG_THREADS, 2) bgmv_mma_kernel(BgArgs a) {
    extern __shared__ __align__(16) float bg_sm[];
    __shared__ int rows_sm[BG_ROWS];

    const int S = a.sl.n;
    float *part = bg_sm;
    float *vcta = part + BG_WARPS * BG_ROWS * BG_PART_STRIDE;
    float *vfull = vcta + S * BG_ROWS * BG_RMAX;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int C = gridDim.x, crank = blockIdx.x;

    const Unit u = resolve_unit(a.tiles, blockIdx.y);
    if (u.cnt == 0) return;                        // uniform over the cluster
    const int n = u.id;
    const int r_n = a.ranks[n];
    if (r_n < 1 || r_n > a.r_max) {
        if (crank == 0 && tid == 0) atomicOr(a.status, LORA_DEV_BAD_RANK);
        return;
    }
    if (tid < BG_ROWS) rows_sm[tid] = tid < u.cnt ? u.row(a.tiles, tid) : -1;
    __syncthreads();

    const int cnt = u.cnt;
    const int nb8 = (r_n + 7) >> 3;

    if (MODE != MODE_EXPAND) {
        // ------------------------------------------------------------ shrink
        const int row_g = rows_sm[g], row_h = rows_sm[g + 8];
        const int n64 = (a.d_in + 63) >> 6;
        const int st_lo = (int)((int64_t)crank * n64 / C), st_hi = (int)((int64_t)(crank + 1) * n64 / C);
        const __nv_bfloat16 *xg = row_g >= 0 ? a.x + (int64_t)row_g * a.ld_x : nullptr;
        const __nv_bfloat16 *xh = row_h >= 0 ? a.x + (int64_t)row_h * a.ld_x : nullptr;
        float *mypart = part + warp * BG_ROWS * BG_PART_STRIDE;

        for (int s = 0; s < S; ++s) {
            const __nv_bfloat16 *An =
                static_cast<const __nv_bfloat16 *>(a.sl.A[s]) + (int64_t)n * a.r_max * a.d_in;
            float acc[8][4];
#pragma unroll
            for (int kb = 0; kb < 8; ++kb)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[kb][e] = 0.f;

            for (int st = st_lo + warp; st < st_hi; st += BG_WARPS) {
                const int j = st * 64 + 16 * t;
                const bool in0 = j + 8 <= a.d_in, in1 = j + 16 <= a.d_in;
                const uint4 z = make_uint4(0, 0, 0, 0);
                const uint4 xg0 = (xg && in0) ? ldg16(xg + j) : z;
                const uint4 xg1 = (xg && in1) ? ldg16(xg + j + 8) : z;
                const uint4 xh0 = (xh && in0) ? ldg16(xh + j) : z;
                const uint4 xh1 = (xh && in1) ? ldg16(xh + j + 8) : z;
                uint4 av0[8], av1[8];
#pragma unroll
                for (int kb = 0; kb < 8; ++kb) {
                    const int k = kb * 8 + g;
                    const bool ok = kb < nb8 && k < r_n;
                    const __nv_bfloat16 *ap = An + (int64_t)k * a.d_in + j;
                    av0[kb] = (ok && in0) ? ldg16(ap) : z;
                    av1[kb] = (ok && in1) ? ldg16(ap + 8) : z;
                }
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    const uint4 &xa = b < 2 ? xg0 : xg1;
                    const uint4 &xb = b < 2 ? xh0 : xh1;
                    const int q = (b & 1) * 2;
                    const uint32_t fa[4] = {u4_get(xa, q), u4_get(xb, q), u4_get(xa, q + 1),
                                            u4_get(xb, q + 1)};
#pragma unroll
                    for (int kb = 0; kb < 8; ++kb) {
                        if (kb < nb8) {
                            const uint4 &av = b < 2 ? av0[kb] : av1[kb];
                            mma16816(acc[kb], fa, u4_get(av, q), u4_get(av, q + 1));
                        }
                    }
                }
            }
            // per-warp partial -> shared, then the block's sum in warp order
#pragma unroll
            for (int kb = 0; kb < 8; ++kb) {
                if (kb < nb8) {
                    const int k = kb * 8 + 2 * t;
                    *reinterpret_cast<float2 *>(&mypart[g * BG_PART_STRIDE + k]) =
                        make_float2(acc[kb][0], acc[kb][1]);
                    *reinterpret_cast<float2 *>(&mypart[(g + 8) * BG_PART_STRIDE + k]) =
                        make_float2(acc[kb][2], acc[kb][3]);
                }
            }
            __syncthreads();
            for (int e = tid; e < BG_ROWS * BG_RMAX; e += BG_THREADS) {
                const int row = e >> 6, k = e & 63;
                float sum = 0.f;
                if (k < nb8 * 8) {
#pragma unroll
                    for (int w = 0; w < BG_WARPS; ++w)
                        sum += part[(w * BG_ROWS + row) * BG_PART_STRIDE + k];
                }
                vcta[(s * BG_ROWS + row) * BG_RMAX + k] = sum;
            }
            __syncthreads();
        }

        // ------------------------------------------------------------ cluster reduce
        cg::cluster_group cluster = cg::this_cluster();
        cluster.sync();
        const float scale = MODE == MODE_FUSED ? a.scales[n] : 1.f;
        for (int e = tid; e < S * BG_ROWS * BG_RMAX; e += BG_THREADS) {
            const int s = e / (BG_ROWS * BG_RMAX);
            const int rem = e - s * BG_ROWS * BG_RMAX;
            const int row = rem >> 6, k = rem & 63;
            float sum = 0.f;
            if (row < cnt && k < r_n) {
                for (int c = 0; c < C; ++c) {
                    const float *peer = cluster.map_shared_rank(vcta, c);
                    sum += peer[e];
                }
            }
            vfull[(s * BG_ROWS + row) * BG_VF_STRIDE + k] = scale * sum;
        }
        cluster.sync();

        if (MODE == MODE_SHRINK) {
            if (crank == 0) {
                for (int e = tid; e < S * BG_ROWS * BG_RMAX; e += BG_THREADS) {
                    const int s = e / (BG_ROWS * BG_RMAX);
                    const int rem = e - s * BG_ROWS * BG_RMAX;
                    const int row = rem >> 6, k = rem & 63;
                    if (row < cnt && k < r_n)
                        a.v[((int64_t)s * a.T + rows_sm[row]) * a.r_max + k] =
                            vfull[(s * BG_ROWS + row) * BG_VF_STRIDE + k];
                }
            }
            return;
        }
    } else {
        const float scale = a.scales[n];
        for (int e = tid; e < S * BG_ROWS * BG_RMAX; e += BG_THREADS) {
            const int s = e / (BG_ROWS * BG_RMAX);
            const int rem = e - s * BG_ROWS * BG_RMAX;
            const int row = rem >> 6, k = rem & 63;
            float val = 0.f;
            if (row < cnt && k < r_n)
                val = scale * a.v[((int64_t)s * a.T + rows_sm[row]) * a.r_max + k];
            vfull[(s * BG_ROWS + row) * BG_VF_STRIDE + k] = val;
        }
    }
    __syncthreads();

    // ---------------------------------------------------------------- expand
    int nbt = 0;
    for (int s = 0; s < S; ++s) nbt += (a.sl.d_out[s] + BG_COLS - 1) / BG_COLS;
    const int b_lo = (int)((int64_t)crank * nbt / C), b_hi = (int)((int64_t)(crank + 1) * nbt / C);
    const int nkb = (r_n + 15) >> 4;
    float *stage = part + warp * BG_ROWS * BG_PART_STRIDE;

    int cur_s = -1, s_first = 0;
    uint32_t ahi[4][4], alo[4][4];
    for (int blk = b_lo + warp; blk < b_hi; blk += BG_WARPS) {
        // which slice, which block inside it
        int s = 0, first = 0;
        while (true) {
            const int nb_s = (a.sl.d_out[s] + BG_COLS - 1) / BG_COLS;
            if (blk < first + nb_s) break;
            first += nb_s;
            ++s;
        }
        if (s != cur_s) {   // fragments of s*v for this slice
            cur_s = s;
            s_first = first;
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
        const int d_out = a.sl.d_out[s];
        const int c0 = (blk - s_first) * BG_COLS;
        const __nv_bfloat16 *Bn =
            static_cast<const __nv_bfloat16 *>(a.sl.B[s]) + (int64_t)n * d_out * a.r_max;

        // y of this block: lane owns columns c0 + 2*lane, +1 of every row
        const int ycol = c0 + 2 * lane;
        const bool ycol_ok = ycol < d_out;
        uint32_t yv[BG_ROWS];
#pragma unroll
        for (int r = 0; r < BG_ROWS; ++r) {
            yv[r] = 0;
            if (r < cnt && ycol_ok)
                yv[r] = *reinterpret_cast<const uint32_t *>(
                    a.y + (int64_t)rows_sm[r] * a.ld_y + a.sl.col_off[s] + ycol);
        }

        float acc[8][4];
#pragma unroll
        for (int nb = 0; nb < 8; ++nb)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[nb][e] = 0.f;
#pragma unroll
        for (int kb = 0; kb < 4; ++kb) {
            if (kb < nkb) {
                const int k = kb * 16 + 4 * t;
                uint2 bv[8];
#pragma unroll
                for (int nb = 0; nb < 8; ++nb) {
                    const int col = c0 + nb * 8 + g;
                    bv[nb] = make_uint2(0, 0);
                    if (col < d_out && k < r_n) {
                        bv[nb] = ldg8(Bn + (int64_t)col * a.r_max + k);
                        if (k + 4 > r_n) {   // rank ends inside this group of 4
                            const int keep = r_n - k;
                            if (keep < 2) bv[nb].x &= 0xffffu;
                            if (keep < 3) bv[nb].y = 0;
                            else bv[nb].y &= 0xffffu;
                        }
                    }
                }
#pragma unroll
                for (int nb = 0; nb < 8; ++nb) {
                    mma16816(acc[nb], ahi[kb], bv[nb].x, bv[nb].y);
                    mma16816(acc[nb], alo[kb], bv[nb].x, bv[nb].y);
                }
            }
        }
        // stage the 16 x 64 fp32 delta, then add it to y row by row
#pragma unroll
        for (int nb = 0; nb < 8; ++nb) {
            *reinterpret_cast<float2 *>(&stage[g * BG_PART_STRIDE + nb * 8 + 2 * t]) =
                make_float2(acc[nb][0], acc[nb][1]);
            *reinterpret_cast<float2 *>(&stage[(g + 8) * BG_PART_STRIDE + nb * 8 + 2 * t]) =
                make_float2(acc[nb][2], acc[nb][3]);
        }
        __syncwarp();
#pragma unroll
        for (int r = 0; r < BG_ROWS; ++r) {
            if (r < cnt && ycol_ok) {
                const float2 d = *reinterpret_cast<const float2 *>(&stage[r * BG_PART_STRIDE + 2 * lane]);
                const uint32_t out = pack_bf16x2(bf16_lo(yv[r]) + d.x, bf16_hi(yv[r]) + d.y);
                *reinterpret_cast<uint32_t *>(a.y + (int64_t)rows_sm[r] * a.ld_y + a.sl.col_off[s] +
                                              ycol) = out;
            }
        }
        __syncwarp();
    }
}

int launch_bgmv(int mode, const BgArgs &a, int n_units, int cluster, cudaStream_t st) {
    const size_t smem = bgmv_smem_bytes(a.sl.n);
    static bool attr_done[3] = {false, false, false};
    const void *fn = mode == MODE_FUSED    ? (const void *)bgmv_mma_kernel<MODE_FUSED>
                     : mode == MODE_SHRINK ? (const void *)bgmv_mma_kernel<MODE_SHRINK>
                                           : (const void *)bgmv_mma_kernel<MODE_EXPAND>;
    if (!attr_done[mode]) {
        cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)bgmv_smem_bytes(LORA_MAX_SLICES));
        attr_done[mode] = true;
    }
    if (n_units <= 0) return LORA_OK;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(cluster, n_units, 1);
    cfg.blockDim = dim3(BG_THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = mode == MODE_EXPAND ? 0 : 1;
    cudaError_t err;
    if (mode == MODE_FUSED)
        err = cudaLaunchKernelEx(&cfg, bgmv_mma_kernel<MODE_FUSED>, a);
    else if (mode == MODE_SHRINK)
        err = cudaLaunchKernelEx(&cfg, bgmv_mma_kernel<MODE_SHRINK>, a);
    else
        err = cudaLaunchKernelEx(&cfg, bgmv_mma_kernel<MODE_EXPAND>, a);
    return err == cudaSuccess ? LORA_OK : LORA_ERR_CUDA;
}

}  // namespace lora
