// Merge and unmerge of one adapter into a base weight (page "LoRA service:
// multi-adapter dynamic loading", section 1: a single-tenant deployment folds
// the adapter into the base weight, W' = W + B A, so serving costs nothing
// extra; the same page, section 12, contrasts it with the per-request adapter
// path):
//
//     W[o][i] += sign * (alpha_n / r_n) * sum_{k < r_n} B[n][o][k] A[n][k][i]
//
// A rank-r_n update of a dense d_out x d_in matrix: every element of W is read
// and written once (4 bytes for bf16) for 2 r_n multiply-adds, so the kernel is
// bound by HBM.  The products run on the 5th-generation tensor cores: a tile
// of 128 output rows x 128 input columns is one tcgen05.mma chain
//     D[128][128] = Bn[o0 : o0+128][0 : 16k] . (An[0 : 16k][i0 : i0+128])^T      (K = r_n padded to 16)
// with both operands K-major in shared memory (8-row x 16-byte core matrices,
// no swizzle): Bn's rows arrive through TMA boxes of 8 ranks x 128 rows, and
// An's transpose is written once per column block by the block's threads.
// The fp32 accumulator sits in tensor memory; four epilogue warps read it
// (tcgen05.ld), scale it, add the W row segment they loaded while the copy and
// the MMA ran, and store W rounded once to bf16.  Padding ranks (k >= r_n) are
// zeroed in both operands before the MMA, so whatever they hold never reaches
// W.  Tiles are taken in column-block order, each block a contiguous run, so a
// block rebuilds An's transpose only when its run crosses into the next column
// block.  At most four blocks share an SM (128 tensor-memory columns each).
//
// fp32 data, or shapes the TMA copies cannot take, go to a plain kernel (one
// thread per element, fp32 products).
#include "kernels.cuh"
#include "ptx.cuh"
#include "tc.cuh"

#include <algorithm>
#include <mutex>

namespace lora {

constexpr int MG_THREADS = 192;              // warp 0 copies + MMA, warp 1 tensor memory, 2-5 epilogue
constexpr uint32_t MG_TMEM_COLS = 128;
constexpr uint32_t MG_OP_BYTES = 16384;      // one operand: 128 rows x 64 ranks bf16
constexpr size_t MG_SMEM = 48 * 1024;        // 2 operands + alignment; caps residency at 4 blocks / SM

struct MgArgs {
    CUtensorMap tmB;          // B as [N*d_out rows][r_max], boxes of 8 ranks x 128 rows, no swizzle
    __nv_bfloat16 *W;
    int64_t ld_w;
    int d_out, d_in;
    const __nv_bfloat16 *A;   // A [N][r_max][d_in]
    int r_max, n;
    const int32_t *ranks;
    const float *alphas;
    float sign;
    int32_t *status;
};

__global__ void __launch_bounds__(MG_THREADS) merge_tc_kernel(const __grid_constant__ MgArgs a) {
    extern __shared__ __align__(1024) unsigned char mg_sm[];
    __shared__ uint32_t tmem_sm;
    __shared__ __align__(8) uint64_t bars[3];   // B tile landed / D ready / D read out
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t base = (smem_u32(mg_sm) + 1023u) & ~1023u;
    const uint32_t bm = base, at = base + MG_OP_BYTES;
    const uint32_t b_full = smem_u32(&bars[0]), b_mma = smem_u32(&bars[1]), b_free = smem_u32(&bars[2]);

    const int r = a.ranks[a.n];
    if (r < 1 || r > a.r_max) {
        if (blockIdx.x == 0 && tid == 0) atomicOr(a.status, LORA_DEV_BAD_RANK);
        return;
    }
    const int n_rt = (a.d_out + 127) >> 7, n_cb = (a.d_in + 127) >> 7;
    const int n_tiles = n_rt * n_cb;
    const int per = (n_tiles + (int)gridDim.x - 1) / (int)gridDim.x;
    const int t_lo = (int)blockIdx.x * per, t_hi = min(n_tiles, t_lo + per);
    if (t_lo >= t_hi) return;
    const float scale = a.sign * a.alphas[a.n] / (float)r;
    const int ksteps = (r + 15) >> 4, ngrp = (r + 7) >> 3;

    if (tid == 0) {
        mbar_init(b_full, 1);
        mbar_init(b_mma, 1);
        mbar_init(b_free, 4);
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    if (warp == 0 && lane == 0) prefetch_tmap(&a.tmB);
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(
                         smem_u32(&tmem_sm)),
                     "r"(MG_TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_sm;
    const uint32_t idesc = idesc_bf16(128, 128);
    bool failed = false;
    int cur_cb = -1;
    uint32_t it = 0;
    for (int t = t_lo; t < t_hi; ++t, ++it) {
        const int cb = t / n_rt, rt = t - cb * n_rt;
        const int i0 = cb * 128, o0 = rt * 128;
        if (cb != cur_cb) {   // An^T for input columns i0 .. i0+127, ranks 0 .. 16*ksteps-1
            cur_cb = cb;
            __syncthreads();   // the last MMA that read the previous transpose has completed
            const __nv_bfloat16 *src = a.A + (int64_t)a.n * a.r_max * a.d_in + i0;
            unsigned short *dst = reinterpret_cast<unsigned short *>(__cvta_shared_to_generic(at));
            for (int idx = tid; idx < 16 * ksteps * 128; idx += MG_THREADS) {
                const int k = idx >> 7, c = idx & 127;
                unsigned short v = 0;
                if (k < r && i0 + c < a.d_in)
                    v = __bfloat16_as_ushort(src[(int64_t)k * a.d_in + c]);
                dst[((k >> 3) * 2048 + (c >> 3) * 128 + (c & 7) * 16 + (k & 7) * 2) >> 1] = v;
            }
            fence_proxy_async();   // the tensor core reads what these generic stores wrote
            __syncthreads();
        }
        if (warp == 0) {
            if (!failed) {
                if (lane == 0) {
                    mbar_expect_tx(b_full, (unsigned)ngrp * 2048u);
                    for (int gq = 0; gq < ngrp; ++gq)
                        tma_2d(bm + (uint32_t)gq * 2048u, &a.tmB, 8 * gq, a.n * a.d_out + o0, b_full);
                }
                __syncwarp();
                warp_wait(b_full, it & 1u, a.status, failed);
            }
            if (!failed) {
                if (r & 15) {   // ranks r .. 16*ksteps-1: zero (loaded padding, or never loaded)
                    for (int gq = r >> 3; gq < 2 * ksteps; ++gq) {
                        const int keep = max(0, r - 8 * gq);
                        for (int row = lane; row < 128; row += 32) {
                            const uint32_t ad = bm + (uint32_t)gq * 2048u + (uint32_t)row * 16u;
                            sts128(ad, keep8(lds128(ad), keep));
                        }
                    }
                    fence_proxy_async();
                    __syncwarp();
                }
                if (it > 0) warp_wait(b_free, (it - 1) & 1u, a.status, failed);   // D read out
            }
            if (!failed) {
                tc_fence_after();
                if (lane == 0) {
                    for (int kk = 0; kk < ksteps; ++kk)
                        tc_mma(tmem, desc_plain(bm + (uint32_t)kk * 4096u),
                               desc_plain(at + (uint32_t)kk * 4096u), idesc, kk > 0 ? 1u : 0u);
                    tc_commit(b_mma);
                }
                __syncwarp();
                warp_wait(b_mma, it & 1u, a.status, failed);   // B tile and An^T free again
            }
        } else if (warp >= 2) {
            const int q = warp & 3;
            const int o = o0 + 32 * q + lane;
            const int ncol = min(128, a.d_in - i0);
            const bool row_ok = o < a.d_out;
            __nv_bfloat16 *wrow = a.W + (int64_t)(row_ok ? o : 0) * a.ld_w + i0;
            uint4 wv[16];
#pragma unroll
            for (int j = 0; j < 16; ++j)   // W first: its latency overlaps the copy and the MMA
                wv[j] = (row_ok && 8 * j < ncol) ? *reinterpret_cast<const uint4 *>(wrow + 8 * j)
                                                 : make_uint4(0, 0, 0, 0);
            const bool ok = warp_wait(b_mma, it & 1u, a.status, failed);
            tc_fence_after();
            if (ok) {
                const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
#pragma unroll
                for (int c16 = 0; c16 < 8; ++c16) {
                    float d[16];
                    tc_ld16(lane_base + (uint32_t)(16 * c16), d);
                    tc_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; ++e) d[e] *= scale;
                    wv[2 * c16] = add8(wv[2 * c16], d);
                    wv[2 * c16 + 1] = add8(wv[2 * c16 + 1], d + 8);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(b_free);
            if (ok) {
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    if (row_ok && 8 * j < ncol) *reinterpret_cast<uint4 *>(wrow + 8 * j) = wv[j];
            }
        }
    }
    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem),
                     "r"(MG_TMEM_COLS)
                     : "memory");
    }
}

// One thread per element of W (grid-stride), fp32 products (fp32 data, or any shape).
template <typename E>
__global__ void merge_simt_kernel(E *W, int64_t ld_w, int d_out, int d_in, const E *A, const E *B,
                                  int r_max, int n, const int32_t *ranks, const float *alphas,
                                  float sign, int32_t *status) {
    const int r = ranks[n];
    if (r < 1 || r > r_max) {
        if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(status, LORA_DEV_BAD_RANK);
        return;
    }
    const float scale = sign * (alphas[n] / (float)r);
    const int64_t total = (int64_t)d_out * d_in;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int o = (int)(e / d_in), i = (int)(e - (int64_t)o * d_in);
        const E *Bo = B + ((int64_t)n * d_out + o) * r_max;
        const E *An = A + (int64_t)n * r_max * d_in + i;
        float acc = 0.f;
        for (int k = 0; k < r; ++k) acc = fmaf(load_elem(Bo + k), load_elem(An + (int64_t)k * d_in), acc);
        E *w = W + (int64_t)o * ld_w + i;
        store_elem(w, load_elem(w) + scale * acc);
    }
}

}  // namespace lora

extern "C" {

int lora_merge_adapter(void *W, int64_t ld_w, int32_t d_out, int32_t d_in, const void *A,
                       const void *B, int32_t N, int32_t r_max, int32_t n, const int32_t *ranks,
                       const float *alphas, int32_t sign, lora_dtype dtype, int32_t *status,
                       void *stream) {
    using namespace lora;
    if (!W || !A || !B || !ranks || !alphas || !status) return LORA_ERR_NULL;
    if (dtype != LORA_BF16 && dtype != LORA_FP32) return LORA_ERR_DTYPE;
    if (d_out < 1 || d_in < 1 || ld_w < d_in || N < 1 || N > LORA_MAX_ADAPTERS || n < 0 || n >= N ||
        (sign != 1 && sign != -1))
        return LORA_ERR_SHAPE;
    if (r_max < 1 || r_max > LORA_MAX_RANK) return LORA_ERR_RANK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    auto al = [](const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
    const bool tc = dtype == LORA_BF16 && r_max <= 64 && (r_max & 7) == 0 && (d_in & 7) == 0 &&
                    (ld_w & 7) == 0 && al(W) && al(B) && (int64_t)N * d_out < ((int64_t)1 << 31);
    if (tc) {
        MgArgs a{};
        if (tensor_map_2d(&a.tmB, B, (uint64_t)r_max, (uint64_t)N * d_out, 8, 128, 0) == LORA_OK) {
            a.W = static_cast<__nv_bfloat16 *>(W);
            a.ld_w = ld_w;
            a.d_out = d_out;
            a.d_in = d_in;
            a.A = static_cast<const __nv_bfloat16 *>(A);
            a.r_max = r_max;
            a.n = n;
            a.ranks = ranks;
            a.alphas = alphas;
            a.sign = (float)sign;
            a.status = status;
            static std::mutex mu;
            static uint64_t attr_done = 0;
            int dev = 0, sms = 148;
            cudaGetDevice(&dev);
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
            {
                std::lock_guard<std::mutex> lock(mu);
                if (!(attr_done & (1ull << (dev & 63)))) {
                    cudaFuncSetAttribute(merge_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)MG_SMEM);
                    attr_done |= 1ull << (dev & 63);
                }
            }
            const int tiles = ((d_out + 127) / 128) * ((d_in + 127) / 128);
            const int grid = std::max(1, std::min(tiles, 4 * sms));
            merge_tc_kernel<<<grid, MG_THREADS, MG_SMEM, st>>>(a);
            return cuda_rc(cudaGetLastError());
        }
    }
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t blocks = ((int64_t)d_out * d_in + 255) / 256;
    const int grid = (int)std::min<int64_t>(blocks, (int64_t)sms * 16);
    if (dtype == LORA_BF16)
        merge_simt_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(
            static_cast<__nv_bfloat16 *>(W), ld_w, d_out, d_in, static_cast<const __nv_bfloat16 *>(A),
            static_cast<const __nv_bfloat16 *>(B), r_max, n, ranks, alphas, (float)sign, status);
    else
        merge_simt_kernel<float><<<grid, 256, 0, st>>>(
            static_cast<float *>(W), ld_w, d_out, d_in, static_cast<const float *>(A),
            static_cast<const float *>(B), r_max, n, ranks, alphas, (float)sign, status);
    return cuda_rc(cudaGetLastError());
}

}  // extern "C"
