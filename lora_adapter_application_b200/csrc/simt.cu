// General multi-LoRA delta kernel on the CUDA cores: any element type the
// library takes (fp32 and bf16), any alignment, ranks up to LORA_MAX_RANK.
// It is the path for fp32 data (fp32 products, no tf32) and for inputs that
// the vectorised kernels cannot take.  One thread block per unit of rows;
// same three modes as the BGMV kernel (fused, shrink only, expand only).
//
//   shrink  one warp per (slice, row, rank) triple: lanes stride over d_in,
//           fp32 products, a fixed-order shuffle tree adds the lanes
//   expand  one thread per output column: y += s * sum_k B[c][k] v[k]
#include "kernels.cuh"

#include <mutex>

namespace lora {

constexpr int SIMT_THREADS = 256;
constexpr int SIMT_ROWS = 16;



size_t simt_smem_bytes(int n_slices, int r_max) {
    return (size_t)n_slices * SIMT_ROWS * r_max * sizeof(float);
}

template <typename E, int MODE>
__global__ void __launch_bounds__(SIMT_THREADS) simt_kernel(SimtArgs a) {
    extern __shared__ float vfull[];   // [S][16][r_max]
    __shared__ int rows_sm[SIMT_ROWS];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int S = a.sl.n;

    const Unit u = resolve_unit(a.tiles, blockIdx.x);
    if (u.cnt == 0) return;
    const int n = u.id;
    const int r_n = a.ranks[n];
    if (r_n < 1 || r_n > a.r_max) {
        if (tid == 0) atomicOr(a.status, LORA_DEV_BAD_RANK);
        return;
    }
    const float scale = MODE == 1 ? 1.f : a.alphas[n] / (float)r_n;
    const E *x = static_cast<const E *>(a.x);
    E *y = static_cast<E *>(a.y);

    // the unit's rows, 16 at a time
    for (int q0 = 0; q0 < u.cnt; q0 += SIMT_ROWS) {
        const int cnt = min(SIMT_ROWS, u.cnt - q0);
        __syncthreads();   // the previous group is done with rows_sm and vfull
        if (tid < SIMT_ROWS) rows_sm[tid] = tid < cnt ? u.row(a.tiles, q0 + tid) : -1;
        __syncthreads();

        if (MODE == 2) {   // expand only: v from global, scaled
            for (int e = tid; e < S * cnt * r_n; e += SIMT_THREADS) {
                const int s = e / (cnt * r_n), rem = e - s * cnt * r_n;
                const int row = rem / r_n, k = rem - row * r_n;
                vfull[(s * SIMT_ROWS + row) * a.r_max + k] =
                    scale * a.v[((int64_t)s * a.T + rows_sm[row]) * a.r_max + k];
            }
        } else {
            for (int e = warp; e < S * cnt * r_n; e += SIMT_THREADS / 32) {
                const int s = e / (cnt * r_n), rem = e - s * cnt * r_n;
                const int row = rem / r_n, k = rem - row * r_n;
                const E *Ak = static_cast<const E *>(a.sl.A[s]) + ((int64_t)n * a.r_max + k) * a.d_in;
                const E *xr = x + (int64_t)rows_sm[row] * a.ld_x;
                float acc = 0.f;
                for (int j = lane; j < a.d_in; j += 32) acc = fmaf(load_elem(Ak + j), load_elem(xr + j), acc);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(FULL, acc, o);
                if (lane == 0) vfull[(s * SIMT_ROWS + row) * a.r_max + k] = scale * acc;
            }
        }
        __syncthreads();

        if (MODE == 1) {   // shrink only: write v
            for (int e = tid; e < S * cnt * r_n; e += SIMT_THREADS) {
                const int s = e / (cnt * r_n), rem = e - s * cnt * r_n;
                const int row = rem / r_n, k = rem - row * r_n;
                a.v[((int64_t)s * a.T + rows_sm[row]) * a.r_max + k] =
                    vfull[(s * SIMT_ROWS + row) * a.r_max + k];
            }
            continue;
        }

        const int total = a.sl.cat_off[S];
        for (int e = tid; e < total; e += SIMT_THREADS) {
            int s = 0;
            while (e >= a.sl.cat_off[s + 1]) ++s;
            const int c = e - a.sl.cat_off[s];
            const E *Bc = static_cast<const E *>(a.sl.B[s]) + ((int64_t)n * a.sl.d_out[s] + c) * a.r_max;
            const float *vs = vfull + s * SIMT_ROWS * a.r_max;
            for (int row = 0; row < cnt; ++row) {
                float acc = 0.f;
                for (int k = 0; k < r_n; ++k) acc = fmaf(load_elem(Bc + k), vs[row * a.r_max + k], acc);
                E *yp = y + (int64_t)rows_sm[row] * a.ld_y + a.sl.col_off[s] + c;
                store_elem(yp, load_elem(yp) + acc);
            }
        }
    }
}

template <typename E>
static cudaError_t launch_simt_t(int mode, const SimtArgs &a, int n_units, cudaStream_t st) {
    const size_t smem = simt_smem_bytes(a.sl.n, a.r_max);
    // the shared-memory limit is a per-device attribute of the kernel: set it once
    // per device and mode (devices 0-63)
    static std::mutex mu;
    static uint64_t attr_done[3] = {0, 0, 0};
    int dev = 0;
    cudaGetDevice(&dev);
    auto set = [&](const void *fn) {
        std::lock_guard<std::mutex> lock(mu);
        const uint64_t bit = 1ull << (dev & 63);
        if (!(attr_done[mode] & bit)) {
            cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)simt_smem_bytes(LORA_MAX_SLICES, LORA_MAX_RANK));
            attr_done[mode] |= bit;
        }
    };
    if (mode == 0) {
        set((const void *)simt_kernel<E, 0>);
        simt_kernel<E, 0><<<n_units, SIMT_THREADS, smem, st>>>(a);
    } else if (mode == 1) {
        set((const void *)simt_kernel<E, 1>);
        simt_kernel<E, 1><<<n_units, SIMT_THREADS, smem, st>>>(a);
    } else {
        set((const void *)simt_kernel<E, 2>);
        simt_kernel<E, 2><<<n_units, SIMT_THREADS, smem, st>>>(a);
    }
    return cudaGetLastError();
}

int launch_simt(int mode, bool bf16, const SimtArgs &a, int n_units, cudaStream_t st) {
    if (n_units <= 0) return LORA_OK;
    cudaError_t e = bf16 ? launch_simt_t<__nv_bfloat16>(mode, a, n_units, st)
                         : launch_simt_t<float>(mode, a, n_units, st);
    return cuda_rc(e);
}

}  // namespace lora
