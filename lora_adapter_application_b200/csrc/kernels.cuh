// Launch parameter blocks and host launchers of the library's kernels.
#pragma once

#include "common.cuh"

#include <cuda.h>

namespace lora {

enum { MODE_FUSED = 0, MODE_SHRINK = 1, MODE_EXPAND = 2 };

// Tensor maps of the fused kernel (bf16 2-D views of the stacked adapters),
// K = 16 ranks per box when r_max % 16 == 0, else 8:
//   A_s as [N*r_max rows][d_in], boxes of K rows x 64 columns, 128-byte swizzle
//   B_s as [N*d_out rows][r_max], boxes of 64 rows x K ranks
constexpr int BG_ABOX_COLS = 64;
constexpr int BG_BBOX_ROWS = 64;
// row_stride: elements between consecutive rows (0 = inner, densely packed)
int tensor_map_2d(CUtensorMap *out, const void *base, uint64_t inner, uint64_t outer,
                  uint32_t box_inner, uint32_t box_outer, bool swizzle128,
                  uint64_t row_stride = 0);

struct BgArgs {
    CUtensorMap tmA[LORA_MAX_SLICES];
    CUtensorMap tmB[LORA_MAX_SLICES];
    const __nv_bfloat16 *x;
    int64_t ld_x;
    int d_in;
    __nv_bfloat16 *y;
    int64_t ld_y;
    float *v;          // [S][T][r_max] fp32 (shrink / expand modes)
    int T;
    Slices sl;
    int r_max;
    const int32_t *ranks;
    const float *scales;
    Tiles tiles;
    int32_t *status;
    int ab16;          // adapters in 16-rank boxes (r_max % 16 == 0): A 64 x 16, B 16 x 64
    int stages;        // ring stages, 2 or 3, over the same ring bytes (set by launch_bgmv)
};

struct SimtArgs {
    const void *x;
    int64_t ld_x;
    int d_in;
    void *y;
    int64_t ld_y;
    float *v;
    int T;
    Slices sl;
    int r_max;
    const int32_t *ranks;
    const float *scales;
    Tiles tiles;
    int32_t *status;
};

// Tensor-core SGMV (contiguous tiles): maps over
//   x      [T][d_in] (row stride ld_x), boxes of 64 columns x lbr rows, 128-byte swizzle
//   A_s    [N*r_max][d_in], boxes of 64 columns x r_max rows, 128-byte swizzle
//   B_s    [N*d_out_s][r_max], boxes of 8 ranks x 128 rows, no swizzle
//   y_s    y + col_off_s as [T][d_out_s] (row stride ld_y), 128-byte swizzle: boxes of
//          64 columns x lbr rows (tmY, loads) and x sbr rows (tmYs, stores)
// (about 4.6 KB of kernel parameters: within the 32 KB CUDA 12.1+ allows)
struct TcArgs {
    CUtensorMap tmX;
    CUtensorMap tmA[LORA_MAX_SLICES];
    CUtensorMap tmB[LORA_MAX_SLICES];
    CUtensorMap tmY[LORA_MAX_SLICES];
    CUtensorMap tmYs[LORA_MAX_SLICES];
    int lbr;           // rows of an x / y load box (8 .. 128, power of two)
    int sbr;           // rows of a y store box (8 .. 128, power of two)
    __nv_bfloat16 *y;
    int64_t ld_y;
    float *v;          // [S][T][r_max] fp32 (shrink / expand modes)
    int T;
    int d_in;
    Slices sl;
    int r_max;
    const int32_t *ranks;
    const float *scales;
    const int4 *contig;
    const int32_t *counts;
    int max_contig;
    int stages;        // ring slots (set by the launcher)
    int C;             // blocks per cluster (set by the launcher)
    int32_t *status;
};

// lora_api.cu: LORA_OK, or LORA_ERR_CUDA after recording e for lora_last_error()
int cuda_rc(cudaError_t e);
// records a failure without a runtime error code (e.g. a driver call) and returns LORA_ERR_CUDA
int cuda_fail(const char *what);

// segments.cu
size_t segments_scratch_bytes(int T, int N);
int launch_build_segments(const int32_t *ids, const lora_meta *m, void *scratch,
                          size_t scratch_bytes, int32_t *status, cudaStream_t st);

// bgmv.cu: bf16, r_max <= 64, vector-aligned data; grid = cluster x n_units
size_t bgmv_smem_bytes(int n_slices);
int launch_bgmv(int mode, const BgArgs &a, int n_units, int cluster, cudaStream_t st);

// sgmv_tc.cu: bf16, r_max % 16 == 0, n_slices * r_max <= 128, 16-byte aligned rows;
// chooses the cluster size and ring depth, launches persistent clusters
size_t sgmv_tc_smem_bytes(int mode, int stages, int SR, int C);
// idle_sms (may be NULL): SMs the launch is expected to leave free (clusters
// beyond the estimated tile count)
int launch_sgmv_tc(int mode, TcArgs &a, cudaStream_t st, int *idle_sms = nullptr);

// simt.cu: any element type and alignment, r_max <= LORA_MAX_RANK
size_t simt_smem_bytes(int n_slices, int r_max);
int launch_simt(int mode, bool bf16, const SimtArgs &a, int n_units, cudaStream_t st);

}  // namespace lora
