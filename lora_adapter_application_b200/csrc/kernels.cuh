// Launch parameter blocks and host launchers of the library's kernels.
#pragma once

#include "common.cuh"

#include <cuda.h>

namespace lora {

enum { MODE_FUSED = 0, MODE_SHRINK = 1, MODE_EXPAND = 2 };

// Tensor maps of the fused kernel (bf16 2-D views of the stacked adapters):
//   A_s as [N*r_max rows][d_in], boxes of 8 rows x 64 columns, 128-byte swizzle
//   B_s as [N*d_out rows][r_max], boxes of 64 rows x 8 ranks
constexpr int BG_ABOX_COLS = 64, BG_ABOX_ROWS = 8;
constexpr int BG_BBOX_RANKS = 8, BG_BBOX_ROWS = 64;
int tensor_map_2d(CUtensorMap *out, const void *base, uint64_t inner, uint64_t outer,
                  uint32_t box_inner, uint32_t box_outer, bool swizzle128);

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

// segments.cu
size_t segments_scratch_bytes(int T, int N);
int launch_build_segments(const int32_t *ids, const lora_meta *m, void *scratch,
                          size_t scratch_bytes, int32_t *status, cudaStream_t st);

// bgmv.cu: bf16, r_max <= 64, vector-aligned data; grid = cluster x n_units
size_t bgmv_smem_bytes(int n_slices);
int launch_bgmv(int mode, const BgArgs &a, int n_units, int cluster, cudaStream_t st);

// simt.cu: any element type and alignment, r_max <= LORA_MAX_RANK
size_t simt_smem_bytes(int n_slices, int r_max);
int launch_simt(int mode, bool bf16, const SimtArgs &a, int n_units, cudaStream_t st);

}  // namespace lora
