// Launch parameter blocks and host launchers of the library's kernels.
#pragma once

#include "common.cuh"

namespace lora {

enum { MODE_FUSED = 0, MODE_SHRINK = 1, MODE_EXPAND = 2 };

struct BgArgs {
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
