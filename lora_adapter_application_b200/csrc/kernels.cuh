// Launch parameter blocks and host launchers of the library's kernels.
#pragma once

#include "common.cuh"

#include <cuda.h>

namespace lora {

enum { MODE_FUSED = 0, MODE_SHRINK = 1, MODE_EXPAND = 2 };

// row_stride: elements between consecutive rows (0 = inner, densely packed);
// swizzle: 0 (none), 32, 64 or 128 bytes
int tensor_map_2d(CUtensorMap *out, const void *base, uint64_t inner, uint64_t outer,
                  uint32_t box_inner, uint32_t box_outer, int swizzle,
                  uint64_t row_stride = 0);
// [rows][inner] viewed as [inner / 64][rows][64] (inner a multiple of 64): boxes of
// 64 columns x box_rows x box_chunks chunks, 128-byte swizzle
int tensor_map_chunks(CUtensorMap *out, const void *base, uint64_t inner, uint64_t rows,
                      uint64_t row_stride, uint32_t box_rows, uint32_t box_chunks);

// Pieces a shrink item may be split into along d_in (fused mode, small batches).
constexpr int BG_KSPLIT_MAX = 2;

// Fused-mode workspace head shared by the gathered-tile kernels: GB_CTL_INTS
// control words (tickets and the exit counter), then one done word per unit.
constexpr int GB_CTL_INTS = 64;
enum { GB_T_SHRINK = 0, GB_T_EXPAND = 1, GB_T_EXIT = 2 };

// The gathered-tile kernel (bgmv.cu): plain pointers, no tensor maps.
struct GbArgs {
    const __nv_bfloat16 *x;
    int64_t ld_x;
    int d_in;
    __nv_bfloat16 *y;
    int64_t ld_y;
    float *v;          // [S][T][r_max] fp32: the caller's (shrink / expand modes) or the workspace's
    int T;
    Slices sl;
    int r_max;
    const int32_t *ranks;
    const float *alphas;
    Tiles tiles;
    int32_t *status;
    int *ctl;          // fused mode: tickets and exit counter (workspace head)
    int *done;         // fused mode: per unit, shrink items finished
    int bc;            // output columns of one expand item (multiple of 32)
    int blk_off[LORA_MAX_SLICES + 1];   // expand items per unit: slice s owns [blk_off[s], blk_off[s+1])
    unsigned wait_limit;   // tries of the bounded wait (WAIT_LIMIT; shorter for the stall test hook)
    int ks;            // fused mode: pieces a shrink item's d_in is split into (1 or 2); piece p writes
                       // its partial v at v + p * vpiece, and the expand adds the pieces in order
    int64_t vpiece;    // floats between the pieces' v (S * T * r_max)
    int dbg_stall;     // test hook: expand items wait for one shrink signal more than exists
};

// The gathered-tile kernel on the tensor cores (bgmv_tc.cu, fused mode only):
// GbArgs (bc a multiple of 128) plus maps over
//   A_s  [N*r_max][d_in], boxes of 64 columns x 8 ranks, 128-byte swizzle (and the
//        chunked view above, one box per 256-column shrink stage)
//   B_s  [N*d_out_s][r_max], boxes of 8 ranks x 128 columns, no swizzle
//   y_s  y + col_off_s as [T][d_out_s] (row stride ld_y), boxes of 128 columns x 1 row
// and the workspace's v pairs (s_n v as bf16 hi + lo per unit and slice).
struct BtArgs {
    CUtensorMap tmA[LORA_MAX_SLICES];
    // A_s as [d_in/64][N*r_max][64] (d_in % 64 == 0): tmA4[g - 1][s] boxes 8g ranks x 4 chunks
    CUtensorMap tmA4[8][LORA_MAX_SLICES];
    int ks;                              // 64-column chunks per shrink stage: 4 with tmA4, else 1
    CUtensorMap tmB[LORA_MAX_SLICES];
    CUtensorMap tmY[LORA_MAX_SLICES];
    GbArgs g;
    unsigned char *vws;
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
    const float *alphas;
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
    const float *alphas;
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

// lora_api.cu: the lora_meta checks every entry point makes (LORA_OK or an error)
int check_meta_args(const lora_meta *m);

// segments.cu
size_t segments_scratch_bytes(int T, int N);
int launch_build_segments(const int32_t *ids, const lora_meta *m, void *scratch,
                          size_t scratch_bytes, int32_t *status, cudaStream_t st);

// bgmv.cu: bf16, r_max <= 64 and a multiple of 8, 16-byte aligned rows; units
// of up to LORA_MAX_TILE_ROWS rows; a persistent grid of one block per SM
// (`blocks` blocks when positive)
size_t bgmv_smem_bytes(int mode);
int launch_bgmv(int mode, const GbArgs &a, int blocks, cudaStream_t st);
// workspace of the fused mode: control words, then one int per unit (the head),
// then v: fp32 [BG_KSPLIT_MAX][S][T][r_max] for this kernel or the v pairs of
// bgmv_tc.cu, whichever is larger
size_t bgmv_workspace_head(int units);
size_t bgmv_workspace_bytes(int units, int T, int n_slices, int r_max);

// bgmv_tc.cu: bf16, r_max <= 64 and a multiple of 8, units of at most 16 rows,
// the 16-byte alignments of bgmv.cu; a persistent grid of two blocks per SM
size_t bgmv_tc_smem_bytes();
// widest expand item the kernel's operand ring holds (columns, a multiple of 128)
int bgmv_tc_max_item_cols();
// v pairs of the fused workspace (after the head)
size_t bgmv_tc_v_bytes(int units, int n_slices, int r_max);
int launch_bgmv_tc(const BtArgs &a, int blocks, cudaStream_t st);

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
