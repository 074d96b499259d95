// C ABI of the multi-LoRA delta library: argument checks and the choice of
// kernel for each unit of work.  Declarations and contracts: lora_delta.h.
#include "kernels.cuh"
#include "ptx.cuh"

#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <mutex>

using namespace lora;

namespace {

thread_local char g_last_error[256] = "";

}  // namespace

namespace lora {

int cuda_rc(cudaError_t e) {
    if (e == cudaSuccess) return LORA_OK;
    snprintf(g_last_error, sizeof(g_last_error), "%s: %s", cudaGetErrorName(e), cudaGetErrorString(e));
    return LORA_ERR_CUDA;
}

int cuda_fail(const char *what) {
    snprintf(g_last_error, sizeof(g_last_error), "%s", what);
    return LORA_ERR_CUDA;
}

}  // namespace lora

namespace {

// A second stream for the gathered-tile launch of a call whose contiguous
// tiles take the tensor-core kernel: forked from and joined back to the
// caller's stream with events, so that its blocks fill the SMs the persistent
// tensor-core grid leaves free.  The two launches touch disjoint rows.  Each
// (device, caller stream) pair has a side stream and events of its own, so
// calls on different caller streams never meet on a shared stream - neither in
// eager use nor while one of them is being captured into a CUDA graph.
struct SideStream {
    int dev = -1;
    cudaStream_t caller = nullptr;
    cudaStream_t stream = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
};
constexpr int kSideStreams = 256;
std::mutex g_side_mu;
SideStream g_side[kSideStreams];
int g_side_used = 0;

// fn(side stream) between a fork from and a join into `caller`: work fn puts on
// `caller` after the fork and work it puts on the side stream may overlap.
// Past kSideStreams distinct caller streams, both launches go to `caller`.
template <class F>
int with_side_stream(cudaStream_t caller, F &&fn) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_rc(e);
    SideStream *ss = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_side_mu);
        for (int i = 0; i < g_side_used; ++i)
            if (g_side[i].dev == dev && g_side[i].caller == caller) {
                ss = &g_side[i];
                break;
            }
        if (!ss && g_side_used < kSideStreams) {
            SideStream n;
            n.dev = dev;
            n.caller = caller;
            if ((e = cudaStreamCreateWithFlags(&n.stream, cudaStreamNonBlocking)) != cudaSuccess ||
                (e = cudaEventCreateWithFlags(&n.fork, cudaEventDisableTiming)) != cudaSuccess ||
                (e = cudaEventCreateWithFlags(&n.join, cudaEventDisableTiming)) != cudaSuccess)
                return cuda_rc(e);
            g_side[g_side_used] = n;
            ss = &g_side[g_side_used++];
        }
    }
    if (!ss) return fn(caller);
    if ((e = cudaEventRecord(ss->fork, caller)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(ss->stream, ss->fork, 0)) != cudaSuccess)
        return cuda_rc(e);
    const int rc = fn(ss->stream);
    if ((e = cudaEventRecord(ss->join, ss->stream)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(caller, ss->join, 0)) != cudaSuccess)
        return cuda_rc(e);
    return rc;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int check_meta(const lora_meta *m) {
    if (!m) return LORA_ERR_NULL;
    if (m->T < 0 || m->T > LORA_MAX_ROWS || m->N < 1 || m->N > LORA_MAX_ADAPTERS)
        return LORA_ERR_SHAPE;
    if (m->rows_per_tile < 1 || m->rows_per_tile > LORA_MAX_TILE_ROWS || m->min_run < 0 || m->long_tile < 1 ||
        m->long_tile > LORA_LONG_TILE)
        return LORA_ERR_SHAPE;
    int32_t mg = 0, mc = 0;
    lora_meta_capacity(m->T, m->N, m->rows_per_tile, m->min_run, m->long_tile, &mg, &mc);
    if (m->max_gather_tiles < mg || m->max_contig_tiles < mc) return LORA_ERR_CAPACITY;
    if (!m->perm || !m->seg_start || !m->seg_adapter || !m->counts || !m->grow ||
        !m->gather_tiles || (mc > 0 && !m->contig_tiles))
        return LORA_ERR_NULL;
    return LORA_OK;
}

struct Call {
    void *y;
    int64_t ld_y;
    const void *x;
    int64_t ld_x;
    int32_t d_in;
    const lora_slice *slices;
    int32_t n_slices;
    int32_t r_max;
    const int32_t *ranks;
    const float *alphas;
    const float *v_in;
    float *v_out;
    const lora_meta *meta;
    void *ws;
    size_t ws_bytes;
    lora_dtype dtype;
    int32_t *status;
    cudaStream_t stream;
};

// need_x / need_y / need_alphas: which operands the mode reads
int check_call(const Call &c, bool need_x, bool need_y, bool need_alphas, bool need_v) {
    if (!c.slices || !c.ranks || !c.status) return LORA_ERR_NULL;
    if (need_x && !c.x) return LORA_ERR_NULL;
    if (need_y && !c.y) return LORA_ERR_NULL;
    if (need_alphas && !c.alphas) return LORA_ERR_NULL;
    if (need_v && !(c.v_in || c.v_out)) return LORA_ERR_NULL;
    if (c.dtype != LORA_BF16 && c.dtype != LORA_FP32) return LORA_ERR_DTYPE;
    int rc = check_meta(c.meta);
    if (rc != LORA_OK) return rc;
    if (c.n_slices < 1 || c.n_slices > LORA_MAX_SLICES) return LORA_ERR_SHAPE;
    if (c.r_max < 1 || c.r_max > LORA_MAX_RANK) return LORA_ERR_RANK;
    if (need_x && (c.d_in < 1 || c.ld_x < c.d_in)) return LORA_ERR_SHAPE;
    for (int s = 0; s < c.n_slices; ++s) {
        const lora_slice &sl = c.slices[s];
        if ((need_x && !sl.A) || (need_y && !sl.B)) return LORA_ERR_NULL;
        if (need_y && (sl.d_out < 1 || sl.col_off < 0 || (int64_t)sl.col_off + sl.d_out > c.ld_y))
            return LORA_ERR_SHAPE;
    }
    if (need_y) {   // each slice owns its columns of y: no two slices overlap
        int64_t total = 0;
        for (int s = 0; s < c.n_slices; ++s) {
            const lora_slice &a = c.slices[s];
            total += a.d_out;
            for (int t = 0; t < s; ++t) {
                const lora_slice &b = c.slices[t];
                if (a.col_off < (int64_t)b.col_off + b.d_out && b.col_off < (int64_t)a.col_off + a.d_out)
                    return LORA_ERR_SHAPE;
            }
        }
        if (total > (int64_t)1 << 30) return LORA_ERR_SHAPE;
    }
    return LORA_OK;
}

// Adapter rows of every slice addressable by 32-bit tensor coordinates
// (row n * d_out + column of the stacked B, n * r_max + rank of A).
bool rows_fit_int32(const Call &c) {
    const int64_t lim = ((int64_t)1 << 31) - 256;
    if ((int64_t)c.meta->N * c.r_max > lim) return false;
    for (int s = 0; s < c.n_slices; ++s)
        if ((int64_t)c.meta->N * c.slices[s].d_out > lim) return false;
    return true;
}

Slices make_slices(const Call &c) {
    Slices s{};
    s.n = c.n_slices;
    s.cat_off[0] = 0;
    for (int i = 0; i < c.n_slices; ++i) {
        s.A[i] = c.slices[i].A;
        s.B[i] = c.slices[i].B;
        s.d_out[i] = c.slices[i].d_out;
        s.col_off[i] = c.slices[i].col_off;
        s.cat_off[i + 1] = s.cat_off[i] + c.slices[i].d_out;
    }
    return s;
}

Tiles make_tiles(const lora_meta *m, bool gather, bool contig) {
    Tiles t{};
    t.counts = m->counts;
    t.grow = m->grow;
    t.gather = reinterpret_cast<const int4 *>(m->gather_tiles);
    t.contig = reinterpret_cast<const int4 *>(m->contig_tiles);
    t.max_gather = m->max_gather_tiles;
    t.max_contig = m->max_contig_tiles;
    t.rows_per_unit = m->rows_per_tile;
    t.subs = contig ? (m->long_tile + m->rows_per_tile - 1) / m->rows_per_tile : 0;
    t.use_gather = gather ? 1 : 0;
    return t;
}

int n_units(const Tiles &t) { return t.max_gather + (t.subs ? t.max_contig * t.subs : 0); }

// The fused BGMV kernel takes the call?  bf16, rank slots of at most 64 in
// multiples of 8, and 16-byte aligned rows, slices and v (it moves data with
// TMA copies).
bool bgmv_ok(int mode, const Call &c, bool need_x, bool need_y) {
    if (c.dtype != LORA_BF16 || c.r_max > 64 || (c.r_max & 7) || !rows_fit_int32(c)) return false;
    if ((int64_t)c.meta->T * c.n_slices * c.r_max > ((int64_t)1 << 31) - 1) return false;
    if (need_x) {
        if ((c.d_in & 7) || (c.ld_x & 7) || !aligned(c.x, 16)) return false;
        for (int s = 0; s < c.n_slices; ++s)
            if (!aligned(c.slices[s].A, 16)) return false;
    }
    if (need_y) {
        if ((c.ld_y & 7) || !aligned(c.y, 16)) return false;
        for (int s = 0; s < c.n_slices; ++s)
            if ((c.slices[s].d_out & 7) || (c.slices[s].col_off & 7) || !aligned(c.slices[s].B, 16))
                return false;
    }
    if (mode != MODE_FUSED && !aligned(mode == MODE_SHRINK ? (const void *)c.v_out : (const void *)c.v_in, 16))
        return false;
    return true;
}

// The tensor-core SGMV kernel takes the contiguous tiles?  bf16, ranks padded
// to a multiple of 16, all slices' ranks in one MMA (n_slices * r_max <= 128),
// 16-byte aligned rows and slices (TMA).
bool tc_ok(const Call &c, bool need_x, bool need_y) {
    if (c.dtype != LORA_BF16 || c.meta->min_run <= 0 || c.meta->max_contig_tiles <= 0) return false;
    if ((c.r_max & 15) || c.n_slices * c.r_max > 128 || !rows_fit_int32(c)) return false;
    if (need_x) {
        if ((c.d_in & 7) || (c.ld_x & 7) || !aligned(c.x, 16)) return false;
        for (int s = 0; s < c.n_slices; ++s)
            if (!aligned(c.slices[s].A, 16)) return false;
    }
    if (need_y) {
        if ((c.ld_y & 7) || !aligned(c.y, 16)) return false;
        for (int s = 0; s < c.n_slices; ++s)
            if ((c.slices[s].d_out & 7) || (c.slices[s].col_off & 7) || !aligned(c.slices[s].B, 16))
                return false;
    }
    return true;
}

// Contiguous tiles on the tensor-core SGMV kernel; false if a tensor map
// cannot be encoded (the caller then keeps those tiles on the other kernels).
bool run_tc(int mode, const Call &c, int *rc, int *idle_sms) {
    const bool need_x = mode != MODE_EXPAND, need_y = mode != MODE_SHRINK;
    const int N = c.meta->N;
    TcArgs a{};
    // rows of the x / y load boxes and of the y store boxes (tuning overrides:
    // LORA_TC_LOAD_ROWS, LORA_TC_STORE_ROWS; powers of two from 8 to 128)
    auto box_rows = [](const char *name, int dflt) {
        const char *e = std::getenv(name);
        const int v = e ? std::atoi(e) : 0;
        return (v >= 8 && v <= 128 && (v & (v - 1)) == 0) ? v : dflt;
    };
    a.lbr = box_rows("LORA_TC_LOAD_ROWS", 128);
    a.sbr = box_rows("LORA_TC_STORE_ROWS", 128);
    if (need_x &&
        tensor_map_2d(&a.tmX, c.x, (uint64_t)c.d_in, (uint64_t)c.meta->T, 64, (uint32_t)a.lbr, 128,
                      (uint64_t)c.ld_x) != LORA_OK)
        return false;
    for (int s = 0; s < c.n_slices; ++s) {
        const lora_slice &sl = c.slices[s];
        if (need_x && tensor_map_2d(&a.tmA[s], sl.A, (uint64_t)c.d_in, (uint64_t)N * c.r_max, 64,
                                    (uint32_t)c.r_max, 128) != LORA_OK)
            return false;
        const __nv_bfloat16 *ys = static_cast<const __nv_bfloat16 *>(c.y) + sl.col_off;
        if (need_y &&
            (tensor_map_2d(&a.tmB[s], sl.B, (uint64_t)c.r_max, (uint64_t)N * sl.d_out, 8, 128,
                           0) != LORA_OK ||
             tensor_map_2d(&a.tmY[s], ys, (uint64_t)sl.d_out, (uint64_t)c.meta->T, 64,
                           (uint32_t)a.lbr, 128, (uint64_t)c.ld_y) != LORA_OK ||
             tensor_map_2d(&a.tmYs[s], ys, (uint64_t)sl.d_out, (uint64_t)c.meta->T, 64,
                           (uint32_t)a.sbr, 128, (uint64_t)c.ld_y) != LORA_OK))
            return false;
    }
    a.y = static_cast<__nv_bfloat16 *>(c.y);
    a.ld_y = c.ld_y;
    a.v = mode == MODE_SHRINK ? c.v_out : const_cast<float *>(c.v_in);
    a.T = c.meta->T;
    a.d_in = c.d_in;
    a.sl = make_slices(c);
    a.r_max = c.r_max;
    a.ranks = c.ranks;
    a.alphas = c.alphas;
    a.contig = reinterpret_cast<const int4 *>(c.meta->contig_tiles);
    a.counts = c.meta->counts;
    a.max_contig = c.meta->max_contig_tiles;
    a.status = c.status;
    *rc = launch_sgmv_tc(mode, a, c.stream, idle_sms);
    return *rc != LORA_ERR_SHAPE;
}

int env_int(const char *name, int dflt) {
    const char *e = std::getenv(name);
    return e ? std::atoi(e) : dflt;
}

int device_sms() {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

// Grid of the gathered-tile kernel: one block per SM.  Tuning / test override:
// LORA_BG_BLOCKS = 1 .. 4096 blocks (the kernel makes progress with any number
// resident).
int bgmv_blocks() {
    const int e = env_int("LORA_BG_BLOCKS", 0);
    return e >= 1 && e <= 4096 ? e : 0;
}

// Output columns of one expand item (one warp's): the narrowest of 128 .. 2048
// that keeps the batch's expected items at most five per warp of the grid (more
// items balance better, each item pays one pipeline fill), and at least 256 when
// the batch has fewer than 64 units (a small batch is bound by one item's
// latency).  Measured on the Llama-3-8B decode layer set (16-row tiles: best
// 256 / 128 / 768-1024 / 128 for qkv / o / gate-up / down) and decode q_proj
// (256).  Tuning override: LORA_BG_ITEM_COLS, a multiple of 32 from 32 to 8192.
int bgmv_item_cols(const Call &c, int est_units) {
    const int e = env_int("LORA_BG_ITEM_COLS", 0);
    if (e >= 32 && e <= 8192 && (e & 31) == 0) return e;
    const int64_t cap = 5LL * 8 * device_sms();
    const int lo = est_units < 64 ? 256 : 128;
    static const int cand[] = {128, 256, 384, 512, 768, 1024, 1536, 2048};
    for (int bc : cand) {
        if (bc < lo) continue;
        int64_t items = 0;
        for (int s = 0; s < c.n_slices; ++s) items += (c.slices[s].d_out + bc - 1) / bc;
        if (items * est_units <= cap) return bc;
    }
    return 2048;
}

// The tensor-core gathered-tile kernel takes a fused call whose units have at
// most 16 rows (the MMA's N) when LORA_BG_TC=1.  It is opt-in: on the Llama-3-8B
// decode layer set it is correct but slower than the mma.sync kernel (one
// producer warp per block issues every copy and bounds the block).
bool bgmv_tc_ok(const Call &c) {
    return c.meta->rows_per_tile <= 16 && env_int("LORA_BG_TC", 0) == 1;
}

// Output columns of one tensor-core expand item: the widest the kernel's ring
// holds (up to four 128-column tiles behind one v pair); tuning override
// LORA_BT_COLS, a multiple of 128 up to that width.
int bgmv_tc_item_cols() {
    const int cap = bgmv_tc_max_item_cols();
    const int e = env_int("LORA_BT_COLS", 0);
    return e >= 128 && e <= cap && (e & 127) == 0 ? e : cap;
}

// Tensor maps of the tensor-core gathered-tile kernel; false when one cannot be encoded.
bool bgmv_tc_maps(const Call &c, BtArgs &b) {
    const int64_t N = c.meta->N;
    for (int s = 0; s < c.n_slices; ++s) {
        const lora_slice &sl = c.slices[s];
        const __nv_bfloat16 *ys = static_cast<const __nv_bfloat16 *>(c.y) + sl.col_off;
        for (int g = 1; b.ks == 4 && g <= c.r_max / 8; ++g)
            if (tensor_map_chunks(&b.tmA4[g - 1][s], sl.A, (uint64_t)c.d_in, (uint64_t)N * c.r_max,
                                  (uint64_t)c.d_in, (uint32_t)(8 * g), 4) != LORA_OK)
                return false;
        if (tensor_map_2d(&b.tmA[s], sl.A, (uint64_t)c.d_in, (uint64_t)N * c.r_max, 64, 8, 128) != LORA_OK ||
            tensor_map_2d(&b.tmB[s], sl.B, (uint64_t)c.r_max, (uint64_t)N * sl.d_out, 8, 128, 0) != LORA_OK ||
            tensor_map_2d(&b.tmY[s], ys, (uint64_t)sl.d_out, (uint64_t)c.meta->T, 128, 1, 0,
                          (uint64_t)c.ld_y) != LORA_OK)
            return false;
    }
    return true;
}

// Pieces a fused call's shrink items are split into along d_in: two when the
// batch is so small that twice its expected shrink items still fit one block per
// SM (decode batches: the items then run on idle SMs, halving the item every
// expand waits for), else one.  Tuning / test override: LORA_BG_KSPLIT = 1 or 2.
int bgmv_ksplit(const Call &c, int est_units) {
    const int e = env_int("LORA_BG_KSPLIT", 0);
    if (e == 1 || e == 2) return e;
    const int gm = c.meta->rows_per_tile <= 16 ? 1 : (c.r_max + 31) / 32;
    const int64_t items = (int64_t)est_units * c.n_slices * gm;
    return (c.d_in >= 1024 && 2 * items <= device_sms()) ? 2 : 1;
}

// The gathered tiles (and the contiguous ones unless tc_took) on a gathered-tile
// kernel, or the general kernel when the data does not suit them, on `stream`.
int launch_rest(int mode, const Call &c, bool gather, bool contig, bool tc_took, cudaStream_t stream) {
    const bool need_x = mode != MODE_EXPAND, need_y = mode != MODE_SHRINK;
    Tiles tiles = make_tiles(c.meta, gather, contig);
    const int units = n_units(tiles);
    if (c.meta->T == 0 || units == 0) return LORA_OK;
    (void)tc_took;
    if (bgmv_ok(mode, c, need_x, need_y)) {
        GbArgs g{};
        g.x = static_cast<const __nv_bfloat16 *>(c.x);
        g.ld_x = c.ld_x;
        g.d_in = c.d_in;
        g.y = static_cast<__nv_bfloat16 *>(c.y);
        g.ld_y = c.ld_y;
        g.T = c.meta->T;
        g.sl = make_slices(c);
        g.r_max = c.r_max;
        g.ranks = c.ranks;
        g.alphas = c.alphas;
        g.tiles = tiles;
        g.status = c.status;
        if (mode == MODE_FUSED) {   // control words, per-unit counters, v: the workspace
            unsigned char *ws = static_cast<unsigned char *>(c.ws);
            g.ctl = reinterpret_cast<int *>(ws);
            g.done = g.ctl + 64;
            g.v = reinterpret_cast<float *>(ws + bgmv_workspace_head(units));
        } else {
            g.v = mode == MODE_SHRINK ? c.v_out : const_cast<float *>(c.v_in);
        }
        const int est = std::min(units, std::min(c.meta->N, c.meta->T) +
                                            (c.meta->T + c.meta->rows_per_tile - 1) / c.meta->rows_per_tile);
        auto set_cols = [&](int bc) {
            g.bc = bc;
            g.blk_off[0] = 0;
            for (int s = 0; s < c.n_slices; ++s)
                g.blk_off[s + 1] = g.blk_off[s] + (c.slices[s].d_out + g.bc - 1) / g.bc;
        };
        g.wait_limit = WAIT_LIMIT;
        if (env_int("LORA_DEBUG_STALL", 0) == 1) {
            // test hook for the bounded wait: expand items wait for a shrink signal
            // that never comes, with a short limit
            g.dbg_stall = 1;
            g.wait_limit = 64;
        }
        if (mode == MODE_FUSED && bgmv_tc_ok(c)) {
            static BtArgs bt;   // ~3.5 KB: kept off the stack; filled and launched under the lock
            static std::mutex bt_mu;
            std::lock_guard<std::mutex> lock(bt_mu);
            bt = BtArgs{};
            bt.ks = c.d_in % 64 == 0 ? 4 : 1;   // 256-column shrink stages when the chunks are whole
            if (bgmv_tc_maps(c, bt)) {
                set_cols(bgmv_tc_item_cols());
                bt.g = g;
                bt.vws = reinterpret_cast<unsigned char *>(g.v);
                return launch_bgmv_tc(bt, bgmv_blocks(), stream);
            }
            // a map could not be encoded: the mma.sync kernel takes the call
        }
        set_cols(bgmv_item_cols(c, std::max(1, est)));
        g.ks = 1;
        if (mode == MODE_FUSED) {
            g.ks = bgmv_ksplit(c, std::max(1, est));
            g.vpiece = (int64_t)c.n_slices * c.meta->T * c.r_max;
        }
        return launch_bgmv(mode, g, bgmv_blocks(), stream);
    }
    SimtArgs a{};
    a.x = c.x;
    a.ld_x = c.ld_x;
    a.d_in = c.d_in;
    a.y = c.y;
    a.ld_y = c.ld_y;
    a.v = mode == MODE_SHRINK ? c.v_out : const_cast<float *>(c.v_in);
    a.T = c.meta->T;
    a.sl = make_slices(c);
    a.r_max = c.r_max;
    a.ranks = c.ranks;
    a.alphas = c.alphas;
    a.tiles = tiles;
    a.status = c.status;
    return launch_simt(mode, c.dtype == LORA_BF16, a, units, stream);
}

// A fused call's contiguous tiles take the tensor-core SGMV kernel unless the
// batch is too small to give every SM a 128-row tile while the layer is wide: a
// cluster expands its tile over every output column as one long piece, and one
// wave of such tiles leaves SMs idle, where the gathered-tile kernel spreads the
// same columns over every warp as items and takes all rows in one launch.
// Measured on B200, the mixed 70B batch (8192 rows, 7892 of them in prompts),
// 16-row tiles and 64-row runs: 8192 -> 28672 layer 227 -> 211 us, 28672 -> 8192
// layer 151 -> 152 us (one launch each); built for the single launch (32-row
// tiles, no runs) 201 and 146 us.  Prefill batches of 11-77k tokens at 4096 wide
// keep the tensor-core kernel (71 against 82 us at 11k tokens).  Override:
// LORA_TC_ROUTE = 1 (the tensor-core kernel whenever it qualifies) or 2 (the
// gathered-tile kernel for every row).
constexpr int64_t TC_WIDE_COLS = 8192;
// Rows per gathered tile when every row of every layer takes the fused kernel:
// a tile reads its adapter once for twice the rows of a 16-row tile, and a batch
// of thousands of rows still has tiles for every SM (the mixed 70B pair: 347 us
// with 32-row tiles, 355 with 16, 351 with 64, all without contiguous runs).
constexpr int32_t WIDE_ROWS_PER_TILE = 32;

// -1: no override; 0: the tensor-core kernel whenever it qualifies; 1: every row
// of every fused call on the gathered-tile kernel.
int route_override() {
    const int e = env_int("LORA_TC_ROUTE", 0);
    return e == 1 ? 0 : e == 2 ? 1 : -1;
}

// The rule itself: a fused call over T rows and `cols` output columns sends every
// row to the gathered-tile kernel.
bool wide_and_few_tiles(int64_t T, int64_t long_tile, int64_t cols, int sms) {
    return (T + long_tile - 1) / long_tile < sms && cols >= TC_WIDE_COLS;
}

bool tc_pays(int mode, const Call &c) {
    const int e = route_override();
    if (e >= 0) return e == 0;
    if (mode != MODE_FUSED) return true;
    int64_t cols = 0;
    for (int s = 0; s < c.n_slices; ++s) cols += c.slices[s].d_out;
    return !wide_and_few_tiles(c.meta->T, c.meta->long_tile, cols, device_sms());
}

int run(int mode, const Call &c, bool gather, bool contig, bool tensor_core = true) {
    const bool need_x = mode != MODE_EXPAND, need_y = mode != MODE_SHRINK;
    if (tensor_core && contig && c.meta->T > 0 && tc_ok(c, need_x, need_y) && tc_pays(mode, c)) {
        // contiguous tiles on the tensor-core kernel (caller's stream), gathered tiles on
        // the side stream: the fork comes first, so the two launches overlap
        return with_side_stream(c.stream, [&](cudaStream_t side) -> int {
            int rc = LORA_OK, idle_sms = 0;
            if (!run_tc(mode, c, &rc, &idle_sms))   // a tensor map could not be encoded
                return launch_rest(mode, c, gather, true, false, c.stream);
            if (rc != LORA_OK) return rc;
            return launch_rest(mode, c, gather, false, true, side);
        });
    }
    return launch_rest(mode, c, gather, contig, false, c.stream);
}

// Workspace a fused call needs for this batch metadata and layer shape.
size_t linear_ws_bytes(const lora_meta *m, int n_slices, int r_max) {
    const Tiles t = make_tiles(m, true, m->min_run > 0);
    return bgmv_workspace_bytes(n_units(t), m->T, n_slices, r_max);
}

// The fused entry points' workspace: present, large enough, 256-byte aligned.
int check_ws(const Call &c) {
    if (!c.ws) return LORA_ERR_NULL;
    if (!aligned(c.ws, 256) || c.ws_bytes < linear_ws_bytes(c.meta, c.n_slices, c.r_max))
        return LORA_ERR_WORKSPACE;
    return LORA_OK;
}

}  // namespace

namespace lora {
int check_meta_args(const lora_meta *m) { return check_meta(m); }
}  // namespace lora

extern "C" {

int lora_version(void) { return 20100; }

const char *lora_last_error(void) { return g_last_error; }

const char *lora_status_string(int status) {
    switch (status) {
        case LORA_OK: return "LORA_OK";
        case LORA_ERR_NULL: return "LORA_ERR_NULL";
        case LORA_ERR_DTYPE: return "LORA_ERR_DTYPE";
        case LORA_ERR_SHAPE: return "LORA_ERR_SHAPE";
        case LORA_ERR_RANK: return "LORA_ERR_RANK";
        case LORA_ERR_ALIGN: return "LORA_ERR_ALIGN";
        case LORA_ERR_WORKSPACE: return "LORA_ERR_WORKSPACE";
        case LORA_ERR_CAPACITY: return "LORA_ERR_CAPACITY";
        case LORA_ERR_CUDA: return "LORA_ERR_CUDA";
        default: return "unknown lora_status";
    }
}

int lora_meta_capacity(int32_t T, int32_t N, int32_t rows_per_tile, int32_t min_run,
                       int32_t long_tile, int32_t *max_gather, int32_t *max_contig) {
    if (!max_gather || !max_contig) return LORA_ERR_NULL;
    if (T < 0 || T > LORA_MAX_ROWS || N < 1 || N > LORA_MAX_ADAPTERS || rows_per_tile < 1 ||
        rows_per_tile > LORA_MAX_TILE_ROWS || min_run < 0 || long_tile < 1 || long_tile > LORA_LONG_TILE)
        return LORA_ERR_SHAPE;
    *max_gather = (T + rows_per_tile - 1) / rows_per_tile + (N < T ? N : T);
    *max_contig = min_run > 0 ? (T + long_tile - 1) / long_tile + T / min_run : 0;
    return LORA_OK;
}

int lora_segment_plan(int32_t T, const int64_t *layer_cols, int32_t n_layers, int32_t sms,
                      int32_t long_tile, int32_t *rows_per_tile, int32_t *min_run,
                      uint8_t *all_gathered) {
    if (!rows_per_tile || !min_run || (n_layers > 0 && !layer_cols)) return LORA_ERR_NULL;
    if (T < 0 || T > LORA_MAX_ROWS || n_layers < 0 || n_layers > LORA_MAX_ADAPTERS || sms < 0 ||
        long_tile < 1 || long_tile > LORA_LONG_TILE || *rows_per_tile < 1 ||
        *rows_per_tile > LORA_MAX_TILE_ROWS || *min_run < 0)
        return LORA_ERR_SHAPE;
    for (int l = 0; l < n_layers; ++l)
        if (layer_cols[l] < 1) return LORA_ERR_SHAPE;
    const int n_sms = sms > 0 ? sms : device_sms();
    const int e = route_override();
    bool every = n_layers > 0;
    for (int l = 0; l < n_layers; ++l) {
        const bool g = e >= 0 ? e == 1 : wide_and_few_tiles(T, long_tile, layer_cols[l], n_sms);
        if (all_gathered) all_gathered[l] = g ? 1 : 0;
        every = every && g;
    }
    if (every && *min_run > 0) {
        *rows_per_tile = WIDE_ROWS_PER_TILE;
        *min_run = 0;
    }
    return LORA_OK;
}

size_t lora_segments_scratch_bytes(int32_t T, int32_t N) {
    if (T < 0 || T > LORA_MAX_ROWS || N < 1 || N > LORA_MAX_ADAPTERS) return 0;
    return segments_scratch_bytes(T, N);
}

int lora_build_segments(const int32_t *ids, const lora_meta *meta, void *scratch,
                        size_t scratch_bytes, int32_t *status, void *stream) {
    int rc = check_meta(meta);
    if (rc != LORA_OK) return rc;
    if (!status || (meta->T > 0 && !ids)) return LORA_ERR_NULL;
    return launch_build_segments(ids, meta, scratch, scratch_bytes, status,
                                 static_cast<cudaStream_t>(stream));
}

size_t lora_shrink_workspace_bytes(int32_t T, int32_t r_max, int32_t n_slices) {
    if (T < 0 || r_max < 1 || n_slices < 1) return 0;
    return (size_t)n_slices * (size_t)T * (size_t)r_max * sizeof(float);
}

size_t lora_linear_workspace_bytes(const lora_meta *meta, int32_t n_slices, int32_t r_max) {
    if (check_meta(meta) != LORA_OK || n_slices < 1 || n_slices > LORA_MAX_SLICES || r_max < 1 ||
        r_max > LORA_MAX_RANK)
        return 0;
    return linear_ws_bytes(meta, n_slices, r_max);
}

int lora_sgmv_shrink(float *v, const void *x, int64_t ld_x, int32_t d_in,
                     const lora_slice *slices, int32_t n_slices, int32_t r_max,
                     const int32_t *ranks, const lora_meta *meta, lora_dtype dtype,
                     int32_t *status, void *stream) {
    Call c{nullptr, 0, x, ld_x, d_in, slices, n_slices, r_max, ranks, nullptr, nullptr, v,
           meta, nullptr, 0, dtype, status, static_cast<cudaStream_t>(stream)};
    int rc = check_call(c, true, false, false, true);
    if (rc != LORA_OK) return rc;
    return run(MODE_SHRINK, c, true, true);
}

int lora_sgmv_expand(void *y, int64_t ld_y, const float *v, const lora_slice *slices,
                     int32_t n_slices, int32_t r_max, const int32_t *ranks,
                     const float *alphas, const lora_meta *meta, lora_dtype dtype,
                     int32_t *status, void *stream) {
    Call c{y, ld_y, nullptr, 0, 0, slices, n_slices, r_max, ranks, alphas, v, nullptr,
           meta, nullptr, 0, dtype, status, static_cast<cudaStream_t>(stream)};
    int rc = check_call(c, false, true, true, true);
    if (rc != LORA_OK) return rc;
    return run(MODE_EXPAND, c, true, true);
}

int lora_bgmv_fused(void *y, int64_t ld_y, const void *x, int64_t ld_x, int32_t d_in,
                    const lora_slice *slices, int32_t n_slices, int32_t r_max,
                    const int32_t *ranks, const float *alphas, const lora_meta *meta,
                    void *workspace, size_t workspace_bytes, lora_dtype dtype, int32_t *status,
                    void *stream) {
    Call c{y, ld_y, x, ld_x, d_in, slices, n_slices, r_max, ranks, alphas, nullptr, nullptr,
           meta, workspace, workspace_bytes, dtype, status, static_cast<cudaStream_t>(stream)};
    int rc = check_call(c, true, true, true, false);
    if (rc == LORA_OK) rc = check_ws(c);
    if (rc != LORA_OK) return rc;
    return run(MODE_FUSED, c, true, true, false);
}

int lora_add_linear(void *y, int64_t ld_y, const void *x, int64_t ld_x, int32_t d_in,
                    const lora_slice *slices, int32_t n_slices, int32_t r_max,
                    const int32_t *ranks, const float *alphas, const lora_meta *meta,
                    void *workspace, size_t workspace_bytes, lora_dtype dtype, int32_t *status,
                    void *stream) {
    Call c{y, ld_y, x, ld_x, d_in, slices, n_slices, r_max, ranks, alphas, nullptr, nullptr,
           meta, workspace, workspace_bytes, dtype, status, static_cast<cudaStream_t>(stream)};
    int rc = check_call(c, true, true, true, false);
    if (rc == LORA_OK) rc = check_ws(c);
    if (rc != LORA_OK) return rc;
    return run(MODE_FUSED, c, true, true);
}

}  // extern "C"
