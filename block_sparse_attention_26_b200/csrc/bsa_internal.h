// bsa_internal.h -- declarations shared by the host API and the kernel files.
#pragma once

#include <cuda_runtime.h>

#include <algorithm>
#include <stddef.h>
#include <stdint.h>

#include "bsa.h"

namespace bsa {

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Streaming multiprocessors of the current device (looked up once per device;
// 148 on a B200).  Grids that should cover the whole GPU are sized from it.
int sm_count();
// CTAs of the extra-token fallback pass (one scratch row of N keys each).
inline int fallback_ctas() { return sm_count(); }

// entries per fine-pass tile of the extra-token union: two lists of at most 256,
// padded to a multiple of 4
constexpr int kGlistCap = 2 * 256 + 4;
inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Certified Sol routing: uncertain blocks listed per row before the exact pass.
constexpr int kUcap = 128;

// Per-row data of the certified routing (32 bytes): the decide kernel keeps
// block b iff raw > hi + c |kbar_b| and drops it iff raw < lo - c |kbar_b|
// (raw = the tensor-core dot product); the definition's threshold lies in
// [thr_lo, thr_hi]; mode 1 sends the row to the exact path.
struct RowInfo {
    float hi, lo, c, thr_lo, thr_hi;
    int32_t mode, pad0, pad1;
};

// Derived sizes of one problem.
struct Dims {
    int B, H, N, d;
    int Bq, Bk;
    int nQB, nKB, nW;      // nW = 32-bit words of a per-row key-block bitmask
    int64_t rows;          // B * H * nQB
    int E;
    bool cube;             // cube tiling (BSA_VSA): blocks past the prefix are cubes of the grid
    int pre_blocks;        // 64-token blocks of the prefix that precede the cubes
};

Dims dims_of(const bsa_params &p);

// Byte offsets of the workspace regions (each 256-byte aligned).  The status
// word comes first; the selection's scratch and the attention calls' scratch
// both start after it and share the same bytes (neither reads the other's).
struct WsLayout {
    size_t status;         // DevStatus
    size_t scores;         // [rows, nKB] f32 block scores (select)
    size_t bitmask;        // [rows, nW] u32 kept-block bitmask (select)
    size_t counts;         // [rows] i32 kept counts (select)
    size_t scan_tmp;       // [ceil(rows / 4096)] i64 per-tile sums of the counts' scan
    size_t kc16, vc16;     // [B*H, nKB, d] bf16 centroids (attention)
    // modified centroids (extra tokens): row r's entries are idx = xoff[r] ..
    // xoff[r] + xcnt[r] - 1; the centroids are stored grouped by source block, entry
    // idx at slot[idx]
    int64_t mc_cap;        // capacity, in entries (rows x the per-row average asked for)
    size_t xk16, xv16;     // [mc_cap, d] bf16 modified centroids, by slot
    size_t xbias;          // [mc_cap] f32 their log2 token counts, by idx
    size_t xcnt;           // [rows] i32 modified centroids per row (cut to what fits)
    size_t xoff;           // [rows + 1] i64 exclusive scan of the uncut counts
    size_t mc_slot;        // [mc_cap] i32 slot of each idx
    size_t mc_ent;         // [mc_cap] u64 left-out tokens of each slot
    size_t mc_cnt3;        // [B*H, nKB, groups] i32 entries per (source block, query-block group)
    size_t mc_off3;        // [B*H*nKB*groups + 1] i64 its exclusive scan
    size_t mc_tile;        // scan tile sums for the two scans
    size_t glist;          // [sparse tiles, kGlistCap] u32 extra-token union per fine-pass tile
    size_t glcnt;          // [sparse tiles] i32 its length
    size_t q16, k16, v16;  // [B, N, H, d] bf16 copies of f32 inputs (attention, f32 only)
    size_t ex_theta;       // [rows] f32 extra-token score bounds
    size_t ex_smax;        // [rows] f32 largest sampled token score
    size_t ex_cut;         // [rows] f32x4 bucket map and final cut of the kept tokens
    size_t ex_buf;         // [rows, 1024] u64 surviving (score, token) pairs
    size_t ex_cnt;         // [rows] i32 survivors per row
    size_t ex_ovf;         // [1 + rows] i32 overflowed rows
    size_t ex_scratch;     // [fallback_ctas(), N] u32 fallback keys
    // certified Sol routing (finite tau)
    size_t r_k16;          // [B*H, nKB, d] bf16 key centroids (the score GEMM's B operand)
    size_t r_knorm;        // [B*H, nKBp] f32 their norms, rounded up
    size_t r_knmax;        // [B*H, nKBp / 32] f32 largest norm per 32-block word
    size_t r_gram;         // [B*H, nsplit, d, d] f64 partial Gram matrices
    size_t r_ksum;         // [B*H, nsplit, d] f64 partial sums
    size_t r_cov;          // [B*H, d, d] f64 centred second moments
    size_t r_hstat;        // [B*H, d + 3] f64 mean key, tr(G)/n, |m|^2, max |kbar|
    size_t r_info;         // [rows] RowInfo
    size_t r_fbl;          // [1 + rows] i32 rows for the exact path
    size_t r_fbs;          // [fallback_ctas(), nKBp] f32 exact scores of one row
    int r_nsplit;
    size_t q8, k8;         // [B, N, H, d] e4m3 copies of Q and K (qk_fp8)
    size_t sq8;            // [B*H, ceil(N / 64)] f32 scales of Q per 64 tokens
    size_t sk8;            // [B*H, nKB] f32 scales of K per key block
    size_t kc8;            // [B*H, nKB, d] e4m3 centroids
    size_t skc8;           // [B*H, ceil(nKB / 64)] f32 scales of the centroids per 64
    size_t v8, vc8;        // [B, N, H, d] e4m3 V, [B*H, nKB, d] e4m3 value centroids (pv_fp8)
    size_t sv8;            // [B*H, d] f32 scale of V per channel (its largest |v| / 448)
    size_t part_o;         // [part_tiles, 128, d] f32 dense-row partial outputs
    size_t part_ml;        // [part_tiles, 128, 2] f32 dense-row partial (max, sum)
    int64_t part_tiles;    // capacity of the partial buffers, in 128-row tiles
    size_t total;
};

WsLayout ws_layout(const bsa_params &p);

// Consecutive 256-byte-aligned regions.
struct Taker {
    size_t off = 0;
    size_t take(size_t bytes)
    {
        const size_t at = off;
        off = align_up(off + bytes, 256);
        return at;
    }
};

// Whether Sol selection takes the certified route (a finite tau); key blocks
// per head padded to a multiple of 128; split count of the key Gram matrix.
bool certified_route(const bsa_params &p);
inline int64_t route_nkbp(const Dims &D) { return ceil_div(D.nKB, 128) * 128; }
int route_nsplit(const Dims &D);
// The selection's scratch regions (status, scores, bitmask, counts and the
// certified route's), taken from T in that order.
void select_regions(const bsa_params &p, const Dims &D, WsLayout &L, Taker &T);
// Certified Sol routing: bitmask (forced blocks included) and kept counts.
cudaError_t launch_route(const bsa_params &p, const Dims &D, const float *qbar, const float *kbar, char *ws,
                         const WsLayout &L, cudaStream_t st);

// Key-chunk split of `nrows` dense rows (1 = no split), limited to max_partials tiles.
int dense_split_for(const Dims &D, int nrows, int64_t max_partials);
// Partial tiles the dense rows of a parameter set need (0 if they are not split).
int64_t dense_partial_tiles(const Dims &D, int nrows);

cudaError_t launch_pool(const bsa_params &p, const Dims &D, const void *q, const void *k,
                        const void *v, float *qbar, float *kbar, float *vbar, int32_t *blk_count,
                        cudaStream_t st);

cudaError_t launch_select(const bsa_params &p, const Dims &D, const float *qbar, const float *kbar,
                          int64_t *row_ptr, int32_t *col_idx, int64_t col_capacity,
                          int32_t *kept_count, char *ws, const WsLayout &L, cudaStream_t st);

cudaError_t launch_attention(const bsa_params &p, const Dims &D, const void *q, const void *k,
                             const void *v, const float *kbar, const float *vbar,
                             const int64_t *row_ptr, const int32_t *col_idx, const int32_t *extra_idx,
                             const int32_t *extra_count, void *out, float *lse, int dense_only,
                             int row_begin, int row_end, char *ws, const WsLayout &L,
                             cudaStream_t st, int phase = 0);

// Selection with the library's static scratch array instead of a workspace.
bool static_select_layout(const bsa_params &p, WsLayout *L, size_t *need);
cudaError_t launch_select_static(const bsa_params &p, const Dims &D, const float *qbar, const float *kbar,
                                 int64_t *row_ptr, int32_t *col_idx, int64_t col_capacity,
                                 int32_t *kept_count, const WsLayout &L, cudaStream_t st);
size_t static_scratch_bytes();

// The QKV projection with pooling in its epilogue (bsa_qkv_pool).
cudaError_t launch_qkv_pool(const bsa_params &p, const Dims &D, const void *x, int d_model, const void *w, void *q,
                            void *k, void *v, float *qbar, float *kbar, float *vbar, int32_t *blk_count,
                            int32_t *status, cudaStream_t st);

// Query-block groups per (b, h) in the modified-centroid listing (about eight
// CTAs per SM over the whole problem).
inline int mc_groups(const Dims &D)
{
    const int64_t bh = (int64_t)D.B * D.H;
    const int64_t g = ceil_div(8 * (int64_t)sm_count(), bh);
    return (int)std::max<int64_t>(1, std::min<int64_t>(g, D.nQB));
}

// Exclusive scan of `rows` int32 counts into int64 row_ptr[rows + 1] (tile_sum:
// ceil(rows / 4096) int64 of scratch).
cudaError_t launch_scan(const int32_t *cnt, int64_t rows, int64_t *row_ptr, int64_t *tile_sum, cudaStream_t st);

// Extra tokens (E > 0): survivor buffer capacity per row, and the launch.
int64_t extra_buffer_capacity();
cudaError_t launch_extra(const bsa_params &p, const Dims &D, const float *qbar, const void *k,
                         int32_t *extra_idx, int32_t *extra_count, char *ws, const WsLayout &L, cudaStream_t st);

// Counts one kernel launch of this library (read by bsa_launch_count).
void count_launch();

// Thread-local host error text.
void set_error(const char *fmt, ...);

}  // namespace bsa
