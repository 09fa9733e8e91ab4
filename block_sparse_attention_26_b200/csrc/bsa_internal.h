// bsa_internal.h -- declarations shared by the host API and the kernel files.
#pragma once

#include <cuda_runtime.h>
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

// Derived sizes of one problem.
struct Dims {
    int B, H, N, d;
    int Bq, Bk;
    int nQB, nKB, nW;      // nW = 32-bit words of a per-row key-block bitmask
    int64_t rows;          // B * H * nQB
    int E;
};

Dims dims_of(const bsa_params &p);

// Byte offsets of the workspace regions (each 256-byte aligned).
struct WsLayout {
    size_t status;         // DevStatus
    size_t scores;         // [rows, nKB] f32 block scores (select)
    size_t bitmask;        // [rows, nW] u32 kept-block bitmask (select)
    size_t counts;         // [rows] i32 kept counts (select)
    size_t kc16, vc16;     // [B*H, nKB, d] bf16 centroids (attention)
    size_t xk16, xv16;     // [rows, min(E, nKB), d] bf16 modified centroids (extra tokens)
    size_t xbias;          // [rows, min(E, nKB)] f32 their log2 token counts
    size_t xcnt;           // [rows] i32 modified centroids per row
    size_t xaff;           // [rows, nW] u32 blocks that gave extra tokens
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
    size_t part_o;         // [part_tiles, 128, d] f32 dense-row partial outputs
    size_t part_ml;        // [part_tiles, 128, 2] f32 dense-row partial (max, sum)
    int64_t part_tiles;    // capacity of the partial buffers, in 128-row tiles
    size_t total;
};

WsLayout ws_layout(const bsa_params &p);

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

// Extra tokens (E > 0): survivor buffer capacity per row, and the launch.
int64_t extra_buffer_capacity();
cudaError_t launch_extra(const bsa_params &p, const Dims &D, const float *qbar, const void *k,
                         int32_t *extra_idx, int32_t *extra_count, char *ws, const WsLayout &L, cudaStream_t st);

// Thread-local host error text.
void set_error(const char *fmt, ...);

}  // namespace bsa
