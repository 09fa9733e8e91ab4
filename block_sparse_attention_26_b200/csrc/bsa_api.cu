// bsa_api.cu -- the extern "C" entry points declared in bsa.h: host-side
// validation, workspace layout and kernel launches.  No device memory is
// allocated here; every launch goes to the caller's stream.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <atomic>

#include "bsa_device.cuh"
#include "bsa_internal.h"

namespace bsa {

static thread_local char g_err[512] = "";

void set_error(const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
}

static std::atomic<int64_t> g_launches{0};

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

int sm_count()
{
    static std::atomic<int> cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 148;
    if (dev < 64) {
        const int c = cache[dev].load(std::memory_order_relaxed);
        if (c > 0) return c;
    }
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
    if (dev < 64) cache[dev].store(n, std::memory_order_relaxed);
    return n;
}

Dims dims_of(const bsa_params &p)
{
    Dims D;
    D.B = p.B;
    D.H = p.H;
    D.N = p.N;
    D.d = p.d;
    D.Bq = p.q_block;
    D.Bk = p.k_block;
    D.nQB = (int)ceil_div(p.N, p.q_block);
    D.nKB = (int)ceil_div(p.N, p.k_block);
    D.nW = (int)ceil_div(D.nKB, 32);
    D.rows = (int64_t)p.B * p.H * D.nQB;
    D.E = p.extra_tokens;
    D.cube = p.method == BSA_VSA;
    D.pre_blocks = D.cube ? p.prefix_len / 64 : 0;
    return D;
}

WsLayout ws_layout(const bsa_params &p)
{
    const Dims D = dims_of(p);
    WsLayout L;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off = align_up(off + bytes, 256);
        return at;
    };
    const int64_t BH = (int64_t)D.B * D.H;
    // the selection's scratch: its regions, then the extra-token passes'
    Taker T;
    select_regions(p, D, L, T);
    const bool ex = D.E > 0;
    L.ex_theta = T.take(ex ? (size_t)D.rows * 4 : 0);
    L.ex_smax = T.take(ex ? (size_t)D.rows * 4 : 0);
    L.ex_cut = T.take(ex ? (size_t)D.rows * 16 : 0);
    L.ex_buf = T.take(ex ? (size_t)D.rows * extra_buffer_capacity() * 8 : 0);
    L.ex_cnt = T.take(ex ? (size_t)D.rows * 4 : 0);
    L.ex_ovf = T.take(ex ? (size_t)(D.rows + 1) * 4 : 0);
    L.ex_scratch = T.take(ex ? (size_t)fallback_ctas() * D.N * 4 : 0);
    const size_t select_end = T.off;
    // the attention calls' scratch, over the same bytes after the status word
    off = align_up(L.status + 2 * sizeof(int32_t), 256);
    L.kc16 = take((size_t)BH * D.nKB * D.d * 2);
    L.vc16 = take((size_t)BH * D.nKB * D.d * 2);
    const int64_t ecap = ex ? std::min(D.E, D.nKB) : 0;
    const int64_t per_row = p.modcent_per_row > 0 ? std::min<int64_t>(p.modcent_per_row, ecap) : ecap;
    L.mc_cap = D.rows * per_row;
    const int64_t n3 = ex ? BH * D.nKB * mc_groups(D) : 0;
    L.xk16 = take((size_t)L.mc_cap * D.d * 2);
    L.xv16 = take((size_t)L.mc_cap * D.d * 2);
    L.xbias = take((size_t)L.mc_cap * 4);
    L.xcnt = take(ex ? (size_t)D.rows * 4 : 0);
    L.xoff = take(ex ? (size_t)(D.rows + 1) * 8 : 0);
    L.mc_slot = take((size_t)L.mc_cap * 4);
    L.mc_ent = take((size_t)L.mc_cap * 8);
    L.mc_cnt3 = take((size_t)n3 * 4);
    L.mc_off3 = take(ex ? (size_t)(n3 + 1) * 8 : 0);
    L.mc_tile = take(ex ? (size_t)ceil_div(std::max<int64_t>(D.rows, n3), 4096) * 8 : 0);
    const size_t ftiles = (size_t)BH * (size_t)((D.N + 127) / 128);
    L.glist = take(ex ? ftiles * kGlistCap * 4 : 0);
    L.glcnt = take(ex ? ftiles * 4 : 0);
    const size_t in16 = p.dtype == BSA_DT_F32 ? (size_t)D.B * D.N * D.H * D.d * 2 : 0;
    L.q16 = take(in16);
    L.k16 = take(in16);
    L.v16 = take(in16);
    // fp8 Q / K (qk_fp8): e4m3 copies and one scale per 64 tokens (per 64 centroids)
    const bool f8 = p.qk_fp8 != 0;
    const size_t ntok = (size_t)D.B * D.N * D.H * D.d;
    L.q8 = take(f8 ? ntok : 0);
    L.k8 = take(f8 ? ntok : 0);
    L.sq8 = take(f8 ? (size_t)BH * ceil_div(D.N, 64) * 4 : 0);
    L.sk8 = take(f8 ? (size_t)BH * D.nKB * 4 : 0);
    L.kc8 = take(f8 ? (size_t)BH * D.nKB * D.d : 0);
    L.skc8 = take(f8 ? (size_t)BH * ceil_div(D.nKB, 64) * 4 : 0);
    // fp8 P V (pv_fp8): e4m3 V and value centroids, one scale per (b, h, channel)
    const bool v8 = p.pv_fp8 != 0;
    L.v8 = take(v8 ? ntok : 0);
    L.vc8 = take(v8 ? (size_t)BH * D.nKB * D.d : 0);
    L.sv8 = take(v8 ? (size_t)BH * D.d * 4 : 0);
    L.part_tiles = dense_partial_tiles(D, p.dense_row_end - p.dense_row_begin);
    L.part_o = take((size_t)L.part_tiles * 128 * D.d * sizeof(float));
    L.part_ml = take((size_t)L.part_tiles * 128 * 2 * sizeof(float));
    L.total = std::max(off, select_end);
    return L;
}

}  // namespace bsa

using namespace bsa;

namespace {

#define FAIL(code, ...)            \
    do {                           \
        set_error(__VA_ARGS__);    \
        return (code);             \
    } while (0)

bool aligned16(const void *ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

bsa_status check_params(const bsa_params *p)
{
    if (p == nullptr) FAIL(BSA_ERR_INVALID_ARG, "params is NULL");
    if (p->B < 1 || p->H < 1 || p->N < 1) FAIL(BSA_ERR_INVALID_ARG, "B, H, N must be >= 1");
    if (p->d != 64 && p->d != 128) FAIL(BSA_ERR_UNSUPPORTED, "d = %d; supported head dims are 64 and 128", p->d);
    if (p->dtype != BSA_DT_BF16 && p->dtype != BSA_DT_F32) FAIL(BSA_ERR_INVALID_ARG, "unknown dtype %d", p->dtype);
    if (p->method != BSA_SOL && p->method != BSA_SLA && p->method != BSA_VSA)
        FAIL(BSA_ERR_UNSUPPORTED, "unknown method %d", p->method);
    if (p->k_block != 64) FAIL(BSA_ERR_UNSUPPORTED, "k_block must be 64");
    if (p->q_block != 64 && p->q_block != 128) FAIL(BSA_ERR_UNSUPPORTED, "q_block must be 64 or 128");
    const int64_t align_elems = p->dtype == BSA_DT_BF16 ? 8 : 4;
    if (p->stride_b <= 0 || p->stride_n <= 0 || p->stride_h <= 0)
        FAIL(BSA_ERR_INVALID_ARG, "strides must be positive");
    if (p->stride_b % align_elems || p->stride_n % align_elems || p->stride_h % align_elems)
        FAIL(BSA_ERR_INVALID_ARG, "strides must be multiples of %lld elements (16 bytes)", (long long)align_elems);
    if (p->stride_h < p->d) FAIL(BSA_ERR_INVALID_ARG, "stride_h smaller than d would overlap heads");
    if (isnan(p->tau)) FAIL(BSA_ERR_INVALID_ARG, "tau is NaN");
    if (p->method != BSA_SOL && !(p->keep_percent > 0.0 && p->keep_percent <= 100.0))
        FAIL(BSA_ERR_INVALID_ARG, "keep_percent must be in (0, 100]");
    if (p->qk_fp8 != 0 && p->qk_fp8 != 1) FAIL(BSA_ERR_INVALID_ARG, "qk_fp8 must be 0 or 1");
    if (p->pv_fp8 != 0 && p->pv_fp8 != 1) FAIL(BSA_ERR_INVALID_ARG, "pv_fp8 must be 0 or 1");
    if (p->pv_fp8 && !p->qk_fp8) FAIL(BSA_ERR_UNSUPPORTED, "pv_fp8 needs qk_fp8 (the all-fp8 mode)");
    if (p->qk_fp8) {
        if (p->dtype != BSA_DT_BF16 || p->d != 128 || p->extra_tokens != 0 || p->method == BSA_VSA)
            FAIL(BSA_ERR_UNSUPPORTED, "qk_fp8 needs bf16 inputs, d = 128, extra_tokens 0 and method Sol or SLA");
    }
    if (p->method == BSA_VSA) {
        if (p->q_block != 64) FAIL(BSA_ERR_UNSUPPORTED, "vsa: query cubes hold 64 tokens (q_block 64)");
        if (p->B != 1) FAIL(BSA_ERR_UNSUPPORTED, "vsa: B must be 1");
        if (p->cube_t < 1 || p->cube_h < 1 || p->cube_w < 1 || p->cube_t * p->cube_h * p->cube_w != 64)
            FAIL(BSA_ERR_UNSUPPORTED, "vsa: cube extents must multiply to 64");
        if (p->grid_t < 1 || p->grid_h < 1 || p->grid_w < 1 || p->grid_t % p->cube_t || p->grid_h % p->cube_h ||
            p->grid_w % p->cube_w)
            FAIL(BSA_ERR_UNSUPPORTED, "vsa: every grid extent must be a multiple of its cube extent");
        if (p->prefix_len % 64) FAIL(BSA_ERR_UNSUPPORTED, "vsa: prefix_len must be a multiple of 64");
        if ((int64_t)p->prefix_len + (int64_t)p->grid_t * p->grid_h * p->grid_w != p->N)
            FAIL(BSA_ERR_INVALID_ARG, "vsa: prefix_len + grid_t * grid_h * grid_w must equal N");
        if (p->dense_row_end > p->prefix_len) FAIL(BSA_ERR_UNSUPPORTED, "vsa: dense rows must lie in the prefix");
        if (p->centroid) FAIL(BSA_ERR_UNSUPPORTED, "vsa: the fine stage has no centroid term (centroid 0)");
        if (p->extra_tokens) FAIL(BSA_ERR_UNSUPPORTED, "vsa: extra_tokens is ignored for vsa; pass 0");
    }
    if (p->sink_blocks < 0) FAIL(BSA_ERR_INVALID_ARG, "sink_blocks < 0");
    if (p->keep_diag != 0 && p->keep_diag != 1) FAIL(BSA_ERR_INVALID_ARG, "keep_diag must be 0 or 1");
    if (p->prefix_len < 0 || p->prefix_len > p->N) FAIL(BSA_ERR_INVALID_ARG, "prefix_len outside [0, N]");
    if (p->dense_row_begin < 0 || p->dense_row_end < p->dense_row_begin || p->dense_row_end > p->N)
        FAIL(BSA_ERR_INVALID_ARG, "dense rows must satisfy 0 <= begin <= end <= N");
    if (p->extra_tokens < 0 || p->extra_tokens > 256) FAIL(BSA_ERR_INVALID_ARG, "extra_tokens outside [0, 256]");
    if (p->modcent_per_row < 0) FAIL(BSA_ERR_INVALID_ARG, "modcent_per_row < 0");
    if (p->extra_tokens > 0) {
        // modified-centroid slots are 30-bit fields of the fine pass's column codes
        const Dims D = dims_of(*p);
        const int64_t ecap = std::min(D.E, D.nKB);
        const int64_t per_row = p->modcent_per_row > 0 ? std::min<int64_t>(p->modcent_per_row, ecap) : ecap;
        if (D.rows * per_row >= (int64_t)1 << 30)
            FAIL(BSA_ERR_UNSUPPORTED, "modified-centroid capacity %lld >= 2^30 entries; lower modcent_per_row",
                 (long long)(D.rows * per_row));
    }
    if (p->centroid != 0 && p->centroid != 1) FAIL(BSA_ERR_INVALID_ARG, "centroid must be 0 or 1");
    const int64_t nKB = ceil_div(p->N, p->k_block);
    if (nKB > 65536) FAIL(BSA_ERR_UNSUPPORTED, "N too large: at most 65536 key blocks");
    const int64_t span = (int64_t)(p->B - 1) * p->stride_b + (int64_t)(p->N - 1) * p->stride_n +
                         (int64_t)(p->H - 1) * p->stride_h + p->d;
    if (span >= (int64_t)1 << 40) FAIL(BSA_ERR_UNSUPPORTED, "tensor span too large");
    return BSA_OK;
}

bsa_status check_ws(const bsa_params *p, void *ws, size_t ws_bytes)
{
    if (ws == nullptr) FAIL(BSA_ERR_WORKSPACE, "workspace is NULL");
    if (!aligned16(ws)) FAIL(BSA_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
    const WsLayout L = ws_layout(*p);
    if (ws_bytes < L.total)
        FAIL(BSA_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, L.total);
    return BSA_OK;
}

bsa_status check_tensor(const void *t, const char *name)
{
    if (t == nullptr) FAIL(BSA_ERR_INVALID_ARG, "%s is NULL", name);
    if (!aligned16(t)) FAIL(BSA_ERR_INVALID_ARG, "%s must be 16-byte aligned", name);
    return BSA_OK;
}

bsa_status from_cuda(cudaError_t e, const char *what)
{
    if (e == cudaSuccess) return BSA_OK;
    set_error("%s: %s", what, cudaGetErrorString(e));
    return BSA_ERR_CUDA;
}

#define TRY(x)                              \
    do {                                    \
        const bsa_status _s = (x);          \
        if (_s != BSA_OK) return _s;        \
    } while (0)

}  // namespace

extern "C" {

void bsa_default_params(bsa_params *p, int32_t method)
{
    if (p == nullptr) return;
    memset(p, 0, sizeof *p);
    p->method = method;
    p->dtype = BSA_DT_BF16;
    p->k_block = 64;
    p->q_block = method == BSA_SLA ? 128 : 64;
    p->tau = 1.3;
    p->keep_percent = 10.0;
    p->sink_blocks = 1;
    p->keep_diag = 1;
    p->centroid = method == BSA_SOL ? 1 : 0;
    if (method == BSA_VSA) {
        p->cube_t = p->cube_h = p->cube_w = 4;
    }
}

bsa_status bsa_workspace_size(const bsa_params *p, size_t *bytes, int64_t *max_nnz)
{
    g_err[0] = 0;
    TRY(check_params(p));
    if (bytes == nullptr) FAIL(BSA_ERR_INVALID_ARG, "bytes is NULL");
    *bytes = ws_layout(*p).total;
    if (max_nnz != nullptr) {
        const Dims D = dims_of(*p);
        *max_nnz = D.rows * D.nKB;
    }
    return BSA_OK;
}

bsa_status bsa_pool(const bsa_params *p, const void *q, const void *k, const void *v, float *qbar,
                    float *kbar, float *vbar, int32_t *blk_count, void *stream)
{
    g_err[0] = 0;
    TRY(check_params(p));
    TRY(check_tensor(q, "q"));
    TRY(check_tensor(k, "k"));
    TRY(check_tensor(v, "v"));
    TRY(check_tensor(qbar, "qbar"));
    TRY(check_tensor(kbar, "kbar"));
    TRY(check_tensor(vbar, "vbar"));
    const Dims D = dims_of(*p);
    return from_cuda(launch_pool(*p, D, q, k, v, qbar, kbar, vbar, blk_count, (cudaStream_t)stream), "bsa_pool");
}

bsa_status bsa_qkv_pool(const bsa_params *p, const void *x, int32_t d_model, const void *w_qkv, void *q, void *k,
                        void *v, float *qbar, float *kbar, float *vbar, int32_t *blk_count, void *ws, void *stream)
{
    g_err[0] = 0;
    TRY(check_params(p));
    if (p->dtype != BSA_DT_BF16) FAIL(BSA_ERR_UNSUPPORTED, "bsa_qkv_pool: bf16 only");
    if (p->method == BSA_VSA) FAIL(BSA_ERR_UNSUPPORTED, "bsa_qkv_pool: cube tiling pools cubes; use bsa_pool");
    if (d_model < 64 || d_model % 64) FAIL(BSA_ERR_UNSUPPORTED, "bsa_qkv_pool: d_model must be a multiple of 64");
    if ((p->H * p->d) % 256) FAIL(BSA_ERR_UNSUPPORTED, "bsa_qkv_pool: H * d must be a multiple of 256");
    TRY(check_tensor(x, "x"));
    TRY(check_tensor(w_qkv, "w_qkv"));
    TRY(check_tensor(q, "q"));
    TRY(check_tensor(k, "k"));
    TRY(check_tensor(v, "v"));
    TRY(check_tensor(qbar, "qbar"));
    TRY(check_tensor(kbar, "kbar"));
    TRY(check_tensor(vbar, "vbar"));
    if (ws != nullptr && !aligned16(ws)) FAIL(BSA_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
    const Dims D = dims_of(*p);
    return from_cuda(launch_qkv_pool(*p, D, x, d_model, w_qkv, q, k, v, qbar, kbar, vbar, blk_count,
                                     static_cast<int32_t *>(ws), (cudaStream_t)stream),
                     "bsa_qkv_pool");
}

bsa_status bsa_select(const bsa_params *p, const float *qbar, const float *kbar, const void *k,
                      int64_t *row_ptr, int32_t *col_idx, int64_t col_capacity, int32_t *kept_count,
                      int32_t *extra_idx, int32_t *extra_count, void *ws, size_t ws_bytes, void *stream)
{
    g_err[0] = 0;
    TRY(check_params(p));
    TRY(check_tensor(qbar, "qbar"));
    TRY(check_tensor(kbar, "kbar"));
    if (row_ptr == nullptr || kept_count == nullptr) FAIL(BSA_ERR_INVALID_ARG, "row_ptr / kept_count is NULL");
    if (col_capacity < 0) FAIL(BSA_ERR_INVALID_ARG, "col_capacity < 0");
    if (col_capacity > 0 && col_idx == nullptr) FAIL(BSA_ERR_INVALID_ARG, "col_idx is NULL");
    if (p->extra_tokens > 0) {
        if (p->dtype != BSA_DT_BF16) FAIL(BSA_ERR_UNSUPPORTED, "extra tokens need bf16 inputs");
        TRY(check_tensor(k, "k"));
        if (extra_idx == nullptr || extra_count == nullptr) FAIL(BSA_ERR_INVALID_ARG, "extra_idx / extra_count is NULL");
    }
    TRY(check_ws(p, ws, ws_bytes));
    const Dims D = dims_of(*p);
    const WsLayout L = ws_layout(*p);
    TRY(from_cuda(launch_select(*p, D, qbar, kbar, row_ptr, col_idx, col_capacity, kept_count,
                                static_cast<char *>(ws), L, (cudaStream_t)stream),
                  "bsa_select"));
    if (p->extra_tokens > 0)
        TRY(from_cuda(launch_extra(*p, D, qbar, k, extra_idx, extra_count, static_cast<char *>(ws), L,
                                   (cudaStream_t)stream),
                      "bsa_select (extra tokens)"));
    return BSA_OK;
}

bsa_status bsa_select_static(const bsa_params *p, const float *qbar, const float *kbar, int64_t *row_ptr,
                             int32_t *col_idx, int64_t col_capacity, int32_t *kept_count, void *stream)
{
    g_err[0] = 0;
    TRY(check_params(p));
    TRY(check_tensor(qbar, "qbar"));
    TRY(check_tensor(kbar, "kbar"));
    if (row_ptr == nullptr || kept_count == nullptr) FAIL(BSA_ERR_INVALID_ARG, "row_ptr / kept_count is NULL");
    if (col_capacity < 0) FAIL(BSA_ERR_INVALID_ARG, "col_capacity < 0");
    if (col_capacity > 0 && col_idx == nullptr) FAIL(BSA_ERR_INVALID_ARG, "col_idx is NULL");
    if (p->extra_tokens > 0) FAIL(BSA_ERR_UNSUPPORTED, "bsa_select_static does not pick extra tokens");
    WsLayout L;
    size_t need = 0;
    if (!static_select_layout(*p, &L, &need))
        FAIL(BSA_ERR_CAPACITY, "bsa_select_static: this problem needs %zu bytes of scratch, the static array holds %zu",
             need, static_scratch_bytes());
    const Dims D = dims_of(*p);
    return from_cuda(launch_select_static(*p, D, qbar, kbar, row_ptr, col_idx, col_capacity, kept_count, L,
                                          (cudaStream_t)stream),
                     "bsa_select_static");
}

}  // extern "C"

namespace {

bsa_status attention_call(const bsa_params *p, const void *q, const void *k, const void *v, const float *kbar,
                          const float *vbar, const int32_t *blk_count, const int64_t *row_ptr,
                          const int32_t *col_idx, const int32_t *extra_idx, const int32_t *extra_count,
                          void *out, float *lse, void *ws, size_t ws_bytes, void *stream, int phase)
{
    g_err[0] = 0;
    TRY(check_params(p));
    TRY(check_tensor(q, "q"));
    TRY(check_tensor(k, "k"));
    TRY(check_tensor(v, "v"));
    TRY(check_tensor(out, "out"));
    if (p->centroid) {
        TRY(check_tensor(kbar, "kbar"));
        TRY(check_tensor(vbar, "vbar"));
    }
    (void)blk_count;
    if (row_ptr == nullptr || col_idx == nullptr) FAIL(BSA_ERR_INVALID_ARG, "row_ptr / col_idx is NULL");
    if (p->extra_tokens > 0) {
        if (p->dtype != BSA_DT_BF16) FAIL(BSA_ERR_UNSUPPORTED, "extra tokens need bf16 inputs");
        if (extra_idx == nullptr || extra_count == nullptr) FAIL(BSA_ERR_INVALID_ARG, "extra_idx / extra_count is NULL");
        TRY(check_tensor(kbar, "kbar"));
        TRY(check_tensor(vbar, "vbar"));
    }
    TRY(check_ws(p, ws, ws_bytes));
    const Dims D = dims_of(*p);
    const WsLayout L = ws_layout(*p);
    return from_cuda(launch_attention(*p, D, q, k, v, kbar, vbar, row_ptr, col_idx, extra_idx, extra_count,
                                      out, lse, 0, p->dense_row_begin, p->dense_row_end,
                                      static_cast<char *>(ws), L, (cudaStream_t)stream, phase),
                     phase == 1 ? "bsa_attention_prepare" : phase == 2 ? "bsa_attention_run" : "bsa_attention");
}

// One warp waits, with a limit of `cycles`, on an mbarrier nothing arrives on;
// the bounded wait gives up, records BSA_DEV_TIMEOUT and the kernel returns.
__global__ void bounded_wait_kernel(int32_t *status, long long cycles)
{
    __shared__ uint64_t bar;
    __shared__ int32_t abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    mbar_wait_for(&bar, 0, &abort_flag, status, 0x5e1f, cycles);
}

}  // namespace

extern "C" {

bsa_status bsa_attention(const bsa_params *p, const void *q, const void *k, const void *v, const float *kbar,
                         const float *vbar, const int32_t *blk_count, const int64_t *row_ptr,
                         const int32_t *col_idx, const int32_t *extra_idx, const int32_t *extra_count,
                         void *out, float *lse, void *ws, size_t ws_bytes, void *stream)
{
    return attention_call(p, q, k, v, kbar, vbar, blk_count, row_ptr, col_idx, extra_idx, extra_count, out, lse,
                          ws, ws_bytes, stream, 0);
}

bsa_status bsa_attention_prepare(const bsa_params *p, const void *q, const void *k, const void *v,
                                 const float *kbar, const float *vbar, const int32_t *blk_count,
                                 const int64_t *row_ptr, const int32_t *col_idx, const int32_t *extra_idx,
                                 const int32_t *extra_count, void *out, float *lse, void *ws, size_t ws_bytes,
                                 void *stream)
{
    return attention_call(p, q, k, v, kbar, vbar, blk_count, row_ptr, col_idx, extra_idx, extra_count, out, lse,
                          ws, ws_bytes, stream, 1);
}

bsa_status bsa_attention_run(const bsa_params *p, const void *q, const void *k, const void *v, const float *kbar,
                             const float *vbar, const int32_t *blk_count, const int64_t *row_ptr,
                             const int32_t *col_idx, const int32_t *extra_idx, const int32_t *extra_count,
                             void *out, float *lse, void *ws, size_t ws_bytes, void *stream)
{
    return attention_call(p, q, k, v, kbar, vbar, blk_count, row_ptr, col_idx, extra_idx, extra_count, out, lse,
                          ws, ws_bytes, stream, 2);
}

int64_t bsa_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

bsa_status bsa_selftest_bounded_wait(void *ws, int64_t cycles, void *stream)
{
    g_err[0] = 0;
    if (ws == nullptr) FAIL(BSA_ERR_INVALID_ARG, "ws is NULL");
    if (!aligned16(ws)) FAIL(BSA_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
    if (cycles < 1 || cycles > 2000000000LL) FAIL(BSA_ERR_INVALID_ARG, "cycles outside [1, 2e9]");
    count_launch();
    bounded_wait_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(static_cast<int32_t *>(ws), (long long)cycles);
    return from_cuda(cudaGetLastError(), "bsa_selftest_bounded_wait");
}

bsa_status bsa_dense_ref_rows(const bsa_params *p, const void *q, const void *k, const void *v,
                              int32_t row_begin, int32_t row_end, void *out, float *lse, void *ws,
                              size_t ws_bytes, void *stream)
{
    g_err[0] = 0;
    TRY(check_params(p));
    TRY(check_tensor(q, "q"));
    TRY(check_tensor(k, "k"));
    TRY(check_tensor(v, "v"));
    TRY(check_tensor(out, "out"));
    if (row_begin < 0 || row_end < row_begin || row_end > p->N)
        FAIL(BSA_ERR_INVALID_ARG, "rows must satisfy 0 <= begin <= end <= N");
    TRY(check_ws(p, ws, ws_bytes));
    if (row_end == row_begin) return BSA_OK;
    const Dims D = dims_of(*p);
    const WsLayout L = ws_layout(*p);
    return from_cuda(launch_attention(*p, D, q, k, v, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, out,
                                      lse, 1, row_begin, row_end, static_cast<char *>(ws), L,
                                      (cudaStream_t)stream),
                     "bsa_dense_ref_rows");
}

bsa_status bsa_device_status(void *ws, void *stream, int32_t *device_status)
{
    g_err[0] = 0;
    if (ws == nullptr || device_status == nullptr) FAIL(BSA_ERR_INVALID_ARG, "ws / device_status is NULL");
    cudaStream_t st = (cudaStream_t)stream;
    TRY(from_cuda(cudaStreamSynchronize(st), "cudaStreamSynchronize"));
    int32_t h[2] = {0, 0};
    TRY(from_cuda(cudaMemcpyAsync(h, ws, sizeof h, cudaMemcpyDeviceToHost, st), "status copy"));
    TRY(from_cuda(cudaMemsetAsync(ws, 0, sizeof h, st), "status reset"));
    TRY(from_cuda(cudaStreamSynchronize(st), "cudaStreamSynchronize"));
    *device_status = h[0];
    if (h[0] != 0) set_error("device status %d (detail %d)", h[0], h[1]);
    return BSA_OK;
}

const char *bsa_status_string(bsa_status s)
{
    switch (s) {
    case BSA_OK: return "ok";
    case BSA_ERR_INVALID_ARG: return "invalid argument";
    case BSA_ERR_UNSUPPORTED: return "unsupported";
    case BSA_ERR_CAPACITY: return "capacity exceeded";
    case BSA_ERR_WORKSPACE: return "workspace missing or too small";
    case BSA_ERR_CUDA: return "CUDA error";
    case BSA_ERR_DEVICE: return "device-side error";
    }
    return "unknown status";
}

const char *bsa_last_error(void) { return g_err; }

}  // extern "C"
