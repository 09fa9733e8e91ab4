// select.cu -- step 2: routing of key blocks per (batch, head, query block).
//
// "BlockSparseAttention - ComfyUI Built-in Node Documentation":
//   "sol-attn inputs", tau: a threshold counted in standard deviations of the
//   row's score distribution (higher = sparser);
//   "sla inputs", keep_percent: the percentage of key blocks kept exactly per
//   query block, sink and diagonal blocks kept in addition;
//   general inputs, sink_conditioning = exact_kv: every query attends exactly
//   to the packed conditioning rows.
//
// Kernels:
//   scores_kernel  S[r, j] = fl32((qbar_r . kbar_j) / sqrt d) with fp64 FMAs in
//                  channel order (the same value the definition gives).  A CTA
//                  computes a 32-row x 128-key tile per pass over kbar, staging
//                  channel slices of kbar in shared memory as fp64.
//   rows_kernel    one warp per row: two-pass fp64 mean / population std,
//                  thr = fl32(mean + tau * std), keep S > thr (Sol) or an exact
//                  radix select of the top k (SLA); forced blocks OR'ed in;
//                  result as a bitmask word per 32 key blocks (ballot) + count.
//   scan_kernel    exclusive scan of the counts -> CSR row_ptr (int64).
//   expand_kernel  bitmask -> ascending CSR column lists (popc prefix per warp).
#include <math.h>

#include <algorithm>
#include <atomic>

#include "bsa_device.cuh"
#include "bsa_internal.h"

namespace bsa {
namespace {

constexpr int kRows = 64;     // query-block rows per CTA (8 per warp)
constexpr int kKeys = 128;    // key blocks per pass
constexpr int kChan = 32;     // channels staged per step

__global__ void __launch_bounds__(256) scores_kernel(const float *__restrict__ qbar,
                                                     const float *__restrict__ kbar, int nQB,
                                                     int nKB, int d, float *__restrict__ S)
{
    extern __shared__ double sel_smem[];
    double(*qs)[128] = reinterpret_cast<double(*)[128]>(sel_smem);
    double(*ks)[kKeys + 1] = reinterpret_cast<double(*)[kKeys + 1]>(sel_smem + kRows * 128);
    const int bh = blockIdx.y;
    const int r0 = blockIdx.x * kRows;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const double rs = sqrt((double)d);

    for (int idx = threadIdx.x; idx < kRows * d; idx += blockDim.x) {
        const int r = idx / d, c = idx % d;
        qs[r][c] = (r0 + r < nQB) ? (double)qbar[((int64_t)bh * nQB + r0 + r) * d + c] : 0.0;
    }
    const float *kb = kbar + (int64_t)bh * nKB * d;
    for (int j0 = 0; j0 < nKB; j0 += kKeys) {
        double acc[8][4];   // 8 rows x 4 keys per thread: 12 shared loads per 32 FMAs
#pragma unroll
        for (int a = 0; a < 8; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) acc[a][b] = 0.0;
        for (int c0 = 0; c0 < d; c0 += kChan) {
            __syncthreads();
            for (int idx = threadIdx.x; idx < kKeys * kChan; idx += blockDim.x) {
                const int j = idx / kChan, c = idx % kChan;
                ks[c][j] = (j0 + j < nKB) ? (double)kb[(int64_t)(j0 + j) * d + c0 + c] : 0.0;
            }
            __syncthreads();
#pragma unroll 2
            for (int c = 0; c < kChan; ++c) {
                double qv[8], kv[4];
#pragma unroll
                for (int a = 0; a < 8; ++a) qv[a] = qs[8 * warp + a][c0 + c];
#pragma unroll
                for (int b = 0; b < 4; ++b) kv[b] = ks[c][lane + 32 * b];
#pragma unroll
                for (int a = 0; a < 8; ++a)
#pragma unroll
                    for (int b = 0; b < 4; ++b) acc[a][b] = __fma_rn(qv[a], kv[b], acc[a][b]);
            }
        }
#pragma unroll
        for (int a = 0; a < 8; ++a) {
            const int r = r0 + 8 * warp + a;
            if (r >= nQB) continue;
            float *row = S + ((int64_t)bh * nQB + r) * nKB;
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const int j = j0 + lane + 32 * b;
                if (j < nKB) row[j] = (float)(acc[a][b] / rs);
            }
        }
    }
}

struct RowArgs {
    const float *S;
    int64_t rows;
    int nQB, nKB, nW, N, Bq, Bk;
    int method;
    double tau;
    int topk;
    int sink_blocks, prefix_blocks, keep_diag;
    uint32_t *bitmask;
    int32_t *count;
};

__device__ __forceinline__ double warp_sum(double v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Order-preserving map of a float to uint32 (larger float -> larger key);
// -0 and +0 map to the same key so that they tie, as in a float comparison.
__device__ __forceinline__ uint32_t ord_key(float f)
{
    uint32_t u = __float_as_uint(f);
    if ((u & 0x7fffffffu) == 0) u = 0;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__global__ void __launch_bounds__(256) rows_kernel(RowArgs a)
{
    __shared__ uint32_t hist_all[8][256];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t r = (int64_t)blockIdx.x * 8 + warp;
    if (r >= a.rows) return;
    const float *s = a.S + r * a.nKB;
    const int i = (int)(r % a.nQB);
    const int nKB = a.nKB;

    // forced: [0, fb) sink/prefix, and the diagonal range [d0, d1]
    const int fb = max(min(a.sink_blocks, nKB), min(a.prefix_blocks, nKB));
    int d0 = 1, d1 = 0;
    if (a.keep_diag) {
        const int q0 = i * a.Bq, q1 = min(a.N, q0 + a.Bq) - 1;
        d0 = q0 / a.Bk;
        d1 = min(q1 / a.Bk, nKB - 1);
    }

    int mode = 0;            // 0: threshold, 1: keep all, 2: none, 3: top-k
    float thr = 0.f;
    uint32_t vk = 0;
    int need = 0;
    if (a.method == BSA_SOL) {
        if (isinf(a.tau) && a.tau < 0) {
            mode = 1;
        } else {
            double sum = 0.0;
            for (int j = lane; j < nKB; j += 32) sum += (double)s[j];
            const double mu = warp_sum(sum) / (double)nKB;
            double sq = 0.0;
            for (int j = lane; j < nKB; j += 32) {
                const double e = __dadd_rn((double)s[j], -mu);
                sq = __dadd_rn(sq, __dmul_rn(e, e));
            }
            const double sigma = sqrt(warp_sum(sq) / (double)nKB);
            if (isinf(a.tau) || !(sigma > 0.0)) {
                mode = 2;
            } else {
                thr = (float)__dadd_rn(mu, __dmul_rn(a.tau, sigma));
            }
        }
    } else {
        // exact k-th largest key by 8-bit radix passes, then ties to the lower index
        uint32_t *hist = hist_all[warp];
        uint32_t prefix = 0, pmask = 0;
        int remaining = a.topk;
        for (int shift = 24; shift >= 0; shift -= 8) {
            for (int t = lane; t < 256; t += 32) hist[t] = 0;
            __syncwarp();
            for (int j = lane; j < nKB; j += 32) {
                const uint32_t u = ord_key(s[j]);
                if ((u & pmask) == prefix) atomicAdd(&hist[(u >> shift) & 255u], 1u);
            }
            __syncwarp();
            int digit = 0, above = 0;
            if (lane == 0) {
                int acc = 0;
                for (int bin = 255; bin >= 0; --bin) {
                    const int c = (int)hist[bin];
                    if (acc + c >= remaining) {
                        digit = bin;
                        above = acc;
                        break;
                    }
                    acc += c;
                }
            }
            digit = __shfl_sync(0xffffffffu, digit, 0);
            above = __shfl_sync(0xffffffffu, above, 0);
            remaining -= above;
            prefix |= (uint32_t)digit << shift;
            pmask |= 0xFFu << shift;
            __syncwarp();
        }
        vk = prefix;
        need = remaining;    // elements equal to vk still to take, lowest index first
        mode = 3;
    }

    int total = 0, eq_taken = 0;
    uint32_t *bm = a.bitmask + r * a.nW;
    const uint32_t lt_mask = (1u << lane) - 1u;
    for (int w = 0; w < a.nW; ++w) {
        const int j = w * 32 + lane;
        const bool valid = j < nKB;
        const float sj = valid ? s[j] : 0.f;
        bool keep = false;
        if (mode == 0) {
            keep = valid && sj > thr;
        } else if (mode == 1) {
            keep = valid;
        } else if (mode == 3) {
            const uint32_t u = ord_key(sj);
            const bool eq = valid && u == vk;
            const uint32_t eqm = __ballot_sync(0xffffffffu, eq);
            const int rank = eq_taken + __popc(eqm & lt_mask);
            keep = valid && (u > vk || (eq && rank < need));
            eq_taken += __popc(eqm);
        }
        keep = keep || (valid && (j < fb || (j >= d0 && j <= d1)));
        const uint32_t word = __ballot_sync(0xffffffffu, keep);
        if (lane == 0) bm[w] = word;
        total += __popc(word);
    }
    if (lane == 0) a.count[r] = total;
}

// Exclusive scan of the kept counts into int64 row_ptr, in three launches:
// each CTA scans a tile of kScanTile rows (4 per thread) and records the
// tile's total; one CTA scans the totals; every row adds its tile's offset.
constexpr int kScanTile = 4096;

__global__ void __launch_bounds__(1024) scan_tiles_kernel(const int32_t *__restrict__ count, int64_t rows,
                                                          int64_t *__restrict__ row_ptr, int64_t *__restrict__ tile_sum)
{
    __shared__ int64_t wsum[32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t r0 = (int64_t)blockIdx.x * kScanTile + 4 * threadIdx.x;
    int64_t v[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) v[e] = r0 + e < rows ? count[r0 + e] : 0;
    const int64_t s = v[0] + v[1] + v[2] + v[3];
    int64_t incl = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int64_t t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int64_t x = wsum[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int64_t t = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += t;
        }
        wsum[lane] = x;
    }
    __syncthreads();
    int64_t base = (warp > 0 ? wsum[warp - 1] : 0) + incl - s;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        if (r0 + e < rows) row_ptr[r0 + e] = base;
        base += v[e];
    }
    if (threadIdx.x == 1023) tile_sum[blockIdx.x] = wsum[31];
}

__global__ void __launch_bounds__(1024) scan_tops_kernel(int64_t *__restrict__ tile_sum, int ntiles,
                                                         int64_t *__restrict__ row_ptr, int64_t rows)
{
    __shared__ int64_t wsum[32];
    __shared__ int64_t carry_s;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) carry_s = 0;
    __syncthreads();
    for (int t0 = 0; t0 < ntiles; t0 += 1024) {
        const int t = t0 + threadIdx.x;
        const int64_t s = t < ntiles ? tile_sum[t] : 0;
        int64_t incl = s;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int64_t y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) wsum[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            int64_t x = wsum[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int64_t y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += y;
            }
            wsum[lane] = x;
        }
        __syncthreads();
        const int64_t carry = carry_s;
        if (t < ntiles) tile_sum[t] = carry + (warp > 0 ? wsum[warp - 1] : 0) + incl - s;
        __syncthreads();
        if (threadIdx.x == 0) carry_s = carry + wsum[31];
        __syncthreads();
    }
    if (threadIdx.x == 0) row_ptr[rows] = carry_s;
}

__global__ void __launch_bounds__(256) scan_add_kernel(int64_t *__restrict__ row_ptr, int64_t rows,
                                                       const int64_t *__restrict__ tile_off)
{
    for (int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; r < rows; r += (int64_t)gridDim.x * blockDim.x)
        row_ptr[r] += tile_off[r / kScanTile];
}


// One warp per row, its words 32 at a time: every lane counts its word's bits
// and a warp scan gives every word its first output slot.  A sparse word (at
// most 4 bits) is written by its own lane, a bit per step; a dense word (the
// kept blocks near the diagonal) by the whole warp at once, lane l testing bit
// l -- so a few dense words do not hold the other lanes for 32 steps.
__global__ void __launch_bounds__(256) expand_kernel(const uint32_t *__restrict__ bitmask,
                                                     const int32_t *__restrict__ count,
                                                     const int64_t *__restrict__ row_ptr,
                                                     int64_t rows, int nW, int64_t capacity,
                                                     int32_t *__restrict__ col,
                                                     int32_t *__restrict__ kept_count,
                                                     int32_t *status)
{
    constexpr int kSparse = 4;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t r = (int64_t)blockIdx.x * 8 + warp;
    if (r >= rows) return;
    const int64_t start = row_ptr[r];
    if (lane == 0) {
        kept_count[r] = count[r];
        if (start + count[r] > capacity) report(status, BSA_DEV_CAPACITY, (int32_t)(r & 0x7fffffff));
    }
    const uint32_t *bm = bitmask + r * nW;
    const uint32_t lt = (1u << lane) - 1u;
    int64_t base = start;
    for (int w0 = 0; w0 < nW; w0 += 32) {
        const int w = w0 + lane;
        const uint32_t word = w < nW ? bm[w] : 0u;
        const int pc = __popc(word);
        int incl = pc;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        const int64_t first = base + (incl - pc);
        // sparse words: each lane its own
        if (pc <= kSparse) {
            int64_t pos = first;
            for (uint32_t m = word; m != 0u; m &= m - 1u, ++pos)
                if (pos < capacity) col[pos] = w * 32 + __ffs(m) - 1;
        }
        // dense words: the warp takes them one by one
        for (uint32_t dense = __ballot_sync(0xffffffffu, pc > kSparse); dense != 0u; dense &= dense - 1u) {
            const int src = __ffs(dense) - 1;
            const uint32_t wd = __shfl_sync(0xffffffffu, word, src);
            const int64_t f = __shfl_sync(0xffffffffu, first, src);
            if ((wd >> lane) & 1u) {
                const int64_t pos = f + __popc(wd & lt);
                if (pos < capacity) col[pos] = (w0 + src) * 32 + lane;
            }
        }
        base += __shfl_sync(0xffffffffu, incl, 31);
    }
}

}  // namespace

cudaError_t launch_scan(const int32_t *cnt, int64_t rows, int64_t *row_ptr, int64_t *tile_sum, cudaStream_t st)
{
    const int ntiles = (int)ceil_div(rows, kScanTile);
    count_launch();
    scan_tiles_kernel<<<(unsigned)ntiles, 1024, 0, st>>>(cnt, rows, row_ptr, tile_sum);
    count_launch();
    scan_tops_kernel<<<1, 1024, 0, st>>>(tile_sum, ntiles, row_ptr, rows);
    const unsigned g = (unsigned)std::min<int64_t>(ceil_div(rows, 256), (int64_t)sm_count() * 8);
    count_launch();
    scan_add_kernel<<<g, 256, 0, st>>>(row_ptr, rows, tile_sum);
    return cudaGetLastError();
}

void select_regions(const bsa_params &p, const Dims &D, WsLayout &L, Taker &T)
{
    const bool route = certified_route(p);
    const int64_t BH = (int64_t)D.B * D.H;
    const size_t rows = (size_t)D.rows;
    L.status = T.take(sizeof(int32_t) * 2);
    // block scores: all of them on the fp64 path; on the certified route only
    // approximate ones, for the extra-token sampler
    L.scores = T.take(!route || p.extra_tokens > 0 ? rows * D.nKB * sizeof(float) : 0);
    L.bitmask = T.take(rows * D.nW * sizeof(uint32_t));
    L.counts = T.take(rows * sizeof(int32_t));
    L.scan_tmp = T.take((size_t)ceil_div(D.rows, kScanTile) * sizeof(int64_t));
    const size_t d = (size_t)D.d;
    const int ns = route ? route_nsplit(D) : 0;
    L.r_nsplit = ns;
    L.r_k16 = T.take(route ? (size_t)BH * D.nKB * d * 2 : 0);
    L.r_knorm = T.take(route ? (size_t)BH * route_nkbp(D) * 4 : 0);
    L.r_knmax = T.take(route ? (size_t)BH * (route_nkbp(D) / 32) * 4 : 0);
    L.r_gram = T.take(route ? (size_t)BH * ns * d * d * 8 : 0);
    L.r_ksum = T.take(route ? (size_t)BH * ns * d * 8 : 0);
    L.r_cov = T.take(route ? (size_t)BH * d * d * 8 : 0);
    L.r_hstat = T.take(route ? (size_t)BH * (d + 3) * 8 : 0);
    L.r_info = T.take(route ? rows * sizeof(RowInfo) : 0);
    L.r_fbl = T.take(route ? (rows + 1) * 4 : 0);
    L.r_fbs = T.take(route ? (size_t)fallback_ctas() * route_nkbp(D) * 4 : 0);
}

cudaError_t launch_select(const bsa_params &p, const Dims &D, const float *qbar, const float *kbar,
                          int64_t *row_ptr, int32_t *col_idx, int64_t col_capacity,
                          int32_t *kept_count, char *ws, const WsLayout &L, cudaStream_t st)
{
    float *S = reinterpret_cast<float *>(ws + L.scores);
    uint32_t *bm = reinterpret_cast<uint32_t *>(ws + L.bitmask);
    int32_t *cnt = reinterpret_cast<int32_t *>(ws + L.counts);
    int32_t *status = reinterpret_cast<int32_t *>(ws + L.status);
    int64_t *tsum = reinterpret_cast<int64_t *>(ws + L.scan_tmp);
    const unsigned g2 = (unsigned)ceil_div(D.rows, 8);

    if (certified_route(p)) {
        cudaError_t e = launch_route(p, D, qbar, kbar, ws, L, st);
        if (e != cudaSuccess) return e;
        e = launch_scan(cnt, D.rows, row_ptr, tsum, st);
        if (e != cudaSuccess) return e;
        count_launch();
        expand_kernel<<<g2, 256, 0, st>>>(bm, cnt, row_ptr, D.rows, D.nW, col_capacity, col_idx, kept_count,
                                          status);
        return cudaGetLastError();
    }

    dim3 g1((unsigned)ceil_div(D.nQB, kRows), (unsigned)(D.B * D.H));
    const int smem = (kRows * 128 + kChan * (kKeys + 1)) * (int)sizeof(double);
    cudaError_t e = cudaFuncSetAttribute(scores_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    count_launch();
    scores_kernel<<<g1, 256, smem, st>>>(qbar, kbar, D.nQB, D.nKB, D.d, S);

    RowArgs a;
    a.S = S;
    a.rows = D.rows;
    a.nQB = D.nQB;
    a.nKB = D.nKB;
    a.nW = D.nW;
    a.N = D.N;
    a.Bq = D.Bq;
    a.Bk = D.Bk;
    a.method = p.method;
    a.tau = p.tau;
    long kk = lround(p.keep_percent * (double)D.nKB / 100.0);
    if (kk < 1) kk = 1;
    if (kk > D.nKB) kk = D.nKB;
    a.topk = (int)kk;
    a.sink_blocks = p.sink_blocks;
    a.prefix_blocks = p.prefix_len > 0 ? (int)ceil_div(p.prefix_len, D.Bk) : 0;
    a.keep_diag = p.keep_diag;
    a.bitmask = bm;
    a.count = cnt;
    count_launch();
    rows_kernel<<<g2, 256, 0, st>>>(a);
    cudaError_t es = launch_scan(cnt, D.rows, row_ptr, tsum, st);
    if (es != cudaSuccess) return es;
    count_launch();
    expand_kernel<<<g2, 256, 0, st>>>(bm, cnt, row_ptr, D.rows, D.nW, col_capacity, col_idx,
                                      kept_count, status);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Selection without caller-provided scratch.
//
// Some callers cannot allocate device memory at all: code that runs inside a
// host framework owning every allocation, a plugin that may not call
// cudaMalloc on its host's streams, or a process whose allocator is locked
// while it serves requests.  For them bsa_select_static() keeps the selection
// scratch (block scores, kept-block bitmasks, per-row counts and the status
// word) in the file-scope device array below instead of a workspace.  The
// array has a fixed size; every GPU that loads the library holds it until the
// process exits.
constexpr size_t kStaticScratchBytes = (size_t)32 << 20;   // 32 MiB
static __device__ __align__(256) unsigned char g_select_scratch[kStaticScratchBytes];

namespace {

constexpr int kMaxDevices = 64;

// The array's device address belongs to the module as loaded into one CUDA
// context; after a device reset the module is loaded again, possibly at
// another address.  Each device's entry therefore remembers the context it was
// looked up in and is looked up again when the current context differs.
struct StaticBase {
    std::atomic<void *> ctx{nullptr};
    std::atomic<char *> base{nullptr};
};
StaticBase g_static_base[kMaxDevices];

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);

CtxGetCurrentFn ctx_get_current_fn()
{
    static std::atomic<CtxGetCurrentFn> fn{nullptr};
    CtxGetCurrentFn f = fn.load(std::memory_order_acquire);
    if (f == nullptr) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess) {
            f = reinterpret_cast<CtxGetCurrentFn>(p);
            fn.store(f, std::memory_order_release);
        }
    }
    return f;
}

// Device address of g_select_scratch on the current device (looked up once per
// device and context; the host-side symbol is only a stand-in and must never
// be passed to a kernel).
cudaError_t static_scratch(char **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    CtxGetCurrentFn get = ctx_get_current_fn();
    if (get == nullptr) return cudaErrorDeviceUninitialized;
    CUcontext ctx = nullptr;
    if (get(&ctx) != CUDA_SUCCESS) return cudaErrorDeviceUninitialized;
    StaticBase &slot = g_static_base[dev];
    char *p = slot.base.load(std::memory_order_acquire);
    if (ctx == nullptr || p == nullptr || slot.ctx.load(std::memory_order_acquire) != (void *)ctx) {
        // (the lookup also makes the device's primary context current when
        // this thread has none yet)
        void *addr = nullptr;
        e = cudaGetSymbolAddress(&addr, g_select_scratch);
        if (e != cudaSuccess) return e;
        if (ctx == nullptr && (get(&ctx) != CUDA_SUCCESS || ctx == nullptr)) return cudaErrorDeviceUninitialized;
        p = static_cast<char *>(addr);
        slot.base.store(nullptr, std::memory_order_release);
        slot.ctx.store((void *)ctx, std::memory_order_release);
        slot.base.store(p, std::memory_order_release);
    }
    *out = p;
    return cudaSuccess;
}

}  // namespace

// Layout of the selection scratch inside the static array; false if it does not fit.
bool static_select_layout(const bsa_params &p, WsLayout *L, size_t *need)
{
    const Dims D = dims_of(p);
    *L = WsLayout();
    Taker T;
    select_regions(p, D, *L, T);
    L->total = T.off;
    *need = T.off;
    return T.off <= kStaticScratchBytes;
}

cudaError_t launch_select_static(const bsa_params &p, const Dims &D, const float *qbar, const float *kbar,
                                 int64_t *row_ptr, int32_t *col_idx, int64_t col_capacity,
                                 int32_t *kept_count, const WsLayout &L, cudaStream_t st)
{
    char *base = nullptr;
    cudaError_t e = static_scratch(&base);
    if (e != cudaSuccess) return e;
    // the status word is the only region read before it is written
    e = cudaMemsetAsync(base + L.status, 0, sizeof(int32_t) * 2, st);
    if (e != cudaSuccess) return e;
    return launch_select(p, D, qbar, kbar, row_ptr, col_idx, col_capacity, kept_count, base, L, st);
}

size_t static_scratch_bytes() { return kStaticScratchBytes; }

}  // namespace bsa
