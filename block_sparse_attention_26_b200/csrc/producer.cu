// producer.cu -- the QKV projection with the pooling step folded into its
// epilogue.
//
// "minimax-h3-chunk-star7" README, "Sol": a producer with fused
// preprocessing builds the attention inputs and reuses the current input
// statistics.  Here: [Q | K | V] = X W^T (X [B*N, d_model] bf16, W
// [3*H*d, d_model] bf16, the usual linear-layer weight layout, heads of Q, then
// K, then V, d rows each), written as bf16 [B, N, H, d] tensors, and in the
// same kernel the block means qbar, kbar, vbar of the rounded outputs (the
// pooling step), so that the 3*N*d read of a separate pooling pass disappears.
//
// Persistent tcgen05 GEMM on CTA pairs (clusters of 2): 256 x 256 output tiles
// (M = 256 tokens, 128 per CTA; N = 256 columns = 256 / d heads of one of Q, K,
// V), one M = 256 UMMA per K = 16 step issued by the even CTA for both
// (cta_group::2): each CTA holds its 128 rows of X and half of the tile's W rows,
// so an SM brings in 32 KB of operands per K step of 64 where a one-SM 128 x 256
// tile needs 48 KB (shared-memory bandwidth is what bounds the one-SM form).
// K steps of 64 through a 4-deep TMA ring per CTA, both CTAs' loads completing
// on the even CTA's barrier; fp32 accumulators double-buffered in each CTA's
// TMEM (512 columns) so that a tile's epilogue overlaps the next tile's MMAs.
// Warps 0-3 run the epilogue (TMEM lane quarter = warp), warp 4 loads, warp 5
// issues the MMAs (even CTA) and owns TMEM.
//
// Epilogue: each thread takes its row, rounds it to bf16 into a staging tile
// laid out for a TMA store (128-byte swizzle), the tile is stored by TMA, and
// the block sums are taken from the staging tile: one thread per (block,
// column), over the block's valid rows in token order in fp64, divided by the
// count and rounded once to f32 -- the pooling step's own arithmetic.  A tile
// starts at a multiple of 128 tokens of its batch, so it holds whole 64- (or
// 128-) token blocks.
#include <math.h>

#include <algorithm>

#include "bsa_device.cuh"
#include "bsa_internal.h"

namespace bsa {
namespace {

constexpr int kPM = 128;       // tokens per CTA (a pair's tile: 256)
constexpr int kPN = 256;       // output columns per tile (128 W rows per CTA)
constexpr int kPK = 64;        // K per stage
constexpr int kPStages = 4;
constexpr int kBandM = 24;     // m tiles (of 256 tokens) per raster band (their A tiles stay in L2)
constexpr int kPThreads = 192;

struct ProdArgs {
    int B, N, H, d, dm;
    int64_t sb, sn, sh;        // output strides (elements)
    int Bq;                    // query block (64 or 128); key blocks are 64
    int nQB, nKB;
    int tiles_m_b, tiles_m, tiles_n, ntiles;
    float *qbar, *kbar, *vbar;
    int32_t *count;
    int32_t *status;
};

struct PLay {
    static constexpr int kABytes = kPM * kPK * 2;           // 16 KB
    static constexpr int kBBytes = kPN / 2 * kPK * 2;       // 16 KB: this CTA's half of the W rows
    static constexpr int kStage = kABytes + kBBytes;
    static constexpr int kOffStages = 0;
    static constexpr int kOffStg = kPStages * kStage;      // staging tile, 64 KB
    static constexpr int kStgBytes = kPM * kPN * 2;
    static constexpr int kOffBar = kOffStg + kStgBytes;    // full[S], empty[S], acc_full[2], acc_empty[2], stg_full, stg_free
    static constexpr int kOffMisc = kOffBar + (2 * kPStages + 6) * 8;
    static constexpr size_t bytes = (size_t)kOffMisc + 16 + 1024;
    static_assert(bytes <= 232448, "producer tile exceeds the per-block shared memory limit");
};

// ------------------------------------------------------------ CTA pairs
__device__ __forceinline__ uint32_t cluster_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// The shared::cluster address of the same shared variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_rank(const void *p, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
    return r;
}

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr)
{
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// 2-D tile load into this CTA's shared memory, completing on an mbarrier that may
// sit in the other CTA of the pair (shared::cluster address).
__device__ __forceinline__ void tma_load_2d_pair(void *dst, const CUtensorMap *map, uint32_t bar_cluster, int c0, int c1)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1)
        : "memory");
}

// D[tmem of both CTAs] (+)= A[smem of both] * B[smem of both]^T, M = 256.
__device__ __forceinline__ void umma_bf16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                               uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

// Arrive on `bar` in both CTAs of the pair once every pair MMA issued so far completes.
__device__ __forceinline__ void umma_commit_pair(uint64_t *bar)
{
    asm volatile(
        "{\n\t.reg .b16 m;\n\tmov.b16 m, 3;\n\t"
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], m;\n\t}" ::"r"(
            smem_u32(bar))
        : "memory");
}

// Tile t of the raster: bands of kBandM m tiles, n-major inside a band.
__device__ __forceinline__ void tile_mn(const ProdArgs &a, int t, int *m, int *n)
{
    const int per_band = kBandM * a.tiles_n;
    const int band = t / per_band;
    const int rem = t - band * per_band;
    const int nb = min(kBandM, a.tiles_m - band * kBandM);
    *n = rem / nb;
    *m = band * kBandM + rem % nb;
}

__global__ void __launch_bounds__(kPThreads, 1)
    qkv_pool_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const ProdArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t crank = cluster_rank();          // 0: the CTA that issues the pair's MMAs
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + PLay::kOffBar);
    uint64_t *full = bars, *empty = bars + kPStages, *acc_full = bars + 2 * kPStages, *acc_empty = acc_full + 2;
    uint64_t *stg_full = acc_empty + 2, *stg_free = stg_full + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + PLay::kOffMisc);
    volatile int32_t *abort_flag = reinterpret_cast<volatile int32_t *>(sm + PLay::kOffMisc + 4);
    uint8_t *stg = sm + PLay::kOffStg;
    const int ksteps = a.dm / kPK;
    const int HT = kPN / a.d;           // heads per tile

    if (threadIdx.x == 0) {
        for (int s = 0; s < kPStages; ++s) {
            mbar_init(&full[s], 1);      // (used in CTA 0: its own arrival; both CTAs' bytes)
            mbar_init(&empty[s], 1);     // released by CTA 0's MMAs, in both CTAs
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], 8); // (used in CTA 0: both CTAs' epilogue warps)
        }
        mbar_init(stg_full, 4);
        mbar_init(stg_free, 4);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 5) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(512));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();                    // both CTAs' barriers exist before either signals the other
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 4) {
        if (lane == 0) {
            prefetch_tmap(&tm_x);
            prefetch_tmap(&tm_w);
            int g = 0;
            bool ok = true;
            for (int t = pair; t < a.ntiles && ok; t += npairs) {
                int m, n;
                tile_mn(a, t, &m, &n);
                const int b = m / a.tiles_m_b, tm = m % a.tiles_m_b;
                const int row0 = b * a.N + tm * (2 * kPM) + (int)crank * kPM;
                for (int kb = 0; kb < ksteps; ++kb, ++g) {
                    const int s = g % kPStages;
                    if (g >= kPStages && !mbar_wait(&empty[s], ((g / kPStages) - 1) & 1, abort_flag, a.status, 80)) {
                        ok = false;
                        break;
                    }
                    uint8_t *st = sm + PLay::kOffStages + s * PLay::kStage;
                    // both CTAs' bytes complete on CTA 0's barrier, which CTA 0 arms for them
                    if (crank == 0) mbar_expect_tx(&full[s], 2 * PLay::kStage);
                    const uint32_t fb = map_rank(&full[s], 0);
                    tma_load_2d_pair(st, &tm_x, fb, kb * kPK, row0);
                    tma_load_2d_pair(st + PLay::kABytes, &tm_w, fb, kb * kPK, n * kPN + (int)crank * (kPN / 2));
                }
            }
            // no copy may still be in flight at exit: the last phase of every slot
            // has been released by the MMAs that read it (CTA 0 waited for its bytes)
            volatile int32_t no_abort = 0;
            for (int s = 0; s < kPStages; ++s) {
                const int nfill = (g - s + kPStages - 1) / kPStages;
                if (nfill > 0) mbar_wait(&empty[s], (nfill - 1) & 1, &no_abort, a.status, 81);
            }
        }
    } else if (warp == 5) {
        if (crank == 0) {
            const uint32_t idesc = idesc_bf16_f32(2 * kPM, kPN, 0, 0);
            int g = 0, it = 0;
            bool ok = true;
            for (int t = pair; t < a.ntiles && ok; t += npairs, ++it) {
                const int ab = it & 1;
                if (it >= 2 && !mbar_wait(&acc_empty[ab], ((it >> 1) - 1) & 1, abort_flag, a.status, 82)) break;
                tc_fence_after();
                for (int kb = 0; kb < ksteps; ++kb, ++g) {
                    const int s = g % kPStages;
                    if (!mbar_wait(&full[s], (g / kPStages) & 1, abort_flag, a.status, 83)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (lane == 0) {
                        const uint32_t sa = smem_u32(sm + PLay::kOffStages + s * PLay::kStage);
#pragma unroll
                        for (int kk = 0; kk < kPK / 16; ++kk) {
                            const uint64_t ad = sdesc_sw128(sa + kk * 32, 16, 1024);
                            const uint64_t bd = sdesc_sw128(sa + PLay::kABytes + kk * 32, 16, 1024);
                            umma_bf16_pair(tmem + 256 * ab, ad, bd, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
                        }
                        umma_commit_pair(&empty[s]);
                        if (kb == ksteps - 1) umma_commit_pair(&acc_full[ab]);
                    }
                    __syncwarp();
                }
            }
        }
    } else {
        // ---------------------------------------------------------------- epilogue
        const int r = threadIdx.x;     // row of this CTA's half = TMEM lane
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        const uint32_t acc_empty0[2] = {map_rank(&acc_empty[0], 0), map_rank(&acc_empty[1], 0)};
        int it = 0;
        for (int t = pair; t < a.ntiles; t += npairs, ++it) {
            const int ab = it & 1;
            int m, n;
            tile_mn(a, t, &m, &n);
            const int b = m / a.tiles_m_b, tm = m % a.tiles_m_b;
            const int tok0 = tm * (2 * kPM) + (int)crank * kPM;   // this CTA's first token of the batch
            const int nvalid = min(kPM, a.N - tok0);
            const int col0 = n * kPN;
            const int which = col0 / (a.H * a.d);               // 0: Q, 1: K, 2: V
            const int h0 = (col0 % (a.H * a.d)) / a.d;
            bool ok = mbar_wait(&acc_full[ab], (it >> 1) & 1, abort_flag, a.status, 84);
            // the staging tile is free once the previous tile's stores have read it
            // and every warp has taken its block sums from it
            if (it > 0) ok = mbar_wait(stg_free, (it - 1) & 1, abort_flag, a.status, 85) && ok;
            ok = __all_sync(0xffffffffu, ok);
            tc_fence_after();
            if (ok && nvalid > 0) {
#pragma unroll 1
                for (int cc = 0; cc < kPN / 32; ++cc) {
                    uint32_t v[32];
                    tmem_ld32(tmem + lane_base + 256 * ab + cc * 32, v);
                    tmem_ld_wait();
                    const int ct = cc * 32;                     // first tile column of the chunk
                    const int hh = ct / a.d, ch = ct % a.d, dc = ch >> 6, c0 = ch & 63;
                    const int R = r * HT + hh;
                    const uint32_t line = smem_u32(stg) + dc * (kPM * HT * 128) + R * 128;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int c16 = (c0 >> 3) + q;
                        st_shared_v4(line + ((c16 ^ (R & 7)) << 4),
                                     pack_bf16x2(__uint_as_float(v[8 * q]), __uint_as_float(v[8 * q + 1])),
                                     pack_bf16x2(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3])),
                                     pack_bf16x2(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5])),
                                     pack_bf16x2(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7])));
                    }
                }
            }
            // the accumulator is in registers / staging: release it to CTA 0's MMAs
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(acc_empty0[ab]);
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(stg_full);
            ok = mbar_wait(stg_full, it & 1, abort_flag, a.status, 86) && ok;
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            if (r == 0 && nvalid > 0) {
                const CUtensorMap *mo = which == 0 ? &tm_q : (which == 1 ? &tm_k : &tm_v);
                for (int dc = 0; dc < a.d / 64; ++dc)
                    tma_store_4d(mo, stg + dc * (kPM * HT * 128), dc * 64, h0, tok0, b);
                bulk_commit();
            }
            // block means of the rounded outputs: one thread per (block, column),
            // rows in token order, fp64
            const int blk = which == 0 ? a.Bq : 64;
            const int nblk = kPM / blk;
            const int nb_total = which == 0 ? a.nQB : a.nKB;
            float *dst = which == 0 ? a.qbar : (which == 1 ? a.kbar : a.vbar);
            for (int item = r; item < nblk * kPN && nvalid > 0; item += kPM) {
                const int j = item / kPN, ct = item % kPN;
                const int hh = ct / a.d, ch = ct % a.d, dc = ch >> 6, c = ch & 63;
                const int r0 = j * blk, r1 = min(nvalid, r0 + blk);
                if (r1 <= r0) continue;
                const uint8_t *base = stg + dc * (kPM * HT * 128);
                double sum = 0.0;
                for (int rr = r0; rr < r1; ++rr) {
                    const int R = rr * HT + hh;
                    const uint16_t bits =
                        *reinterpret_cast<const uint16_t *>(base + R * 128 + ((((c >> 3) ^ (R & 7))) << 4) + (c & 7) * 2);
                    sum = __dadd_rn(sum, (double)__uint_as_float((uint32_t)bits << 16));
                }
                const int bi = tok0 / blk + j;
                if (bi < nb_total)
                    dst[(((int64_t)b * a.H + h0 + hh) * nb_total + bi) * a.d + ch] =
                        __double2float_rn(sum / (double)(r1 - r0));
                if (which == 1 && b == 0 && hh == 0 && ch == 0 && a.count != nullptr) a.count[bi] = r1 - r0;
            }
            if (r == 0) bulk_wait_read0();
            __syncwarp();
            if (lane == 0) mbar_arrive(stg_free);
        }
        if (r == 0) bulk_wait0();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();                    // no MMA, copy or arrival of the pair is still aimed at this CTA
    if (warp == 5) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode()
{
    static EncodeTiledFn fn = nullptr;
    if (fn == nullptr) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// Row-major bf16 matrix [rows, cols]; box = 64 columns x box_rows rows.
bool map_matrix(CUtensorMap *m, const void *base, int64_t rows, int64_t cols, int box_rows)
{
    EncodeTiledFn f = encode();
    if (!f) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    cuuint32_t es[2] = {1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 [B, N, H, d] output; box = 64 channels x ht heads x 128 tokens x 1.
bool map_out(CUtensorMap *m, void *base, const bsa_params &p, int ht)
{
    EncodeTiledFn f = encode();
    if (!f) return false;
    cuuint64_t dims[4] = {(cuuint64_t)p.d, (cuuint64_t)p.H, (cuuint64_t)p.N, (cuuint64_t)p.B};
    cuuint64_t strides[3] = {(cuuint64_t)p.stride_h * 2, (cuuint64_t)p.stride_n * 2, (cuuint64_t)p.stride_b * 2};
    cuuint32_t box[4] = {64, (cuuint32_t)ht, (cuuint32_t)kPM, 1};
    cuuint32_t es[4] = {1, 1, 1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, base, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_qkv_pool(const bsa_params &p, const Dims &D, const void *x, int d_model, const void *w, void *q,
                            void *k, void *v, float *qbar, float *kbar, float *vbar, int32_t *blk_count,
                            int32_t *status, cudaStream_t st)
{
    ProdArgs a;
    a.B = D.B;
    a.N = D.N;
    a.H = D.H;
    a.d = D.d;
    a.dm = d_model;
    a.sb = p.stride_b;
    a.sn = p.stride_n;
    a.sh = p.stride_h;
    a.Bq = D.Bq;
    a.nQB = D.nQB;
    a.nKB = D.nKB;
    a.tiles_m_b = (int)ceil_div(D.N, 2 * kPM);
    a.tiles_m = a.tiles_m_b * D.B;
    a.tiles_n = 3 * D.H * D.d / kPN;
    a.ntiles = a.tiles_m * a.tiles_n;
    a.qbar = qbar;
    a.kbar = kbar;
    a.vbar = vbar;
    a.count = blk_count;
    a.status = status;
    CUtensorMap tx, tw, tq, tk, tv;
    const int ht = kPN / D.d;
    if (!map_matrix(&tx, x, (int64_t)D.B * D.N, d_model, kPM) ||
        !map_matrix(&tw, w, 3LL * D.H * D.d, d_model, kPN / 2) ||
        !map_out(&tq, q, p, ht) || !map_out(&tk, k, p, ht) || !map_out(&tv, v, p, ht)) {
        set_error("cuTensorMapEncodeTiled failed for the projection");
        return cudaErrorInvalidValue;
    }
    const size_t smem = PLay::bytes;
    cudaError_t e = cudaFuncSetAttribute(qkv_pool_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int pairs = std::max(1, std::min(a.ntiles, sm_count() / 2));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(2 * pairs));
    cfg.blockDim = dim3(kPThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    count_launch();
    return cudaLaunchKernelEx(&cfg, qkv_pool_kernel, tx, tw, tq, tk, tv, a);
}

}  // namespace bsa
