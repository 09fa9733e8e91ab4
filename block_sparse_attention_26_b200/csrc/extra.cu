// extra.cu -- extra tokens: for every query block, the E highest-scoring
// tokens outside its kept blocks ("BlockSparseAttention - ComfyUI Built-in
// Node Documentation", general inputs, extra_tokens: each query block also
// attends exactly to this many top-scoring tokens beyond its selected blocks).
//
// Token score of query block i and token j: the pooled query rounded to the
// input dtype (bf16, round to nearest even) dotted with k_j.  Ranking: score
// descending, ties to the lower token index; output in ascending token order.
// Query blocks whose rows all run dense get none (their sparse result is
// replaced anyway).
//
// Exact top-E without materialising the scores:
//   theta_kernel     one warp per row: scores of the tokens of the row's best
//                    unselected blocks (by pooled block score); their E-th
//                    largest, lowered by a safety margin, is a lower bound of
//                    the row's true E-th score (they are real candidates).
//   filter_kernel    tcgen05: S = Qt K^T for 128 query blocks x 128 tokens per
//                    tile, streamed over all tokens once.  Each row's
//                    unselected tokens are counted into 88 linear buckets from
//                    its bound up, and kept (score key, token) in token order,
//                    only from a floor that rises as the pass goes: the highest
//                    bucket already holding E counted tokens.  A token of the
//                    true top E is never below a floor, so every one of them is
//                    kept (the bucket map is monotone); about 1.5-3k tokens per
//                    row are.  Two warps share each row, one per 64-token block
//                    of a tile, and swap per-tile counts so the row's list stays
//                    in order.
//   finalize_kernel  one warp per row: the kept tokens at or above the final cut
//                    bucket (the highest holding E counted tokens), then their
//                    exact E-th largest by radix select, ties resolved by token
//                    order, compaction.
//   fallback_kernel  rows whose survivors overflowed the buffer: all candidate
//                    scores into a scratch row, radix select over the row.
#include <float.h>
#include <math.h>

#include <algorithm>

#include "bsa_device.cuh"
#include "bsa_internal.h"

namespace bsa {
namespace {

constexpr int kRowsPerCta = 128;   // query blocks per filter CTA (UMMA M)
constexpr int kTok = 128;          // tokens per filter tile (UMMA N)
constexpr int kSampleBlocks = 0;   // best unselected blocks beyond ceil(E/64) sampled for theta
constexpr int kBuckets = 88;       // pass-A histogram buckets per row
constexpr int kHistPitch = kBuckets + 1;   // words per row: a row's buckets fall in distinct banks
constexpr int kStagePitch = 33;            // words per staged row
constexpr int kLaneMax = 3;                // most set bits per row a warp walks row by row
constexpr float kSpan = 2.f;       // buckets cover [theta, theta + kSpan * (sampled max - theta)]

// Order-preserving map of a float to uint32 (larger float -> larger key).
__device__ __forceinline__ uint32_t ord_key(float f)
{
    uint32_t u = __float_as_uint(f);
    if ((u & 0x7fffffffu) == 0) u = 0;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_to_float(uint32_t k)
{
    const uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
    return __uint_as_float(u);
}

struct ExArgs {
    int B, H, N, d, nQB, nKB, nW, Bq, E, cap;
    int64_t rows;
    int64_t sb, sn, sh;                // K element strides
    const __nv_bfloat16 *k;
    const float *qbar;
    const float *S;                    // [rows, nKB] pooled block scores
    const uint32_t *bitmask;           // [rows, nW] kept blocks
    int dense_begin, dense_end;
    float *theta;                      // [rows] raw-dot lower bounds (+inf: no extras)
    float *smax;                       // [rows] largest sampled score
    float4 *cut;                       // [rows] bucket map {w, c} and the final cut, as y of fma_rz(x, w, c)
    unsigned long long *buf;           // [rows, cap] (ord key << 32 | token)
    int32_t *cnt;                      // [rows] survivors (may exceed cap)
    int32_t *ovf;                      // [0]: count, [1..]: overflowed rows
    int32_t *extra_idx;                // [rows, E]
    int32_t *extra_count;              // [rows]
    uint32_t *scratch;                 // [gridDim, N] fallback keys
    int32_t *status;
};

__device__ __forceinline__ bool row_all_dense(const ExArgs &a, int64_t r)
{
    const int i = (int)(r % a.nQB);
    const int lo = i * a.Bq, hi = min(a.N, lo + a.Bq);
    return lo >= a.dense_begin && hi <= a.dense_end;
}

__device__ __forceinline__ bool is_kept(const uint32_t *bm, int blk) { return (bm[blk >> 5] >> (blk & 31)) & 1u; }

// Exact k-th largest of n uint32 keys (k >= 1), warp-wide: returns the key v_k and,
// in *need, how many keys equal to v_k belong to the top k.  hist: 256 words.
template <typename KeyAt>
__device__ uint32_t warp_kth(KeyAt key_at, int n, int k, uint32_t *hist, int *need)
{
    const int lane = threadIdx.x & 31;
    uint32_t prefix = 0, pmask = 0;
    int remaining = k;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int t = lane; t < 256; t += 32) hist[t] = 0;
        __syncwarp();
        for (int j = lane; j < n; j += 32) {
            const uint32_t u = key_at(j);
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
    *need = remaining;
    return prefix;
}

// ------------------------------------------------------------------ theta

__global__ void __launch_bounds__(256) theta_kernel(ExArgs a)
{
    __shared__ float qs[8][128];
    __shared__ uint32_t hist[8][256];
    __shared__ uint32_t keys[8][512];
    __shared__ int blks[8][16];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t r = (int64_t)blockIdx.x * 8 + warp;
    if (r >= a.rows) return;
    if (row_all_dense(a, r)) {
        if (lane == 0) {
            a.theta[r] = INFINITY;
            a.smax[r] = INFINITY;
        }
        return;
    }
    const int bh = (int)(r / a.nQB);
    const int b = bh / a.H, h = bh % a.H;
    const uint32_t *bm = a.bitmask + r * a.nW;
    const float *srow = a.S + r * a.nKB;
    for (int c = lane; c < a.d; c += 32) qs[warp][c] = __bfloat162float(__float2bfloat16_rn(a.qbar[r * a.d + c]));
    // Good unselected blocks by pooled score until the sample holds E tokens (a
    // partial last block holds fewer than 64), at most 8 blocks = 512 tokens: one
    // scan in which each lane keeps its two best blocks, then picks among the
    // lanes' candidates.  Any sample of real candidates gives a valid bound; a
    // better sample gives a tighter one.
    float b1 = -INFINITY, b2 = -INFINITY;
    int i1 = -1, i2 = -1;
    for (int j = lane; j < a.nKB; j += 32) {
        if (is_kept(bm, j)) continue;
        const float v = srow[j];
        if (i1 < 0 || v > b1) {
            b2 = b1;
            i2 = i1;
            b1 = v;
            i1 = j;
        } else if (i2 < 0 || v > b2) {
            b2 = v;
            i2 = j;
        }
    }
    int got = 0, ntok = 0;
    for (int t = 0; t < 8 && ntok < a.E + 64 * kSampleBlocks; ++t) {
        float best = i1 >= 0 ? b1 : -INFINITY;
        int bi = i1, bl = i1 >= 0 ? lane : 32;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ob = __shfl_xor_sync(0xffffffffu, best, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            const int ol = __shfl_xor_sync(0xffffffffu, bl, o);
            if (oi >= 0 && (bi < 0 || ob > best || (ob == best && ol < bl))) {
                best = ob;
                bi = oi;
                bl = ol;
            }
        }
        if (bi < 0) break;
        if (lane == bl) {   // the winning lane moves to its second candidate
            b1 = b2;
            i1 = i2;
            i2 = -1;
        }
        if (lane == 0) blks[warp][got] = bi;
        __syncwarp();
        ++got;
        ntok += min(64, a.N - bi * 64);
    }
    // token scores of the sampled blocks (raw dot products)
    int n = 0;
    for (int u = 0; u < got; ++u) {
        const int blk = blks[warp][u];
        const int t0 = blk * 64, t1 = min(a.N, t0 + 64);
        for (int t = t0 + lane; t < t1; t += 32) {
            const __nv_bfloat16 *kr = a.k + (int64_t)b * a.sb + (int64_t)t * a.sn + (int64_t)h * a.sh;
            float dot = 0.f;
            for (int c = 0; c < a.d; c += 8) {
                const uint4 w = *reinterpret_cast<const uint4 *>(kr + c);
                const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    dot = fmaf(qs[warp][c + 2 * e], __uint_as_float(ww[e] << 16), dot);
                    dot = fmaf(qs[warp][c + 2 * e + 1], __uint_as_float(ww[e] & 0xffff0000u), dot);
                }
            }
            keys[warp][n + (t - t0)] = ord_key(dot);
        }
        n += t1 - t0;
    }
    __syncwarp();
    float th = -INFINITY;
    uint32_t mx = 0;
    for (int j = lane; j < n; j += 32) mx = max(mx, keys[warp][j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (n >= a.E) {
        int need;
        const uint32_t *kk = keys[warp];
        const uint32_t vk = warp_kth([&](int j) { return kk[j]; }, n, a.E, hist[warp], &need);
        const float v = key_to_float(vk);
        th = v - (1e-3f * fabsf(v) + 1e-3f);   // covers fp32 accumulation-order differences
    }
    if (lane == 0) {
        a.theta[r] = th;
        a.smax[r] = n > 0 ? key_to_float(mx) : -INFINITY;
    }
}

// ------------------------------------------------------------------ filter

__device__ __forceinline__ void red_shared_add1(uint32_t addr)
{
    asm volatile("red.shared.add.u32 [%0], 1;" ::"r"(addr) : "memory");
}

template <int D>
struct FLay {
    static constexpr int kFS = D == 128 ? 3 : 4;            // K ring depth
    static constexpr int kQBytes = kRowsPerCta * D * 2;
    static constexpr int kKBytes = kTok * D * 2;
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kQBytes;
    static constexpr int kOffBar = kOffK + kFS * kKBytes;   // k_full[FS], k_empty[FS], s_full[2], s_free[2], done
    static constexpr int kOffMisc = kOffBar + (2 * kFS + 5) * 8;
    static constexpr int kOffHist = kOffMisc + 16;                              // [128 rows][kHistPitch] u32
    static constexpr int kOffPar = kOffHist + kRowsPerCta * kHistPitch * 4;     // [128 rows] {w, c}
    static constexpr int kOffPair = kOffPar + kRowsPerCta * 8;                   // [2][2 groups][128 rows] i32
    static constexpr int kOffStage = kOffPair + 4 * kRowsPerCta * 4;            // [8 warps][32 rows][33] u32
    static constexpr int kOffBase = kOffStage + 8 * 32 * kStagePitch * 4;       // [8 warps][32] i32
    static constexpr int kOffList = kOffBase + 8 * 32 * 4;                      // [8 warps][1024] u16
    static constexpr size_t bytes = (size_t)kOffList + 8 * 1024 * 2 + 1024;
    static_assert(bytes <= 232448, "filter tile exceeds the per-block shared memory limit");
};


// Warps 0-7 read the scores: warp w takes the rows of TMEM lane quarter w & 3
// and, of each 128-token tile, key block 2t + (w >> 2).  Warp 8 loads K tiles,
// warp 9 issues the MMAs and owns TMEM.
template <int D>
__global__ void __launch_bounds__(320, 1) filter_kernel(const __grid_constant__ CUtensorMap tm_k, ExArgs a)
{
    using L = FLay<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.y;
    const int b = bh / a.H, h = bh % a.H;
    const int i0 = blockIdx.x * kRowsPerCta;
    const int ntiles = (a.N + kTok - 1) / kTok;
    // key tiles in the order t_first, t_first + 1, ..., wrapping: t_first sits a few
    // frames' worth of tiles before the CTA's query rows, where scores run highest
    const int t_first = max(0, min(ntiles - 1, (int)(((int64_t)(i0 + kRowsPerCta / 2) * a.Bq) / kTok)) - 32);
    auto tile_at = [&](int t) { const int u = t_first + t; return u >= ntiles ? u - ntiles : u; };
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::kOffBar);
    uint64_t *k_full = bars, *k_empty = bars + L::kFS, *s_full = bars + 2 * L::kFS, *s_free = s_full + 2,
             *bar_done = s_full + 4;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + L::kOffMisc);
    volatile int32_t *abort_flag = reinterpret_cast<volatile int32_t *>(sm + L::kOffMisc + 4);
    uint32_t *hist = reinterpret_cast<uint32_t *>(sm + L::kOffHist);   // [row][kHistPitch]
    float2 *par = reinterpret_cast<float2 *>(sm + L::kOffPar);         // [row] bucket map

    // Per-row bucket map.  y = fma_rz(x, w, 2^23 + 1 - th w) clamped to 2^23 +
    // kBuckets - 1, so that for x >= th the bits of y are 0x4B000000 + 1 +
    // trunc((x - th) w) up to rounding (bucket 0 takes the rounding slack just
    // below th).  w spreads the buckets over [th, th + kSpan (smax - th)]: the
    // sampled maximum need not bound the row, so the range reaches well past
    // it, and the last bucket is open-ended.  y is monotone in x, which is all
    // exactness needs.  th = +inf
    // marks rows without extra tokens; -FLT_MAX stands in for "no bound".
    const int r = threadIdx.x & (kRowsPerCta - 1);
    const int64_t row = (int64_t)bh * a.nQB + min(i0 + r, a.nQB - 1);
    const bool live = i0 + r < a.nQB;
    const float th0 = live ? a.theta[row] : INFINITY;
    const float th = fmaxf(th0, -FLT_MAX);
    const float hi = live ? a.smax[row] : 0.f;
    const float inv_w = (hi > th && hi < INFINITY) ? (float)kBuckets / (kSpan * (hi - th)) : 0.f;
    const float cw = 8388609.f - th * inv_w;

    if (threadIdx.x == 0) {
        for (int s = 0; s < L::kFS; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&s_free[i], 8);
        }
        mbar_init(bar_done, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 9) {
        tmem_alloc(tmem_slot, 256);
        tmem_relinquish();
    }
    if (warp < 4) {
        // rounded pooled queries of the 128 rows -> the A operand (128-byte swizzle)
        const int i = i0 + r;
        const float *q = a.qbar + row * D;
        const uint32_t base = smem_u32(sm + L::kOffQ) + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll 1
        for (int ch = 0; ch < D / 8; ++ch) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) w[e] = i < a.nQB ? pack_bf16x2(q[8 * ch + 2 * e], q[8 * ch + 2 * e + 1]) : 0u;
            const int dc = ch >> 3, c16 = ch & 7;
            st_shared_v4(base + dc * (kRowsPerCta * 128) + ((c16 ^ (r & 7)) << 4), w[0], w[1], w[2], w[3]);
        }
        fence_async_smem();
        for (int k = 0; k < kBuckets; ++k) hist[r * kHistPitch + k] = 0;
        par[r] = make_float2(inv_w, cw);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 8) {
        if (lane == 0) {
            prefetch_tmap(&tm_k);
            for (int t = 0; t < ntiles; ++t) {
                const int s = t % L::kFS;
                if (t >= L::kFS && !mbar_wait(&k_empty[s], ((t / L::kFS) - 1) & 1, abort_flag, a.status, 40)) break;
                mbar_expect_tx(&k_full[s], L::kKBytes);
                uint8_t *dst = sm + L::kOffK + s * L::kKBytes;
                for (int half = 0; half < 2; ++half)
                    for (int dc = 0; dc < D / 64; ++dc)
                        tma_load_4d(dst + dc * (kTok * 128) + half * (64 * 128), &tm_k, &k_full[s], dc * 64, h,
                                    tile_at(t) * kTok + half * 64, b);
            }
            volatile int32_t no_abort = 0;
            for (int s = 0; s < L::kFS; ++s) {
                const int n = (ntiles - s + L::kFS - 1) / L::kFS;
                if (n > 0) mbar_wait(&k_full[s], (n - 1) & 1, &no_abort, a.status, 41);
            }
        }
    } else if (warp == 9) {
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16_f32(kRowsPerCta, kTok, 0, 0);
            const uint32_t q_addr = smem_u32(sm + L::kOffQ), k_addr = smem_u32(sm + L::kOffK);
            for (int t = 0; t < ntiles; ++t) {
                const int s = t % L::kFS, sb = t & 1;
                if (!mbar_wait(&k_full[s], (t / L::kFS) & 1, abort_flag, a.status, 42)) break;
                if (t >= 2 && !mbar_wait(&s_free[sb], ((t >> 1) - 1) & 1, abort_flag, a.status, 43)) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t ad = sdesc_sw128(q_addr + (kk >> 2) * (kRowsPerCta * 128) + (kk & 3) * 32, 16, 1024);
                    const uint64_t bd =
                        sdesc_sw128(k_addr + s * L::kKBytes + (kk >> 2) * (kTok * 128) + (kk & 3) * 32, 16, 1024);
                    umma_bf16(tmem + 128 * sb, ad, bd, idesc, kk > 0 ? 1u : 0u);
                }
                umma_commit(&s_full[sb]);
                umma_commit(&k_empty[s]);
            }
            umma_commit(bar_done);
            volatile int32_t no_abort = 0;
            mbar_wait(bar_done, 0, &no_abort, a.status, 44);
        }
    } else {
        const int g = warp >> 2, sub = warp & 3;
        const bool active = th0 < INFINITY;
        const float ytop = 8388608.f + (float)(kBuckets - 1);
        int32_t *pair = reinterpret_cast<int32_t *>(sm + L::kOffPair);
        uint32_t *stage = reinterpret_cast<uint32_t *>(sm + L::kOffStage) + warp * 32 * kStagePitch;
        int32_t *base = reinterpret_cast<int32_t *>(sm + L::kOffBase) + warp * 32;
        uint16_t *list = reinterpret_cast<uint16_t *>(sm + L::kOffList) + warp * 1024;
        unsigned long long *out = a.buf + row * a.cap;
        // hist + 4 (kHistPitch r + bucket) = hbase0 + 4 kHistPitch r + 4 bits(y), wrapping mod 2^32
        const uint32_t hbase0 = smem_u32(hist) - 4u * 0x4B000000u;
        const uint32_t hrow = hbase0 + 4u * (uint32_t)(kHistPitch * r);
        // Tokens are counted and kept only from the floor up.  The floor is the
        // highest bucket already holding E counted tokens at or above it; it only
        // rises, so the true top E are all at or above every floor taken, and
        // every token kept scores at least the floor of its time.
        int floor_k = 0;
        auto raise_floor = [&]() {
            uint32_t acc = 0;
            for (int k0 = kBuckets - 8; k0 + 7 > floor_k; k0 -= 8) {   // eight loads in flight
                uint32_t h8[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) h8[j] = hist[r * kHistPitch + k0 + j];
#pragma unroll
                for (int j = 7; j >= 0; --j) {
                    acc += h8[j];
                    if (acc >= (uint32_t)a.E && k0 + j > floor_k) {
                        floor_k = k0 + j;
                        return;
                    }
                }
            }
        };
        const uint32_t *bm = a.bitmask + row * a.nW;
        int cnt = 0;   // survivors of this row so far (both warps of the row agree)
        const uint32_t lane_base = (uint32_t)(sub * 32) << 16;
        uint32_t word = bm[min((2 * tile_at(0) + g) >> 5, a.nW - 1)];
        for (int t = 0; t < ntiles; ++t) {
            const int sb = t & 1;
            const int blk = 2 * tile_at(t) + g;
            // bitmask word of the next tile's block, fetched a tile early
            const uint32_t word_next = bm[min((2 * tile_at(t + 1 < ntiles ? t + 1 : t) + g) >> 5, a.nW - 1)];
            // After an abort every wait fails at once: the loop still runs to the
            // end with no work, so both warps of a row meet at every pair barrier.
            const bool go = __all_sync(0xffffffffu, mbar_wait(&s_full[sb], (t >> 1) & 1, abort_flag, a.status, 45));
            tc_fence_after();
            uint32_t v[64];
            if (go) {
                tmem_ld32(tmem + lane_base + 128 * sb + 64 * g, *reinterpret_cast<uint32_t(*)[32]>(v));
                tmem_ld32(tmem + lane_base + 128 * sb + 64 * g + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
                tmem_ld_wait();
            } else {
#pragma unroll
                for (int e = 0; e < 64; ++e) v[e] = 0u;
            }
            const int tok0 = blk * 64;
            const bool use = go && active && blk < a.nKB && !((word >> (blk & 31)) & 1u);
            const int nvalid = max(0, min(64, a.N - tok0));
            const float ythr = 8388608.f + (float)floor_k;   // the floor in bucket space
            uint32_t m0 = 0, m1 = 0;
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const float y0 = __fmaf_rz(__uint_as_float(v[e]), inv_w, cw);
                const float y1 = __fmaf_rz(__uint_as_float(v[32 + e]), inv_w, cw);
                m0 |= (y0 >= ythr) ? (1u << e) : 0u;
                m1 |= (y1 >= ythr) ? (1u << e) : 0u;
            }
            if (!use) m0 = m1 = 0;
            if (nvalid < 64) {   // tokens past the end
                m0 &= nvalid >= 32 ? 0xffffffffu : (1u << nvalid) - 1u;
                m1 &= nvalid <= 32 ? 0u : (1u << (nvalid - 32)) - 1u;
            }
            const int cmine = __popc(m0) + __popc(m1);
            int out_at = cnt;   // this row's first output slot for this block
            {
                // the row's other warp holds the tile's other block: swap counts so
                // that block 2t's survivors precede block 2t + 1's
                pair[((t & 1) * 2 + g) * kRowsPerCta + r] = cmine;
                named_bar_sync(2 + sub, 64);
                const int cother = pair[((t & 1) * 2 + (g ^ 1)) * kRowsPerCta + r];
                if (g == 1) out_at += cother;
                cnt += cmine + cother;
            }
            // Set bits, 32 values of a row at a time.  With few bits per row each
            // row's thread walks its own, taking the value of bit e out of the
            // registers through a select tree on e.  With more, the whole warp
            // takes them 32 at a time: each row with bits stages its values and
            // lists (lane, bit) entries at its exclusive offset, then every lane
            // handles one entry per round.
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const uint32_t *vh = v + 32 * hf;
                const uint32_t m = hf ? m1 : m0;
                const int c = __popc(m);
                const int cmax = __reduce_max_sync(0xffffffffu, c);
                if (cmax == 0) continue;
                if (cmax <= kLaneMax) {
                    for (uint32_t mm = m; mm != 0u; mm &= mm - 1u) {
                        const int e = __ffs(mm) - 1;
                        const uint32_t x = select32(vh, e);
                        const float y = fminf(__fmaf_rz(__uint_as_float(x), inv_w, cw), ytop);
                        red_shared_add1(hrow + 4u * (uint32_t)__float_as_int(y));
                        const int pos = out_at + (int)__popc(m & ((1u << e) - 1u));
                        if (pos < a.cap)
                            out[pos] = ((unsigned long long)ord_key(__uint_as_float(x)) << 32) |
                                       (uint32_t)(tok0 + 32 * hf + e);
                    }
                } else {
                    int incl = c;
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) {
                        const int y = __shfl_up_sync(0xffffffffu, incl, o);
                        if (lane >= o) incl += y;
                    }
                    const int total = __shfl_sync(0xffffffffu, incl, 31);
                    if (m != 0u) {
#pragma unroll
                        for (int e = 0; e < 32; ++e) stage[lane * kStagePitch + e] = vh[e];
                        int j = incl - c;
                        base[lane] = out_at - j;   // output slot = base + list index
                        for (uint32_t mm = m; mm != 0u; mm &= mm - 1u)
                            list[j++] = (uint16_t)((lane << 5) | (__ffs(mm) - 1));
                    }
                    __syncwarp();
                    for (int i0l = 0; i0l < total; i0l += 32) {
                        const int idx = i0l + lane;
                        if (idx < total) {
                            const uint32_t ent = list[idx];
                            const int e = (int)(ent & 31u), o = (int)(ent >> 5);
                            const int rr = sub * 32 + o;
                            const uint32_t x = stage[o * kStagePitch + e];
                            const float2 wc = par[rr];
                            const float y = fminf(__fmaf_rz(__uint_as_float(x), wc.x, wc.y), ytop);
                            red_shared_add1(hbase0 + 4u * (uint32_t)(kHistPitch * rr) + 4u * (uint32_t)__float_as_int(y));
                            const int pos = base[o] + idx;
                            if (pos < a.cap) {
                                const int64_t row_o = (int64_t)bh * a.nQB + min(i0 + rr, a.nQB - 1);
                                a.buf[row_o * a.cap + pos] = ((unsigned long long)ord_key(__uint_as_float(x)) << 32) |
                                                             (uint32_t)(tok0 + 32 * hf + e);
                            }
                        }
                    }
                    __syncwarp();
                }
                out_at += c;
            }
            word = word_next;
            if (t < 32 || (t & 7) == 7) raise_floor();   // every tile while it climbs
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_free[sb]);
        }
        named_bar_sync(1, 256);   // every count of the CTA is in
        if (g == 0 && live) {
            a.cnt[row] = cnt;
            // the final cut: the highest bucket with at least E counted tokens at or
            // above it; no token below it can be in the top E
            uint32_t acc = 0;
            int kcut = -1;
            for (int k = kBuckets - 1; k >= 0; --k) {
                acc += hist[r * kHistPitch + k];
                if (acc >= (uint32_t)a.E) {
                    kcut = k;
                    break;
                }
            }
            a.cut[row] = make_float4(inv_w, cw, kcut < 0 ? -INFINITY : 8388608.f + (float)kcut, 0.f);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// ------------------------------------------------------------------ finalize

__global__ void __launch_bounds__(256) finalize_kernel(ExArgs a)
{
    __shared__ uint32_t hist[8][256];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t r = (int64_t)blockIdx.x * 8 + warp;
    if (r >= a.rows) return;
    int32_t *out = a.extra_idx + r * a.E;
    const int cnt = row_all_dense(a, r) ? 0 : a.cnt[r];
    if (cnt > a.cap) {
        if (lane == 0) {
            const int slot = atomicAdd(&a.ovf[0], 1);
            a.ovf[1 + slot] = (int32_t)r;
        }
        return;
    }
    unsigned long long *buf = a.buf + r * a.cap;
    const uint32_t lt = (1u << lane) - 1u;
    int n = cnt;
    const float4 cu = a.cut[r];
    if (cnt > a.E && cu.z > -INFINITY) {
        // keep the entries at or above the final cut bucket (the filter's own bucket
        // map, recomputed from the score), in place and in order
        int wpos = 0;
        for (int j0 = 0; j0 < cnt; j0 += 32) {
            const int j = j0 + lane;
            const unsigned long long e = j < cnt ? buf[j] : 0ull;
            const float y = __fmaf_rz(key_to_float((uint32_t)(e >> 32)), cu.x, cu.y);
            const bool keep = j < cnt && y >= cu.z;
            const uint32_t bal = __ballot_sync(0xffffffffu, keep);
            __syncwarp();
            if (keep) buf[wpos + __popc(bal & lt)] = e;
            wpos += __popc(bal);
        }
        __syncwarp();
        n = wpos;
    }
    uint32_t vk = 0;
    int need = 0;
    if (n > a.E) vk = warp_kth([&](int j) { return (uint32_t)(buf[j] >> 32); }, n, a.E, hist[warp], &need);
    // the survivors are two ascending token runs (the filter wraps around the key
    // tiles): the second run starts at the one place where the token decreases
    int split = 0;
    for (int j0 = 1; j0 < n && split == 0; j0 += 32) {
        const int j = j0 + lane;
        const bool down = j < n && (uint32_t)buf[j] < (uint32_t)buf[j - 1];
        const uint32_t dm = __ballot_sync(0xffffffffu, down);
        if (dm) split = j0 + __ffs(dm) - 1;
    }
    // in ascending token order: keep key > v_k, and the first `need` equal ones
    int taken = 0, eq_taken = 0;
    for (int j0 = 0; j0 < n; j0 += 32) {
        const int i = j0 + lane;
        const bool valid = i < n;
        const int j = i + split < n ? i + split : i + split - n;
        const unsigned long long e = valid ? buf[j] : 0ull;
        const uint32_t key = (uint32_t)(e >> 32);
        bool keep;
        if (n <= a.E) {
            keep = valid;
        } else {
            const bool eq = valid && key == vk;
            const uint32_t eqm = __ballot_sync(0xffffffffu, eq);
            keep = valid && (key > vk || (eq && eq_taken + __popc(eqm & lt) < need));
            eq_taken += __popc(eqm);
        }
        const uint32_t km = __ballot_sync(0xffffffffu, keep);
        if (keep) out[taken + __popc(km & lt)] = (int32_t)(uint32_t)e;
        taken += __popc(km);
    }
    for (int j = taken + lane; j < a.E; j += 32) out[j] = -1;
    if (lane == 0) a.extra_count[r] = taken;
}

// ------------------------------------------------------------------ fallback

__global__ void __launch_bounds__(256) fallback_kernel(ExArgs a)
{
    __shared__ float qs[128];
    __shared__ uint32_t hist[256];
    __shared__ int s_digit, s_above, s_row;
    __shared__ int wsum[8];
    uint32_t *keys = a.scratch + (int64_t)blockIdx.x * a.N;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int item = blockIdx.x;; item += gridDim.x) {
        __syncthreads();
        if (item >= a.ovf[0]) break;
        if (tid == 0) s_row = a.ovf[1 + item];
        __syncthreads();
        const int64_t r = s_row;
        const int bh = (int)(r / a.nQB);
        const int b = bh / a.H, h = bh % a.H;
        const uint32_t *bm = a.bitmask + r * a.nW;
        for (int c = tid; c < a.d; c += blockDim.x)
            qs[c] = __bfloat162float(__float2bfloat16_rn(a.qbar[r * a.d + c]));
        __syncthreads();
        int ncand = 0;
        for (int t = tid; t < a.N; t += blockDim.x) {
            uint32_t key = 0;            // below every real score: never selected
            if (!is_kept(bm, t >> 6)) {
                const __nv_bfloat16 *kr = a.k + (int64_t)b * a.sb + (int64_t)t * a.sn + (int64_t)h * a.sh;
                float dot = 0.f;
                for (int c = 0; c < a.d; c += 8) {
                    const uint4 w = *reinterpret_cast<const uint4 *>(kr + c);
                    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        dot = fmaf(qs[c + 2 * e], __uint_as_float(ww[e] << 16), dot);
                        dot = fmaf(qs[c + 2 * e + 1], __uint_as_float(ww[e] & 0xffff0000u), dot);
                    }
                }
                key = max(ord_key(dot), 1u);
                ++ncand;
            }
            keys[t] = key;
        }
        // candidates in the row
        for (int o = 16; o > 0; o >>= 1) ncand += __shfl_xor_sync(0xffffffffu, ncand, o);
        if (lane == 0) wsum[warp] = ncand;
        __syncthreads();
        int total = 0;
        for (int w = 0; w < 8; ++w) total += wsum[w];
        const int k = min(a.E, total);
        // exact k-th largest key by 8-bit radix passes over the row
        uint32_t prefix = 0, pmask = 0;
        int remaining = k;
        if (k > 0) {
            for (int shift = 24; shift >= 0; shift -= 8) {
                for (int t = tid; t < 256; t += blockDim.x) hist[t] = 0;
                __syncthreads();
                for (int t = tid; t < a.N; t += blockDim.x) {
                    const uint32_t u = keys[t];
                    if (u != 0 && (u & pmask) == prefix) atomicAdd(&hist[(u >> shift) & 255u], 1u);
                }
                __syncthreads();
                if (tid == 0) {
                    int acc = 0;
                    for (int bin = 255; bin >= 0; --bin) {
                        const int c = (int)hist[bin];
                        if (acc + c >= remaining) {
                            s_digit = bin;
                            s_above = acc;
                            break;
                        }
                        acc += c;
                    }
                }
                __syncthreads();
                remaining -= s_above;
                prefix |= (uint32_t)s_digit << shift;
                pmask |= 0xFFu << shift;
            }
        }
        const uint32_t vk = prefix;
        // ascending compaction: keys above v_k, then the first `remaining` equal ones
        int32_t *out = a.extra_idx + r * a.E;
        int taken = 0, eq_taken = 0;
        const uint32_t lt = (1u << lane) - 1u;
        for (int t0 = 0; t0 < a.N && k > 0; t0 += blockDim.x) {
            const int t = t0 + tid;
            const uint32_t u = t < a.N ? keys[t] : 0u;
            const bool eq = u != 0 && u == vk;
            const uint32_t eqm = __ballot_sync(0xffffffffu, eq);
            if (lane == 0) wsum[warp] = __popc(eqm);
            __syncthreads();
            int eq_before = eq_taken;
            for (int w = 0; w < warp; ++w) eq_before += wsum[w];
            int eq_all = 0;
            for (int w = 0; w < 8; ++w) eq_all += wsum[w];
            const bool keep = u != 0 && (u > vk || (eq && eq_before + __popc(eqm & lt) < remaining));
            __syncthreads();
            const uint32_t km = __ballot_sync(0xffffffffu, keep);
            if (lane == 0) wsum[warp] = __popc(km);
            __syncthreads();
            int before = taken;
            for (int w = 0; w < warp; ++w) before += wsum[w];
            int all = 0;
            for (int w = 0; w < 8; ++w) all += wsum[w];
            if (keep) out[before + __popc(km & lt)] = t;
            taken += all;
            eq_taken += eq_all;
            __syncthreads();
        }
        for (int j = taken + tid; j < a.E; j += blockDim.x) out[j] = -1;
        if (tid == 0) a.extra_count[r] = taken;
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

bool make_k_map(CUtensorMap *m, const void *base, const Dims &D, int64_t sb, int64_t sn, int64_t sh)
{
    static EncodeTiledFn fn = nullptr;
    if (fn == nullptr) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    if (!fn) return false;
    cuuint64_t dims[4] = {(cuuint64_t)D.d, (cuuint64_t)D.H, (cuuint64_t)D.N, (cuuint64_t)D.B};
    cuuint64_t strides[3] = {(cuuint64_t)sh * 2, (cuuint64_t)sn * 2, (cuuint64_t)sb * 2};
    cuuint32_t box[4] = {64, 1, 64, 1};
    cuuint32_t es[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
cudaError_t launch_filter(dim3 grid, const CUtensorMap &tm, const ExArgs &a, cudaStream_t st)
{
    const int bytes = (int)FLay<D>::bytes;
    cudaError_t e = cudaFuncSetAttribute(filter_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    count_launch();
    filter_kernel<D><<<grid, 320, bytes, st>>>(tm, a);
    return cudaGetLastError();
}

}  // namespace

int64_t extra_buffer_capacity() { return 4096; }

cudaError_t launch_extra(const bsa_params &p, const Dims &D, const float *qbar, const void *k,
                         int32_t *extra_idx, int32_t *extra_count, char *ws, const WsLayout &L, cudaStream_t st)
{
    ExArgs a;
    a.B = D.B;
    a.H = D.H;
    a.N = D.N;
    a.d = D.d;
    a.nQB = D.nQB;
    a.nKB = D.nKB;
    a.nW = D.nW;
    a.Bq = D.Bq;
    a.E = D.E;
    a.cap = (int)extra_buffer_capacity();
    a.rows = D.rows;
    a.sb = p.stride_b;
    a.sn = p.stride_n;
    a.sh = p.stride_h;
    a.k = static_cast<const __nv_bfloat16 *>(k);
    a.qbar = qbar;
    a.S = reinterpret_cast<const float *>(ws + L.scores);
    a.bitmask = reinterpret_cast<const uint32_t *>(ws + L.bitmask);
    a.dense_begin = p.dense_row_begin;
    a.dense_end = p.dense_row_end;
    a.theta = reinterpret_cast<float *>(ws + L.ex_theta);
    a.smax = reinterpret_cast<float *>(ws + L.ex_smax);
    a.cut = reinterpret_cast<float4 *>(ws + L.ex_cut);
    a.buf = reinterpret_cast<unsigned long long *>(ws + L.ex_buf);
    a.cnt = reinterpret_cast<int32_t *>(ws + L.ex_cnt);
    a.ovf = reinterpret_cast<int32_t *>(ws + L.ex_ovf);
    a.extra_idx = extra_idx;
    a.extra_count = extra_count;
    a.scratch = reinterpret_cast<uint32_t *>(ws + L.ex_scratch);
    a.status = reinterpret_cast<int32_t *>(ws + L.status);

    cudaError_t e = cudaMemsetAsync(a.ovf, 0, sizeof(int32_t), st);
    if (e != cudaSuccess) return e;
    const unsigned g8 = (unsigned)ceil_div(D.rows, 8);
    count_launch();
    theta_kernel<<<g8, 256, 0, st>>>(a);
    CUtensorMap tm;
    if (!make_k_map(&tm, k, D, p.stride_b, p.stride_n, p.stride_h)) {
        set_error("cuTensorMapEncodeTiled failed for the extra-token scorer");
        return cudaErrorInvalidValue;
    }
    dim3 grid((unsigned)ceil_div(D.nQB, kRowsPerCta), (unsigned)(D.B * D.H));
    if (D.d == 64) {
        e = launch_filter<64>(grid, tm, a, st);
    } else {
        e = launch_filter<128>(grid, tm, a, st);
    }
    if (e != cudaSuccess) return e;
    count_launch();
    finalize_kernel<<<g8, 256, 0, st>>>(a);
    count_launch();
    fallback_kernel<<<(unsigned)fallback_ctas(), 256, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace bsa
