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
//                    tile, streamed over all tokens; each row's thread keeps
//                    the candidate tokens scoring >= its bound, in token order.
//   finalize_kernel  one warp per row: exact E-th largest of the survivors by
//                    radix select, ties resolved by token order, compaction.
//   fallback_kernel  rows whose survivors overflowed the buffer: all candidate
//                    scores into a scratch row, radix select over the row.
#include <math.h>

#include <algorithm>

#include "bsa_device.cuh"
#include "bsa_internal.h"

namespace bsa {
namespace {

constexpr int kRowsPerCta = 128;   // query blocks per filter CTA (UMMA M)
constexpr int kTok = 128;          // tokens per filter tile (UMMA N)
constexpr int kFS = 4;             // K ring depth of the filter kernel
constexpr int kSampleBlocks = 4;   // best unselected blocks beyond ceil(E/64) sampled for theta

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
        if (lane == 0) a.theta[r] = INFINITY;
        return;
    }
    const int bh = (int)(r / a.nQB);
    const int b = bh / a.H, h = bh % a.H;
    const uint32_t *bm = a.bitmask + r * a.nW;
    const float *srow = a.S + r * a.nKB;
    for (int c = lane; c < a.d; c += 32) qs[warp][c] = __bfloat162float(__float2bfloat16_rn(a.qbar[r * a.d + c]));
    // best unselected blocks by pooled score (m rounds of warp argmax)
    const int m = min(8, (a.E + 63) / 64 + kSampleBlocks);   // at most 512 sampled tokens
    int got = 0;
    for (int t = 0; t < m; ++t) {
        float best = -INFINITY;
        int bi = -1;
        for (int j = lane; j < a.nKB; j += 32) {
            if (is_kept(bm, j)) continue;
            bool taken = false;
            for (int u = 0; u < got; ++u) taken |= blks[warp][u] == j;
            if (taken) continue;
            const float v = srow[j];
            if (bi < 0 || v > best || (v == best && j < bi)) {
                best = v;
                bi = j;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ob = __shfl_xor_sync(0xffffffffu, best, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (oi >= 0 && (bi < 0 || ob > best || (ob == best && oi < bi))) {
                best = ob;
                bi = oi;
            }
        }
        if (bi < 0) break;
        if (lane == 0) blks[warp][got] = bi;
        __syncwarp();
        ++got;
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
    if (n >= a.E) {
        int need;
        const uint32_t *kk = keys[warp];
        const uint32_t vk = warp_kth([&](int j) { return kk[j]; }, n, a.E, hist[warp], &need);
        const float v = key_to_float(vk);
        th = v - (1e-3f * fabsf(v) + 1e-3f);   // covers fp32 accumulation-order differences
    }
    if (lane == 0) a.theta[r] = th;
}

// ------------------------------------------------------------------ filter

template <int D>
struct FLay {
    static constexpr int kQBytes = kRowsPerCta * D * 2;
    static constexpr int kKBytes = kTok * D * 2;
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kQBytes;
    static constexpr int kOffBar = kOffK + kFS * kKBytes;   // k_full[FS], k_empty[FS], s_full[2], s_free[2], done
    static constexpr int kOffMisc = kOffBar + (2 * kFS + 5) * 8;
    static constexpr size_t bytes = (size_t)kOffMisc + 16 + 1024;
};

template <int D>
__global__ void __launch_bounds__(192, 1) filter_kernel(const __grid_constant__ CUtensorMap tm_k, ExArgs a)
{
    using L = FLay<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.y;
    const int b = bh / a.H, h = bh % a.H;
    const int i0 = blockIdx.x * kRowsPerCta;
    const int ntiles = (a.N + kTok - 1) / kTok;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::kOffBar);
    uint64_t *k_full = bars, *k_empty = bars + kFS, *s_full = bars + 2 * kFS, *s_free = s_full + 2,
             *bar_done = s_full + 4;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + L::kOffMisc);
    volatile int32_t *abort_flag = reinterpret_cast<volatile int32_t *>(sm + L::kOffMisc + 4);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kFS; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&s_free[i], 4);
        }
        mbar_init(bar_done, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 5) {
        tmem_alloc(tmem_slot, 256);
        tmem_relinquish();
    }
    if (warp < 4) {
        // rounded pooled queries of the 128 rows -> the A operand (128-byte swizzle)
        const int r = threadIdx.x;
        const int i = i0 + r;
        const float *q = a.qbar + ((int64_t)bh * a.nQB + min(i, a.nQB - 1)) * D;
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
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 4) {
        if (lane == 0) {
            prefetch_tmap(&tm_k);
            for (int t = 0; t < ntiles; ++t) {
                const int s = t % kFS;
                if (t >= kFS && !mbar_wait(&k_empty[s], ((t / kFS) - 1) & 1, abort_flag, a.status, 40)) break;
                mbar_expect_tx(&k_full[s], L::kKBytes);
                uint8_t *dst = sm + L::kOffK + s * L::kKBytes;
                for (int half = 0; half < 2; ++half)
                    for (int dc = 0; dc < D / 64; ++dc)
                        tma_load_4d(dst + dc * (kTok * 128) + half * (64 * 128), &tm_k, &k_full[s], dc * 64, h,
                                    t * kTok + half * 64, b);
            }
            volatile int32_t no_abort = 0;
            for (int s = 0; s < kFS; ++s) {
                const int n = (ntiles - s + kFS - 1) / kFS;
                if (n > 0) mbar_wait(&k_full[s], (n - 1) & 1, &no_abort, a.status, 41);
            }
        }
    } else if (warp == 5) {
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16_f32(kRowsPerCta, kTok, 0, 0);
            const uint32_t q_addr = smem_u32(sm + L::kOffQ), k_addr = smem_u32(sm + L::kOffK);
            for (int t = 0; t < ntiles; ++t) {
                const int s = t % kFS, sb = t & 1;
                if (!mbar_wait(&k_full[s], (t / kFS) & 1, abort_flag, a.status, 42)) break;
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
        const int r = threadIdx.x;
        const int i = i0 + r;
        const int64_t row = (int64_t)bh * a.nQB + min(i, a.nQB - 1);
        const bool live = i < a.nQB;
        const float th = live ? a.theta[row] : INFINITY;
        const uint32_t *bm = a.bitmask + row * a.nW;
        unsigned long long *out = a.buf + row * a.cap;
        int cnt = 0;
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        uint32_t word = 0;
        int word_idx = -1;
        for (int t = 0; t < ntiles; ++t) {
            const int sb = t & 1;
            bool ok = mbar_wait(&s_full[sb], (t >> 1) & 1, abort_flag, a.status, 45);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
#pragma unroll 1
            for (int c0 = 0; c0 < kTok; c0 += 32) {
                uint32_t v[32];
                tmem_ld32(tmem + lane_base + 128 * sb + c0, v);
                tmem_ld_wait();
                if (th == INFINITY) continue;
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int tok = t * kTok + c0 + e;
                    const float sc = __uint_as_float(v[e]);
                    if (tok >= a.N || !(sc >= th)) continue;
                    const int blk = tok >> 6;
                    if ((blk >> 5) != word_idx) {
                        word_idx = blk >> 5;
                        word = bm[word_idx];
                    }
                    if ((word >> (blk & 31)) & 1u) continue;
                    if (cnt < a.cap) out[cnt] = ((unsigned long long)ord_key(sc) << 32) | (uint32_t)tok;
                    ++cnt;
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_free[sb]);
        }
        if (live) a.cnt[row] = cnt;
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
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
    const unsigned long long *buf = a.buf + r * a.cap;
    uint32_t vk = 0;
    int need = 0;
    if (cnt > a.E) vk = warp_kth([&](int j) { return (uint32_t)(buf[j] >> 32); }, cnt, a.E, hist[warp], &need);
    // survivors are in ascending token order: keep key > v_k, and the first `need` equal ones
    int taken = 0, eq_taken = 0;
    const uint32_t lt = (1u << lane) - 1u;
    for (int j0 = 0; j0 < cnt; j0 += 32) {
        const int j = j0 + lane;
        const bool valid = j < cnt;
        const unsigned long long e = valid ? buf[j] : 0ull;
        const uint32_t key = (uint32_t)(e >> 32);
        bool keep;
        if (cnt <= a.E) {
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

}  // namespace

int64_t extra_buffer_capacity() { return 1024; }

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
    theta_kernel<<<g8, 256, 0, st>>>(a);
    CUtensorMap tm;
    if (!make_k_map(&tm, k, D, p.stride_b, p.stride_n, p.stride_h)) {
        set_error("cuTensorMapEncodeTiled failed for the extra-token scorer");
        return cudaErrorInvalidValue;
    }
    dim3 grid((unsigned)ceil_div(D.nQB, kRowsPerCta), (unsigned)(D.B * D.H));
    if (D.d == 64) {
        e = cudaFuncSetAttribute(filter_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)FLay<64>::bytes);
        if (e != cudaSuccess) return e;
        filter_kernel<64><<<grid, 192, FLay<64>::bytes, st>>>(tm, a);
    } else {
        e = cudaFuncSetAttribute(filter_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)FLay<128>::bytes);
        if (e != cudaSuccess) return e;
        filter_kernel<128><<<grid, 192, FLay<128>::bytes, st>>>(tm, a);
    }
    finalize_kernel<<<g8, 256, 0, st>>>(a);
    fallback_kernel<<<148, 256, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace bsa
