// route.cu -- Sol routing (step 2 for a finite tau) with certified tensor-core
// block scores.
//
// "BlockSparseAttention - ComfyUI Built-in Node Documentation", "sol-attn
// inputs", tau: per (batch, head, query block) row of pooled scores
// S_b = fl32(qbar . kbar_b / sqrt d), the blocks above mean + tau * std of the
// row are kept.  The masks must equal those of the definition bit for bit:
// the scores are the fl32 rounding of an fp64 dot product (FMA per channel in
// channel order), the row mean and population std are taken in fp64 over the
// nKB rounded scores, thr = fl32(mu + tau * sigma), keep iff S_b > thr.
//
// Computing every S_b in fp64 costs 2*rows*nKB*d fp64 FLOP.  Instead:
//
//   gram / gram_reduce  per head, the fp64 mean m and centred second moment
//                       C = (1/n) sum_b (kbar_b - m)(kbar_b - m)^T of the key
//                       centroids (split over key blocks, reduced in order).
//   rowstat             per row, fp64 mu = qbar.m / sqrt d and
//                       sigma^2 = qbar^T C qbar / d -- the mean and std of the
//                       exact scores x_b = qbar.kbar_b / sqrt d -- with
//                       rigorous bounds on their rounding errors and on the
//                       definition's own rounding of the scores to fp32.  The
//                       result is an interval [thr_lo, thr_hi] of fp32 values
//                       that holds the definition's threshold (one to three
//                       values wide in practice).
//   decide              tcgen05 bf16 GEMM of the rounded pooled queries and
//                       key centroids, fp32 accumulation in TMEM.  The error
//                       of each product against the exact dot product is at
//                       most c0 |qbar| |kbar_b| (bf16 rounding of both
//                       operands, 2^-8, plus a generous allowance of 2^-12 for
//                       the accumulation).  A block whose score interval lies
//                       wholly above the threshold interval is kept, wholly
//                       below it dropped; the few others (about 9 of 3248 per
//                       row on the long workload) are listed and, at the end
//                       of the CTA, get their S_b exactly as the definition
//                       computes them, decided against [thr_lo, thr_hi].  A
//                       row with a block inside that interval, more listed
//                       blocks than the list holds, or a std that may be zero
//                       goes to
//   fallback            every S_b of the row exactly, then mean, std and
//                       threshold in the definition's own order of operations
//                       (sequential fp64 sums): the exact mask.
//   count               forced blocks OR'ed in, kept count per row.
//
// The decision rules are sound for any input: only the fraction of rows that
// reach the fallback depends on the data.
#include <float.h>
#include <math.h>

#include <algorithm>

#include "bsa_device.cuh"
#include "bsa_internal.h"

namespace bsa {
namespace {

constexpr int kTM = 128;   // query blocks per decide CTA (UMMA M)
constexpr int kTN = 128;   // key blocks per decide tile (UMMA N)
constexpr int kGramRows = 32;   // key blocks staged per gram step

struct RouteArgs {
    int B, H, N, d, nQB, nKB, nKBp, nW, Bq, Bk;
    int64_t rows;
    int nsplit, chunk;
    double tau;
    int fb;           // forced leading blocks: max(sink blocks, prefix blocks)
    int keep_diag;
    const float *qbar, *kbar;
    __nv_bfloat16 *k16;
    float *knorm;     // [BH, nKBp], 0 beyond nKB
    float *knmax;     // [BH, nKBp / 32] largest norm of each 32-block word
    double *gram, *ksum, *cov, *hstat;   // hstat: [BH, d + 3]
    RowInfo *info;
    int32_t *fbl;
    float *fbs;
    uint32_t *bitmask;
    int32_t *count;
    float *S;         // approximate scores for the extra-token sampler (or null)
    int32_t *status;
};

// Bits of word w (blocks 32w .. 32w+31) that lie in [a, b).
__device__ __forceinline__ uint32_t range_bits(int w, int a, int b)
{
    const int lo = max(a - 32 * w, 0), hi = min(b - 32 * w, 32);
    if (hi <= lo) return 0u;
    const uint32_t upto = hi >= 32 ? 0xffffffffu : ((1u << hi) - 1u);
    const uint32_t below = lo >= 32 ? 0xffffffffu : ((1u << lo) - 1u);
    return upto & ~below;
}

struct Forced {
    int fb, d0, d1;   // [0, fb) and [d0, d1] (empty if d1 < d0)
    __device__ uint32_t bits(int w) const { return range_bits(w, 0, fb) | range_bits(w, d0, d1 + 1); }
};

__device__ __forceinline__ Forced forced_of(const RouteArgs &a, int i)
{
    Forced f;
    f.fb = min(a.fb, a.nKB);
    f.d0 = 1;
    f.d1 = 0;
    if (a.keep_diag) {
        const int q0 = i * a.Bq, q1 = min(a.N, q0 + a.Bq) - 1;
        f.d0 = q0 / a.Bk;
        f.d1 = min(q1 / a.Bk, a.nKB - 1);
    }
    return f;
}

// ------------------------------------------------------------------ prep

// bf16 copies of the key centroids (the decide GEMM's B operand) and their
// Euclidean norms rounded up to f32; one warp per key block (padding blocks
// up to nKBp get norm 0).
__global__ void __launch_bounds__(256) route_prep_kernel(RouteArgs a)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t gb = (int64_t)blockIdx.x * 8 + warp;   // over BH * nKBp
    const int64_t BH = (int64_t)a.B * a.H;
    if (gb >= BH * a.nKBp) return;
    const int64_t bh = gb / a.nKBp;
    const int j = (int)(gb % a.nKBp);
    if (j >= a.nKB) {
        if (lane == 0) a.knorm[gb] = 0.f;
        return;
    }
    const float *k = a.kbar + (bh * a.nKB + j) * a.d;
    __nv_bfloat16 *o = a.k16 + (bh * a.nKB + j) * a.d;
    double s2 = 0.0;
    for (int c = 2 * lane; c < a.d; c += 64) {
        const float2 v = *reinterpret_cast<const float2 *>(k + c);
        s2 = fma((double)v.x, (double)v.x, s2);
        s2 = fma((double)v.y, (double)v.y, s2);
        *reinterpret_cast<__nv_bfloat162 *>(o + c) = __floats2bfloat162_rn(v.x, v.y);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s2 += __shfl_xor_sync(0xffffffffu, s2, off);
    // sqrt of an fp64 sum of squares: relative error far below 2^-40
    if (lane == 0) a.knorm[bh * a.nKBp + j] = __double2float_ru(sqrt(s2) * (1.0 + 0x1p-40));
}

// Largest key-centroid norm of each 32-block word (one thread per word).
__global__ void __launch_bounds__(256) knmax_kernel(RouteArgs a)
{
    const int64_t nwp = a.nKBp / 32;
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (int64_t)a.B * a.H * nwp) return;
    const float4 *k4 = reinterpret_cast<const float4 *>(a.knorm + i * 32);
    float m = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const float4 v = k4[e];
        m = fmaxf(m, fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w)));
    }
    a.knmax[i] = m;
}

// ------------------------------------------------------------------ gram

// Column j of the 8 a rowstat thread owns in a D-wide fp64 tile: pairs 2tx,
// 2tx + 1 spaced D/4 apart, so that the NTX = D/8 threads of a row read one
// contiguous run of shared memory per pair (no bank conflicts).
template <int D>
__device__ __forceinline__ int tile_col(int tx, int j)
{
    return 2 * tx + (j & 1) + (D / 4) * (j >> 1);
}

// Partial sums over one chunk of key blocks: G = sum_b kbar_b kbar_b^T and
// s = sum_b kbar_b, in fp64.  G is symmetric: a CTA computes one 64 x 64 tile
// (I, J), I <= J, of it (three tiles for D = 128, one for D = 64); thread
// (ty, tx) owns rows 4ty..4ty+3 of block I and columns 2tx, 2tx + 1, 2tx + 32,
// 2tx + 33 of block J.  The tile-(0, 0) CTAs also take the sums.
template <int D>
__global__ void __launch_bounds__(256) gram_kernel(RouteArgs a)
{
    constexpr int NTILE = D == 128 ? 3 : 1;
    __shared__ double kd[kGramRows][D];
    const int tile = blockIdx.x % NTILE, split = blockIdx.x / NTILE;
    const int I = tile == 2 ? 1 : 0, J = tile == 0 ? 0 : 1;
    const int64_t bh = blockIdx.y;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    const int b0 = split * a.chunk, b1 = min(a.nKB, b0 + a.chunk);
    double acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.0;
    double ssum = 0.0;
    const bool sums = tile == 0 && threadIdx.x < D;
    const float *kb = a.kbar + bh * (int64_t)a.nKB * D;
    const int ra = 64 * I + 4 * ty, cb = 64 * J + 2 * tx;
    for (int c0 = b0; c0 < b1; c0 += kGramRows) {
        const int nb = min(kGramRows, b1 - c0);
        __syncthreads();
        for (int idx = threadIdx.x; idx < kGramRows * D / 4; idx += 256) {
            const int r = idx / (D / 4), c4 = idx % (D / 4);
            const float4 v = r < nb ? *reinterpret_cast<const float4 *>(&kb[(int64_t)(c0 + r) * D + 4 * c4])
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
            *reinterpret_cast<double2 *>(&kd[r][4 * c4]) = make_double2(v.x, v.y);
            *reinterpret_cast<double2 *>(&kd[r][4 * c4 + 2]) = make_double2(v.z, v.w);
        }
        __syncthreads();
        if (sums)
            for (int r = 0; r < nb; ++r) ssum += kd[r][threadIdx.x];
#pragma unroll 4
        for (int r = 0; r < kGramRows; ++r) {
            const double2 a01 = *reinterpret_cast<const double2 *>(&kd[r][ra]);
            const double2 a23 = *reinterpret_cast<const double2 *>(&kd[r][ra + 2]);
            const double2 b01 = *reinterpret_cast<const double2 *>(&kd[r][cb]);
            const double2 b23 = *reinterpret_cast<const double2 *>(&kd[r][cb + 32]);
            const double av[4] = {a01.x, a01.y, a23.x, a23.y};
            const double bv[4] = {b01.x, b01.y, b23.x, b23.y};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fma(av[i], bv[j], acc[i][j]);
        }
    }
    double *g = a.gram + ((int64_t)bh * a.nsplit + split) * D * D;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        *reinterpret_cast<double2 *>(&g[(ra + i) * D + cb]) = make_double2(acc[i][0], acc[i][1]);
        *reinterpret_cast<double2 *>(&g[(ra + i) * D + cb + 32]) = make_double2(acc[i][2], acc[i][3]);
    }
    if (sums) a.ksum[((int64_t)bh * a.nsplit + split) * D + threadIdx.x] = ssum;
}

// Max over the 256 threads of a block (result valid in every thread).
__device__ __forceinline__ float block_max(float v)
{
    __shared__ float part[8];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = v;
    __syncthreads();
    float r = part[0];
    for (int w = 1; w < 8; ++w) r = fmaxf(r, part[w]);
    __syncthreads();
    return r;
}

// Per head: m = s / n, C = G / n - m m^T, and the scalars tr(G)/n, |m|^2 and
// the largest key-centroid norm (hstat[bh] = {m[0..D), tr(G)/n, |m|^2, max
// |kbar_b|}).  Partials are added in split order.  Grid (D * D / 256, BH): CTA x
// takes entries 256 x .. 256 x + 255 of C (each CTA forms m itself); CTA 0 of a
// head also writes hstat.
template <int D>
__global__ void __launch_bounds__(256) gram_reduce_kernel(RouteArgs a)
{
    __shared__ double m[D];
    __shared__ double diag[D];
    const int64_t bh = blockIdx.y;
    const double n = (double)a.nKB;
    for (int c = threadIdx.x; c < D; c += blockDim.x) {
        double s = 0.0;
        for (int sp = 0; sp < a.nsplit; ++sp) s += a.ksum[(bh * a.nsplit + sp) * D + c];
        m[c] = s / n;
    }
    __syncthreads();
    double *cov = a.cov + bh * D * D;
    {
        const int idx = blockIdx.x * 256 + threadIdx.x;
        const int r = idx / D, c = idx % D;
        // only the tiles on and above the diagonal of 64 x 64 blocks were computed
        const int src = (r >> 6) > (c >> 6) ? c * D + r : idx;
        double g = 0.0;
        for (int sp = 0; sp < a.nsplit; ++sp) g += a.gram[(bh * a.nsplit + sp) * D * D + src];
        g /= n;
        cov[idx] = g - m[r] * m[c];
    }
    if (blockIdx.x != 0) return;
    for (int c = threadIdx.x; c < D; c += blockDim.x) {
        double g = 0.0;
        for (int sp = 0; sp < a.nsplit; ++sp) g += a.gram[(bh * a.nsplit + sp) * D * D + c * D + c];
        diag[c] = g / n;
    }
    float kmax = 0.f;
    for (int j = threadIdx.x; j < a.nKB; j += blockDim.x) kmax = fmaxf(kmax, a.knorm[bh * a.nKBp + j]);
    kmax = block_max(kmax);
    if (threadIdx.x == 0) {
        double tr = 0.0, mm = 0.0;
        for (int c = 0; c < D; ++c) {
            tr += diag[c];
            mm += m[c] * m[c];
        }
        double *hs = a.hstat + bh * (D + 3);
        for (int c = 0; c < D; ++c) hs[c] = m[c];
        hs[D] = tr;
        hs[D + 1] = mm;
        hs[D + 2] = (double)kmax;
    }
}

// ------------------------------------------------------------------ rowstat

// Rows of one head, 128 per CTA: Y = Qbar C in fp64 (thread (ty, tx): rows
// 4ty..4ty+3, columns tile_col(tx, 0..7)), then per row sigma^2 d = qbar . y,
// mu sqrt d = qbar . m and |qbar|^2, and from them the threshold interval and
// the decide kernel's constants.
template <int D>
__global__ void __launch_bounds__(D * 4) rowstat_kernel(RouteArgs a)
{
    constexpr int NTX = D / 8, NT = D * 4;
    extern __shared__ uint8_t rs_smem[];
    double *C = reinterpret_cast<double *>(rs_smem);                  // [D][D]
    float *Qt = reinterpret_cast<float *>(rs_smem + D * D * 8);       // [D][kTM]
    double *hm = reinterpret_cast<double *>(rs_smem + D * D * 8 + D * kTM * 4);   // [D + 3]
    const int64_t bh = blockIdx.y;
    const int i0 = blockIdx.x * kTM;
    const int tx = threadIdx.x % NTX, ty = threadIdx.x / NTX;
    const double *cov = a.cov + bh * D * D;
    for (int idx = threadIdx.x; idx < D * D; idx += NT) C[idx] = cov[idx];
    for (int idx = threadIdx.x; idx < D + 3; idx += NT) hm[idx] = a.hstat[bh * (D + 3) + idx];
    // transposed staging: consecutive threads take consecutive rows, so that the
    // shared-memory stores fall in distinct banks
    for (int idx = threadIdx.x; idx < kTM * D / 4; idx += NT) {
        const int r = idx % kTM, c4 = idx / kTM;
        const float4 v = i0 + r < a.nQB ? *reinterpret_cast<const float4 *>(&a.qbar[(bh * a.nQB + i0 + r) * D + 4 * c4])
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
        Qt[(4 * c4) * kTM + r] = v.x;
        Qt[(4 * c4 + 1) * kTM + r] = v.y;
        Qt[(4 * c4 + 2) * kTM + r] = v.z;
        Qt[(4 * c4 + 3) * kTM + r] = v.w;
    }
    __syncthreads();
    double acc[4][8];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.0;
#pragma unroll 2
    for (int c = 0; c < D; ++c) {
        const float4 q4 = *reinterpret_cast<const float4 *>(&Qt[c * kTM + 4 * ty]);
        const double qv[4] = {(double)q4.x, (double)q4.y, (double)q4.z, (double)q4.w};
        double cv[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const double2 t = *reinterpret_cast<const double2 *>(&C[c * D + tile_col<D>(tx, 2 * j)]);
            cv[2 * j] = t.x;
            cv[2 * j + 1] = t.y;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[i][j] = fma(qv[i], cv[j], acc[i][j]);
    }
    // row reductions over this thread's 8 columns, then over the NTX threads of the row
    double quad[4], qm[4], qn2[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        quad[i] = qm[i] = qn2[i] = 0.0;
        const int row_i = i0 + 4 * ty + i;
        const float *qrow = a.qbar + (bh * a.nQB + min(row_i, a.nQB - 1)) * D;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int col = tile_col<D>(tx, j);
            const double q = row_i < a.nQB ? (double)qrow[col] : 0.0;
            quad[i] = fma(acc[i][j], q, quad[i]);
            qm[i] = fma(q, hm[col], qm[i]);
            qn2[i] = fma(q, q, qn2[i]);
        }
#pragma unroll
        for (int off = NTX / 2; off > 0; off >>= 1) {
            quad[i] += __shfl_xor_sync(0xffffffffu, quad[i], off);
            qm[i] += __shfl_xor_sync(0xffffffffu, qm[i], off);
            qn2[i] += __shfl_xor_sync(0xffffffffu, qn2[i], off);
        }
    }
    if (tx != 0) return;
    const double n = (double)a.nKB;
    const double rs = sqrt((double)D);
    const double trG = hm[D], mm = hm[D + 1];
    const double trC = fmax(0.0, trG - mm);
    // fp64 rounding allowance for sums of up to n + 2D + 64 terms (generous)
    const double g1 = (n + 2.0 * D + 64.0) * 0x1p-53 * 1.25;
    const double up = 1.0 + 0x1p-50;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int row_i = i0 + 4 * ty + i;
        if (row_i >= a.nQB) continue;
        RowInfo info;
        info.pad0 = info.pad1 = 0;
        const double qn = sqrt(qn2[i]) * up;
        const double kr = sqrt(trG) * up;                         // RMS of |kbar_b|
        // sigma^2 of the exact scores: qbar^T C qbar / d
        const double dQ = g1 * qn2[i] * (trG + mm + trC) + 1e-300;
        const double s2lo = fmax(0.0, quad[i] - dQ) / D, s2hi = (quad[i] + dQ) / D;
        const double sig_lo = sqrt(s2lo) * (1.0 - 0x1p-50), sig_hi = sqrt(s2hi) * up;
        const double mu = qm[i] / rs;
        const double dmu = g1 * qn * kr / rs + 0x1p-52 * fabs(mu);
        const double rx = sqrt((fabs(mu) + dmu) * (fabs(mu) + dmu) + sig_hi * sig_hi) * up;   // RMS of the scores
        // the definition rounds each score to f32 (2^-24 relative), its fp64 dot
        // products and sums add far less; both move its mean and std by at most
        const double d_o = 0x1p-24 * rx * (1.0 + 0x1p-20) + 0x1p-44 * qn * kr / rs + (n + 8.0) * 0x1p-52 * rx;
        double tlo, thi;
        if (a.tau >= 0.0) {
            tlo = mu - dmu - d_o + a.tau * (sig_lo - d_o);
            thi = mu + dmu + d_o + a.tau * (sig_hi + d_o);
        } else {
            tlo = mu - dmu - d_o + a.tau * (sig_hi + d_o);
            thi = mu + dmu + d_o + a.tau * (sig_lo - d_o);
        }
        const double slack = 0x1p-50 * (fabs(mu) + fabs(a.tau) * sig_hi + rx);
        tlo -= slack;
        thi += slack;
        info.thr_lo = __double2float_rd(tlo);
        info.thr_hi = __double2float_ru(thi);
        // raw units (dot products without the 1/sqrt d): keep iff raw - E_b is at
        // or above sqrt(d) * nextup(thr_hi); drop iff raw + E_b <= sqrt(d) * thr_lo;
        // E_b = c0 |qbar| |kbar_b| bounds the bf16 tensor-core product's error
        // (and the definition's fp64 chain, 2^-43)
        const double c0 = 0x1p-8 + 0x1p-18 + 0x1p-12 * (1.0 + 0x1p-8) + 0x1p-43;
        const double tup = (double)nextafterf(info.thr_hi, INFINITY);
        const double hi_raw = rs * tup, lo_raw = rs * (double)info.thr_lo;
        // absolute slack: products of values near the bottom of the f32 range may
        // be flushed (128 x 2^-126), and bf16 rounding of subnormals is absolute
        const double abs_slack = 0x1p-110 + 0x1p-120 * qn;
        info.c = __double2float_ru(c0 * qn * (1.0 + 0x1p-20));
        info.hi = __double2float_ru(hi_raw + 0x1p-20 * fabs(hi_raw) + abs_slack);
        info.lo = __double2float_rd(lo_raw - 0x1p-20 * fabs(lo_raw) - abs_slack);
        // a std that may be zero, products that might overflow f32, or anything
        // not finite leave the row to the exact path
        const bool ok = sig_lo - d_o > 0.0 && qn * hm[D + 2] < 0x1p100 && isfinite(info.thr_lo) &&
                        isfinite(info.thr_hi) && isfinite(info.hi) && isfinite(info.lo) && isfinite(info.c);
        info.mode = ok ? 0 : 1;
        a.info[bh * a.nQB + row_i] = info;
    }
}

// ------------------------------------------------------------------ exact scores

// S_b exactly as the definition computes it: fp64 FMA per channel in channel
// order from 0, divided by sqrt(d) in fp64, rounded to f32.  The chain is
// serial; the key row is loaded 32 values ahead of it.
template <int D, typename QT>
__device__ __forceinline__ float exact_score(const QT *qd, const float *k, double rs)
{
    constexpr int CH = 8;              // float4 per chunk (32 values)
    constexpr int NCH = D / (4 * CH);
    const float4 *k4 = reinterpret_cast<const float4 *>(k);
    float4 cur[CH], nxt[CH];
#pragma unroll
    for (int e = 0; e < CH; ++e) cur[e] = __ldg(k4 + e);
    double acc = 0.0;
#pragma unroll
    for (int ch = 0; ch < NCH; ++ch) {
        if (ch + 1 < NCH) {
#pragma unroll
            for (int e = 0; e < CH; ++e) nxt[e] = __ldg(k4 + (ch + 1) * CH + e);
        }
#pragma unroll
        for (int e = 0; e < CH; ++e) {
            const int c = 4 * (ch * CH + e);
            acc = __fma_rn((double)qd[c], (double)cur[e].x, acc);
            acc = __fma_rn((double)qd[c + 1], (double)cur[e].y, acc);
            acc = __fma_rn((double)qd[c + 2], (double)cur[e].z, acc);
            acc = __fma_rn((double)qd[c + 3], (double)cur[e].w, acc);
        }
        if (ch + 1 < NCH) {
#pragma unroll
            for (int e = 0; e < CH; ++e) cur[e] = nxt[e];
        }
    }
    return __double2float_rn(__ddiv_rn(acc, rs));
}

// Two of them at once (independent chains, one instruction stream), each with
// its own query row.
template <int D>
__device__ __forceinline__ void exact_score2(const float *q0, const float *q1, const float *k0, const float *k1,
                                             double rs, float *s0, float *s1)
{
    const float4 *a4 = reinterpret_cast<const float4 *>(k0);
    const float4 *b4 = reinterpret_cast<const float4 *>(k1);
    const float4 *p4 = reinterpret_cast<const float4 *>(q0);
    const float4 *q4 = reinterpret_cast<const float4 *>(q1);
    double x = 0.0, y = 0.0;
    float4 ka = __ldg(a4), kb = __ldg(b4);
#pragma unroll 4
    for (int c4 = 0; c4 < D / 4; ++c4) {
        const float4 na = c4 + 1 < D / 4 ? __ldg(a4 + c4 + 1) : ka;
        const float4 nb = c4 + 1 < D / 4 ? __ldg(b4 + c4 + 1) : kb;
        const float4 pv = p4[c4], qv = q4[c4];
        x = __fma_rn((double)pv.x, (double)ka.x, x);
        y = __fma_rn((double)qv.x, (double)kb.x, y);
        x = __fma_rn((double)pv.y, (double)ka.y, x);
        y = __fma_rn((double)qv.y, (double)kb.y, y);
        x = __fma_rn((double)pv.z, (double)ka.z, x);
        y = __fma_rn((double)qv.z, (double)kb.z, y);
        x = __fma_rn((double)pv.w, (double)ka.w, x);
        y = __fma_rn((double)qv.w, (double)kb.w, y);
        ka = na;
        kb = nb;
    }
    *s0 = __double2float_rn(__ddiv_rn(x, rs));
    *s1 = __double2float_rn(__ddiv_rn(y, rs));
}

template <typename QT>
__device__ __forceinline__ float exact_score_d(const QT *qd, const float *k, int d, double rs)
{
    return d == 128 ? exact_score<128>(qd, k, rs) : exact_score<64>(qd, k, rs);
}

__device__ __forceinline__ void push_fallback(const RouteArgs &a, int64_t r)
{
    const int pos = atomicAdd(&a.fbl[0], 1);
    a.fbl[1 + pos] = (int32_t)r;
}

// ------------------------------------------------------------------ decide

template <int D>
struct DLay {
    static constexpr int kStages = D == 128 ? 4 : 6;
    static constexpr int kQBytes = kTM * D * 2;
    static constexpr int kKBytes = kTN * D * 2;
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kQBytes;
    static constexpr int kOffBar = kOffK + kStages * kKBytes;   // k_full[S], k_empty[S], s_full[2], s_free[2], done
    static constexpr int kOffMisc = kOffBar + (2 * kStages + 5) * 8;
    static constexpr int kOffUcnt = kOffMisc + 16;             // [kTM] i32 undecided blocks per row
    static constexpr int kOffAmb = kOffUcnt + kTM * 4;         // [kTM] i32 a row's exact pass was inconclusive
    static constexpr int kOffUl = kOffAmb + kTM * 4;           // [kTM][kUcap] u16 the undecided blocks
    static constexpr int kOffKx = kOffUl + kTM * kUcap * 2;    // [nKBp / 32] f32 largest key norm per word
    static size_t bytes(int nwp) { return (size_t)kOffKx + (size_t)nwp * 4 + 1024; }
};

// Warps 0-7 read the scores (warp w: TMEM lane quarter w & 3, columns 64 (w >> 2)
// .. +63 of each 128-block tile); warp 8 loads key tiles by TMA; warp 9 issues
// the MMAs and owns TMEM.  One CTA per 128 rows of a head, streaming all key
// tiles; S double-buffered in TMEM.
template <int D>
__global__ void __launch_bounds__(320, 1) decide_kernel(const __grid_constant__ CUtensorMap tm_k, RouteArgs a)
{
    using L = DLay<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.y;
    const int i0 = blockIdx.x * kTM;
    const int ntiles = (a.nKB + kTN - 1) / kTN;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::kOffBar);
    uint64_t *k_full = bars, *k_empty = bars + L::kStages, *s_full = bars + 2 * L::kStages, *s_free = s_full + 2,
             *bar_done = s_full + 4;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + L::kOffMisc);
    volatile int32_t *abort_flag = reinterpret_cast<volatile int32_t *>(sm + L::kOffMisc + 4);
    int32_t *ucnt_s = reinterpret_cast<int32_t *>(sm + L::kOffUcnt);
    int32_t *amb_s = reinterpret_cast<int32_t *>(sm + L::kOffAmb);
    uint16_t *ul_s = reinterpret_cast<uint16_t *>(sm + L::kOffUl);
    float *kx_s = reinterpret_cast<float *>(sm + L::kOffKx);

    const int r = threadIdx.x & (kTM - 1);
    const bool live = i0 + r < a.nQB;
    const int64_t row = (int64_t)bh * a.nQB + min(i0 + r, a.nQB - 1);

    if (threadIdx.x == 0) {
        for (int s = 0; s < L::kStages; ++s) {
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
        // pooled queries rounded to bf16 -> the A operand (K-major, 128-byte swizzle)
        const float4 *q4 = reinterpret_cast<const float4 *>(a.qbar + row * D);
        const uint32_t base = smem_u32(sm + L::kOffQ) + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll 4
        for (int ch = 0; ch < D / 8; ++ch) {
            const float4 x = live ? q4[2 * ch] : make_float4(0.f, 0.f, 0.f, 0.f);
            const float4 y = live ? q4[2 * ch + 1] : make_float4(0.f, 0.f, 0.f, 0.f);
            const int dc = ch >> 3, c16 = ch & 7;
            st_shared_v4(base + dc * (kTM * 128) + ((c16 ^ (r & 7)) << 4), pack_bf16x2(x.x, x.y),
                         pack_bf16x2(x.z, x.w), pack_bf16x2(y.x, y.y), pack_bf16x2(y.z, y.w));
        }
        fence_async_smem();
        ucnt_s[r] = 0;
        amb_s[r] = 0;
    } else if (warp < 8) {
        const float *src = a.knmax + (int64_t)bh * (a.nKBp / 32);
        for (int i = threadIdx.x - 128; i < a.nKBp / 32; i += 128) kx_s[i] = src[i];
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 8) {
        if (lane == 0) {
            prefetch_tmap(&tm_k);
            for (int t = 0; t < ntiles; ++t) {
                const int s = t % L::kStages;
                if (t >= L::kStages &&
                    !mbar_wait(&k_empty[s], ((t / L::kStages) - 1) & 1, abort_flag, a.status, 60))
                    break;
                mbar_expect_tx(&k_full[s], L::kKBytes);
                uint8_t *dst = sm + L::kOffK + s * L::kKBytes;
                for (int dc = 0; dc < D / 64; ++dc)
                    tma_load_3d(dst + dc * (kTN * 128), &tm_k, &k_full[s], dc * 64, t * kTN, bh);
            }
            volatile int32_t no_abort = 0;
            for (int s = 0; s < L::kStages; ++s) {
                const int nfill = (ntiles - s + L::kStages - 1) / L::kStages;
                if (nfill > 0) mbar_wait(&k_full[s], (nfill - 1) & 1, &no_abort, a.status, 61);
            }
        }
    } else if (warp == 9) {
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16_f32(kTM, kTN, 0, 0);
            const uint32_t q_addr = smem_u32(sm + L::kOffQ), k_addr = smem_u32(sm + L::kOffK);
            for (int t = 0; t < ntiles; ++t) {
                const int s = t % L::kStages, sb = t & 1;
                if (!mbar_wait(&k_full[s], (t / L::kStages) & 1, abort_flag, a.status, 62)) break;
                if (t >= 2 && !mbar_wait(&s_free[sb], ((t >> 1) - 1) & 1, abort_flag, a.status, 63)) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t ad = sdesc_sw128(q_addr + (kk >> 2) * (kTM * 128) + (kk & 3) * 32, 16, 1024);
                    const uint64_t bd =
                        sdesc_sw128(k_addr + s * L::kKBytes + (kk >> 2) * (kTN * 128) + (kk & 3) * 32, 16, 1024);
                    umma_bf16(tmem + 128 * sb, ad, bd, idesc, kk > 0 ? 1u : 0u);
                }
                umma_commit(&s_full[sb]);
                umma_commit(&k_empty[s]);
            }
            umma_commit(bar_done);
            volatile int32_t no_abort = 0;
            mbar_wait(bar_done, 0, &no_abort, a.status, 64);
        }
    } else {
        const int g = warp >> 2, sub = warp & 3;
        const RowInfo info = a.info[row];
        const bool work = live && info.mode == 0;
        const Forced fo = forced_of(a, min(i0 + r, a.nQB - 1));
        const float inv_rs = (float)(1.0 / sqrt((double)D));
        const float *kn_head = a.knorm + (int64_t)bh * a.nKBp;
        uint32_t *bm = a.bitmask + row * a.nW;
        uint16_t *ul = ul_s + r * kUcap;
        const uint32_t lane_base = (uint32_t)(sub * 32) << 16;
        for (int t = 0; t < ntiles; ++t) {
            const int sb = t & 1;
            const bool go = __all_sync(0xffffffffu, mbar_wait(&s_full[sb], (t >> 1) & 1, abort_flag, a.status, 65));
            tc_fence_after();
            uint32_t v[64];
            if (go) {
                tmem_ld32(tmem + lane_base + 128 * sb + 64 * g, *reinterpret_cast<uint32_t(*)[32]>(v));
                tmem_ld32(tmem + lane_base + 128 * sb + 64 * g + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
                tmem_ld_wait();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_free[sb]);   // the scores are in registers
            if (!go || !live) continue;
            const int j0 = t * kTN + 64 * g;
#pragma unroll
            for (int w2 = 0; w2 < 2; ++w2) {
                const int wi = (j0 >> 5) + w2;
                if (wi >= a.nW) break;
                const uint32_t *vw = v + 32 * w2;
                if (a.S != nullptr) {
                    float *srow = a.S + row * a.nKB;
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (32 * wi + e < a.nKB) srow[32 * wi + e] = __uint_as_float(vw[e]) * inv_rs;
                }
                if (!work) continue;
                // word-wide bounds from the word's largest key norm: every block of
                // the word has l_b >= lmin and u_b <= umax, so most scores are
                // decided by two compares; the rest get their own bounds
                const float kmx = kx_s[wi];
                const float lmin = fmaf(-info.c, kmx, info.lo);
                const float umax = fmaf(info.c, kmx, info.hi);
                uint32_t kw = 0u, slow = 0u;
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const float x = __uint_as_float(vw[e]);
                    kw |= x > umax ? (1u << e) : 0u;
                    slow |= (x < lmin || x > umax) ? 0u : (1u << e);
                }
                const uint32_t valid = range_bits(wi, 0, a.nKB);
                slow &= valid & ~fo.bits(wi);
                uint32_t uw = 0u;
                for (uint32_t m = slow; m != 0u; m &= m - 1u) {
                    const int e = __ffs(m) - 1;
                    const float x = __uint_as_float(select32(vw, e));
                    const float kn = __ldg(kn_head + 32 * wi + e);
                    if (x > fmaf(info.c, kn, info.hi))
                        kw |= 1u << e;
                    else if (!(x < fmaf(-info.c, kn, info.lo)))
                        uw |= 1u << e;
                }
                bm[wi] = kw & valid;
                for (uint32_t m = uw; m != 0u; m &= m - 1u) {
                    const int pos = atomicAdd(&ucnt_s[r], 1);
                    if (pos < kUcap) ul[pos] = (uint16_t)(32 * wi + __ffs(m) - 1);
                }
            }
        }
        named_bar_sync(1, 256);
        // The undecided blocks' scores exactly as the definition computes them,
        // decided against [thr_lo, thr_hi]; a row with an inconclusive block, more
        // undecided blocks than the list holds, or mode 1 goes to the exact path.
        // The CTA's listed (row, block) pairs are spread evenly over its 256
        // threads (flat index f: row by binary search in the rows' list offsets),
        // so that no thread walks a long row alone.  The rows' f32 queries, list
        // offsets and threshold intervals are staged in the K ring, idle once every
        // tile has been read (the MMA warp's last S is in registers by now).
        constexpr int QP = D + 4;
        float *qs = reinterpret_cast<float *>(sm + L::kOffK);                   // [kTM][QP]
        int32_t *pre_s = reinterpret_cast<int32_t *>(qs + kTM * QP);           // [kTM + 1] list offsets
        float2 *thr_s = reinterpret_cast<float2 *>(pre_s + kTM + 4);           // [kTM] (thr_lo, thr_hi)
        static_assert(kTM * QP * 4 + (kTM + 4) * 4 + kTM * 8 <= L::kStages * L::kKBytes, "decide: K ring too small");
        for (int idx = threadIdx.x; idx < kTM * D / 4; idx += 256) {
            const int rr = idx / (D / 4), c4 = idx % (D / 4);
            const float4 v = i0 + rr < a.nQB
                                 ? *reinterpret_cast<const float4 *>(a.qbar + ((int64_t)bh * a.nQB + i0 + rr) * D + 4 * c4)
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
            *reinterpret_cast<float4 *>(qs + rr * QP + 4 * c4) = v;
        }
        if (g == 0) {
            // this row's listed blocks that take the exact score here (none for a
            // row sent to the exact path or past the end)
            const int u = ucnt_s[r];
            const bool listed = live && info.mode == 0 && u <= kUcap;
            if (live && !listed) push_fallback(a, row);
            ucnt_s[r] = listed ? u : 0;
            thr_s[r] = make_float2(info.thr_lo, info.thr_hi);
        }
        named_bar_sync(1, 256);
        if (warp == 0) {
            // exclusive scan of the 128 counts, 4 a lane
            const int c0 = ucnt_s[4 * lane], c1 = ucnt_s[4 * lane + 1], c2 = ucnt_s[4 * lane + 2],
                      c3 = ucnt_s[4 * lane + 3];
            const int sum = c0 + c1 + c2 + c3;
            int incl = sum;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            const int excl = incl - sum;
            pre_s[4 * lane] = excl;
            pre_s[4 * lane + 1] = excl + c0;
            pre_s[4 * lane + 2] = excl + c0 + c1;
            pre_s[4 * lane + 3] = excl + c0 + c1 + c2;
            if (lane == 31) pre_s[kTM] = incl;
        }
        named_bar_sync(1, 256);
        const int total = pre_s[kTM];
        const float *kb = a.kbar + (int64_t)bh * a.nKB * D;
        const double rs = sqrt((double)D);
        // row and block of flat index f (the last row whose list starts at or before f)
        auto locate = [&](int f, int &rr, int &jj) {
            int lo = 0, hi = kTM - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (pre_s[mid] <= f)
                    lo = mid;
                else
                    hi = mid - 1;
            }
            rr = lo;
            jj = ul_s[lo * kUcap + (f - pre_s[lo])];
        };
        auto decide1 = [&](int rr, int jj, float sv) {
            const float2 th = thr_s[rr];
            const int64_t rw = (int64_t)bh * a.nQB + i0 + rr;
            if (sv > th.y)
                atomicOr(&a.bitmask[rw * a.nW + (jj >> 5)], 1u << (jj & 31));
            else if (!(sv <= th.x) && atomicExch(&amb_s[rr], 1) == 0)
                push_fallback(a, rw);
        };
        for (int f = threadIdx.x; f < total; f += 512) {
            int r0, j0;
            locate(f, r0, j0);
            if (f + 256 < total) {
                // two independent chains side by side
                int r1, j1;
                locate(f + 256, r1, j1);
                float s0, s1;
                exact_score2<D>(qs + r0 * QP, qs + r1 * QP, kb + (int64_t)j0 * D, kb + (int64_t)j1 * D, rs, &s0, &s1);
                decide1(r0, j0, s0);
                decide1(r1, j1, s1);
            } else {
                decide1(r0, j0, exact_score<D>(qs + r0 * QP, kb + (int64_t)j0 * D, rs));
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// ------------------------------------------------------------------ exact

// ------------------------------------------------------------------ fallback

// Rows whose threshold could not be bracketed tightly enough: every score
// exactly, then mean, population std and threshold in the definition's order
// of operations (sequential fp64 sums over the blocks in index order).  The
// row's scores sit in shared memory when they fit (nKBp <= kFbSmem), else in
// the CTA's global scratch row.
constexpr int kFbSmem = 16384;

__global__ void __launch_bounds__(512) fallback_rows_kernel(RouteArgs a)
{
    extern __shared__ float fb_smem[];
    __shared__ double qd[128];
    __shared__ float thr_s;
    __shared__ int keep_s;
    __shared__ double red_d[16], red_s[16];
    __shared__ int red_i[16];
    const int nfb = a.fbl[0];
    float *srow = a.nKBp <= kFbSmem ? fb_smem : a.fbs + (int64_t)blockIdx.x * a.nKBp;
    const double rs = sqrt((double)a.d);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int f = blockIdx.x; f < nfb; f += gridDim.x) {
        const int64_t r = a.fbl[1 + f];
        const int64_t bh = r / a.nQB;
        __syncthreads();
        for (int c = threadIdx.x; c < a.d; c += blockDim.x) qd[c] = (double)a.qbar[r * a.d + c];
        __syncthreads();
        // every score exactly, and in the same pass the smallest exponent of a
        // nonzero score and the sum of |score| (for the exactness test below)
        int emin = 1 << 20;
        double sabs = 0.0, ssum = 0.0;
        for (int j = threadIdx.x; j < a.nKB; j += blockDim.x) {
            const float sv = exact_score_d(qd, a.kbar + (bh * a.nKB + j) * a.d, a.d, rs);
            srow[j] = sv;
            if (sv != 0.f) emin = min(emin, ilogbf(sv));
            sabs += fabs((double)sv);
            ssum += (double)sv;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            emin = min(emin, __shfl_xor_sync(0xffffffffu, emin, o));
            sabs += __shfl_xor_sync(0xffffffffu, sabs, o);
            ssum += __shfl_xor_sync(0xffffffffu, ssum, o);
        }
        if (lane == 0) {
            red_i[warp] = emin;
            red_d[warp] = sabs;
            red_s[warp] = ssum;
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            const int nwarp = (int)(blockDim.x >> 5);
            int e = red_i[0];
            double sa = red_d[0];
            for (int w = 1; w < nwarp; ++w) {
                e = min(e, red_i[w]);
                sa += red_d[w];
            }
            // Every score is a multiple of 2^(e - 23).  If the sum of |scores|
            // stays below 2^(e - 23 + 53) (here with a factor 2 to spare), every
            // partial sum in any order is exactly representable in fp64, so the
            // definition's sequential sum equals a sum in any order.
            const bool exact_sum = e == (1 << 20) || sa < ldexp(1.0, e - 23 + 52);
            const int n = a.nKB;
            double mu = 0.0;
            if (exact_sum) {
                for (int w = 0; w < nwarp; ++w) mu += red_s[w];
            } else {
                int j = 0;
                for (; j + 8 <= n; j += 8) {
                    float v[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) v[e] = srow[j + e];
#pragma unroll
                    for (int e = 0; e < 8; ++e) mu = __dadd_rn(mu, (double)v[e]);
                }
                for (; j < n; ++j) mu = __dadd_rn(mu, (double)srow[j]);
            }
            mu = __ddiv_rn(mu, (double)n);
            double var = 0.0;
            int j = 0;
            for (; j + 8 <= n; j += 8) {
                double e2[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const double dv = __dadd_rn((double)srow[j + e], -mu);
                    e2[e] = __dmul_rn(dv, dv);
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) var = __dadd_rn(var, e2[e]);
            }
            for (; j < n; ++j) {
                const double dv = __dadd_rn((double)srow[j], -mu);
                var = __dadd_rn(var, __dmul_rn(dv, dv));
            }
            var = __ddiv_rn(var, (double)n);
            const double sigma = __dsqrt_rn(var);
            thr_s = __double2float_rn(__dadd_rn(mu, __dmul_rn(a.tau, sigma)));
            keep_s = sigma > 0.0;
        }
        __syncthreads();
        const float thr = thr_s;
        const bool any = keep_s != 0;
        for (int w = threadIdx.x; w < a.nW; w += blockDim.x) {
            uint32_t word = 0u;
            for (int e = 0; e < 32; ++e) {
                const int j = 32 * w + e;
                if (any && j < a.nKB && srow[j] > thr) word |= 1u << e;
            }
            a.bitmask[r * a.nW + w] = word;
        }
    }
}

// ------------------------------------------------------------------ count

__global__ void __launch_bounds__(256) route_count_kernel(RouteArgs a)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t r = (int64_t)blockIdx.x * 8 + warp;
    if (r >= a.rows) return;
    const Forced fo = forced_of(a, (int)(r % a.nQB));
    uint32_t *bm = a.bitmask + r * a.nW;
    int c = 0;
    for (int w = lane; w < a.nW; w += 32) {
        const uint32_t word = bm[w] | fo.bits(w);
        bm[w] = word;
        c += __popc(word);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) c += __shfl_xor_sync(0xffffffffu, c, off);
    if (lane == 0) a.count[r] = c;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

// bf16 [BH, nKB, d]; box = 64 channels x 128 key blocks x 1 head.
bool make_k16_map(CUtensorMap *m, const void *base, int BH, int nKB, int d)
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
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)nKB, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)nKB * d * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)kTN, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
cudaError_t launch_route_d(const RouteArgs &a, cudaStream_t st)
{
    const int64_t BH = (int64_t)a.B * a.H;
    count_launch();
    route_prep_kernel<<<(unsigned)ceil_div(BH * a.nKBp, 8), 256, 0, st>>>(a);
    count_launch();
    knmax_kernel<<<(unsigned)ceil_div(BH * (a.nKBp / 32), 256), 256, 0, st>>>(a);
    count_launch();
    gram_kernel<D><<<dim3((unsigned)(a.nsplit * (D == 128 ? 3 : 1)), (unsigned)BH), 256, 0, st>>>(a);
    count_launch();
    gram_reduce_kernel<D><<<dim3(D * D / 256, (unsigned)BH), 256, 0, st>>>(a);
    const int rs_smem = D * D * 8 + D * kTM * 4 + (D + 3) * 8;
    cudaError_t e = cudaFuncSetAttribute(rowstat_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, rs_smem);
    if (e != cudaSuccess) return e;
    const dim3 gt((unsigned)ceil_div(a.nQB, kTM), (unsigned)BH);
    count_launch();
    rowstat_kernel<D><<<gt, D * 4, rs_smem, st>>>(a);
    CUtensorMap tm;
    if (!make_k16_map(&tm, a.k16, (int)BH, a.nKB, D)) {
        set_error("cuTensorMapEncodeTiled failed for the routing scores");
        return cudaErrorInvalidValue;
    }
    const int bytes = (int)DLay<D>::bytes(a.nKBp / 32);
    if (bytes > 232448) {
        set_error("routing: too many key blocks for the score tiles' shared memory");
        return cudaErrorInvalidValue;
    }
    e = cudaFuncSetAttribute(decide_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    count_launch();
    decide_kernel<D><<<gt, 320, bytes, st>>>(tm, a);
    const unsigned g8 = (unsigned)ceil_div(a.rows, 8);
    const int fb_smem = a.nKBp <= kFbSmem ? a.nKBp * 4 : 0;
    if (fb_smem > 48 * 1024) {
        e = cudaFuncSetAttribute(fallback_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, fb_smem);
        if (e != cudaSuccess) return e;
    }
    count_launch();
    fallback_rows_kernel<<<(unsigned)fallback_ctas(), 512, fb_smem, st>>>(a);
    count_launch();
    route_count_kernel<<<g8, 256, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace

bool certified_route(const bsa_params &p) { return p.method == BSA_SOL && isfinite(p.tau); }

int route_nsplit(const Dims &D) { return (int)std::min<int64_t>(16, std::max<int64_t>(1, ceil_div(D.nKB, 384))); }

cudaError_t launch_route(const bsa_params &p, const Dims &D, const float *qbar, const float *kbar, char *ws,
                         const WsLayout &L, cudaStream_t st)
{
    RouteArgs a;
    a.B = D.B;
    a.H = D.H;
    a.N = D.N;
    a.d = D.d;
    a.nQB = D.nQB;
    a.nKB = D.nKB;
    a.nKBp = (int)route_nkbp(D);
    a.nW = D.nW;
    a.Bq = D.Bq;
    a.Bk = D.Bk;
    a.rows = D.rows;
    a.nsplit = L.r_nsplit;
    a.chunk = (int)(ceil_div(ceil_div(D.nKB, a.nsplit), kGramRows) * kGramRows);
    a.tau = p.tau;
    a.fb = std::max(p.sink_blocks, p.prefix_len > 0 ? (int)ceil_div(p.prefix_len, D.Bk) : 0);
    a.keep_diag = p.keep_diag;
    a.qbar = qbar;
    a.kbar = kbar;
    a.k16 = reinterpret_cast<__nv_bfloat16 *>(ws + L.r_k16);
    a.knorm = reinterpret_cast<float *>(ws + L.r_knorm);
    a.knmax = reinterpret_cast<float *>(ws + L.r_knmax);
    a.gram = reinterpret_cast<double *>(ws + L.r_gram);
    a.ksum = reinterpret_cast<double *>(ws + L.r_ksum);
    a.cov = reinterpret_cast<double *>(ws + L.r_cov);
    a.hstat = reinterpret_cast<double *>(ws + L.r_hstat);
    a.info = reinterpret_cast<RowInfo *>(ws + L.r_info);
    a.fbl = reinterpret_cast<int32_t *>(ws + L.r_fbl);
    a.fbs = reinterpret_cast<float *>(ws + L.r_fbs);
    a.bitmask = reinterpret_cast<uint32_t *>(ws + L.bitmask);
    a.count = reinterpret_cast<int32_t *>(ws + L.counts);
    a.S = p.extra_tokens > 0 ? reinterpret_cast<float *>(ws + L.scores) : nullptr;
    a.status = reinterpret_cast<int32_t *>(ws + L.status);
    cudaError_t e = cudaMemsetAsync(a.fbl, 0, sizeof(int32_t), st);
    if (e != cudaSuccess) return e;
    return D.d == 64 ? launch_route_d<64>(a, st) : launch_route_d<128>(a, st);
}

}  // namespace bsa
