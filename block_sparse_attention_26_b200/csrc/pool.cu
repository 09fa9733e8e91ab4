// pool.cu -- step 1: block mean pooling of Q, K and V.
//
// "minimax-h3-chunk-star7" README, sections "SLA" (Q=128, K=64 block routing)
// and "Sol" (Q64/K64 routing; unselected blocks approximated by their K/V
// centroid): Q is pooled per query block for routing, K per key block for
// routing and, with V, for the centroids.
//
// HBM-bound: every input byte is read once with 16-byte non-caching loads.
// A CTA owns one (tensor, batch, block) and streams the block's tokens; a
// thread owns 16 contiguous bytes of a token row (8 bf16 or 4 f32 channels of
// one head).  Sums are kept in fp64 in token order, so the mean is the exact
// block mean rounded once to f32 (ties with the definition bit for bit).
#include "bsa_device.cuh"
#include "bsa_internal.h"

namespace bsa {
namespace {

template <typename T>
struct Vec;
template <>
struct Vec<__nv_bfloat16> {
    static constexpr int kN = 8;
    __device__ static void add(double (&acc)[8], const uint4 &r)
    {
        const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            acc[2 * i] += (double)__uint_as_float(w[i] << 16);
            acc[2 * i + 1] += (double)__uint_as_float(w[i] & 0xFFFF0000u);
        }
    }
};
template <>
struct Vec<float> {
    static constexpr int kN = 4;
    __device__ static void add(double (&acc)[4], const uint4 &r)
    {
        acc[0] += (double)__uint_as_float(r.x);
        acc[1] += (double)__uint_as_float(r.y);
        acc[2] += (double)__uint_as_float(r.z);
        acc[3] += (double)__uint_as_float(r.w);
    }
};

struct PoolArgs {
    const void *src[3];
    float *dst[3];
    int nb[3];
    int blk[3];
    int64_t sb, sn, sh;
    int N, H, d;
    int32_t *count;       // written for the key blocks (tensor 1)
    // cube tiling: blocks past the prefix's pre_blocks are cubes of the grid
    int cube, pre_blocks, P, gH, gW, cT, cH, cW, ncx, ncy;
};

// Token of slot t (0..63) of block i: the prefix's own tokens, or the cube's
// tokens t-major inside the cube, cubes t-major over the grid.  As the cube's
// first token plus a slot offset that does not depend on the cube.
__device__ __forceinline__ int cube_origin(const PoolArgs &a, int i)
{
    if (i < a.pre_blocks) return i * 64;
    const int c = i - a.pre_blocks;
    const int cx = c % a.ncx, cy = (c / a.ncx) % a.ncy, ct = c / (a.ncx * a.ncy);
    return a.P + (ct * a.cT * a.gH + cy * a.cH) * a.gW + cx * a.cW;
}

__device__ __forceinline__ int slot_offset(const PoolArgs &a, int i, int t)
{
    if (i < a.pre_blocks) return t;
    const int dx = t % a.cW, dy = (t / a.cW) % a.cH, dt = t / (a.cW * a.cH);
    return (dt * a.gH + dy) * a.gW + dx;
}

template <typename T, int UNROLL>
__global__ void __launch_bounds__(128) pool_kernel(PoolArgs a)
{
    constexpr int V = Vec<T>::kN;
    const int z = blockIdx.z;
    const int i = blockIdx.x;
    const int b = blockIdx.y;
    const int nbz = z == 0 ? a.nb[0] : a.nb[1];
    if (i >= nbz) return;
    const int blk = z == 0 ? a.blk[0] : a.blk[1];
    const int t0 = i * blk;
    const int n = min(a.N, t0 + blk) - t0;
    const T *base = static_cast<const T *>(z == 0 ? a.src[0] : (z == 1 ? a.src[1] : a.src[2]));
    float *dst = z == 0 ? a.dst[0] : (z == 1 ? a.dst[1] : a.dst[2]);
    const int cols = a.H * a.d / V;
    __shared__ int slot_off[64];
    int origin = 0;
    if (a.cube) {
        // the block's token offsets once per CTA (integer divisions are slow)
        if (threadIdx.x < 64) slot_off[threadIdx.x] = slot_offset(a, i, threadIdx.x);
        origin = cube_origin(a, i);
        __syncthreads();
    }
    for (int col = threadIdx.x; col < cols; col += blockDim.x) {
        const int h = (col * V) / a.d;
        const int c = (col * V) % a.d;
        const T *p = base + (int64_t)b * a.sb + (int64_t)t0 * a.sn + (int64_t)h * a.sh + c;
        double acc[V];
#pragma unroll
        for (int e = 0; e < V; ++e) acc[e] = 0.0;
        int t = 0;
        if (a.cube) {
            const T *pb = base + (int64_t)b * a.sb + (int64_t)origin * a.sn + (int64_t)h * a.sh + c;
            for (; t + UNROLL <= n; t += UNROLL) {
                uint4 r[UNROLL];
#pragma unroll
                for (int u = 0; u < UNROLL; ++u) r[u] = ld_nc_v4(pb + (int64_t)slot_off[t + u] * a.sn);
#pragma unroll
                for (int u = 0; u < UNROLL; ++u) Vec<T>::add(acc, r[u]);
            }
            for (; t < n; ++t) Vec<T>::add(acc, ld_nc_v4(pb + (int64_t)slot_off[t] * a.sn));
        }
        for (; t + UNROLL <= n; t += UNROLL) {
            uint4 r[UNROLL];
#pragma unroll
            for (int u = 0; u < UNROLL; ++u) r[u] = ld_nc_v4(p + (int64_t)(t + u) * a.sn);
#pragma unroll
            for (int u = 0; u < UNROLL; ++u) Vec<T>::add(acc, r[u]);
        }
        for (; t < n; ++t) Vec<T>::add(acc, ld_nc_v4(p + (int64_t)t * a.sn));
        float *o = dst + (((int64_t)b * a.H + h) * nbz + i) * a.d + c;
        float res[V];
#pragma unroll
        for (int e = 0; e < V; ++e) res[e] = (float)(acc[e] / (double)n);
        if constexpr (V == 8) {
            reinterpret_cast<float4 *>(o)[0] = make_float4(res[0], res[1], res[2], res[3]);
            reinterpret_cast<float4 *>(o)[1] = make_float4(res[4], res[5], res[6], res[7]);
        } else {
            reinterpret_cast<float4 *>(o)[0] = make_float4(res[0], res[1], res[2], res[3]);
        }
    }
    if (z == 1 && b == 0 && threadIdx.x == 0 && a.count != nullptr) a.count[i] = n;
}

}  // namespace

cudaError_t launch_pool(const bsa_params &p, const Dims &D, const void *q, const void *k,
                        const void *v, float *qbar, float *kbar, float *vbar, int32_t *blk_count,
                        cudaStream_t st)
{
    PoolArgs a;
    a.src[0] = q;
    a.src[1] = k;
    a.src[2] = v;
    a.dst[0] = qbar;
    a.dst[1] = kbar;
    a.dst[2] = vbar;
    a.nb[0] = D.nQB;
    a.nb[1] = a.nb[2] = D.nKB;
    a.blk[0] = D.Bq;
    a.blk[1] = a.blk[2] = D.Bk;
    a.sb = p.stride_b;
    a.sn = p.stride_n;
    a.sh = p.stride_h;
    a.N = D.N;
    a.H = D.H;
    a.d = D.d;
    a.count = blk_count;
    a.cube = D.cube;
    a.pre_blocks = D.pre_blocks;
    a.P = p.prefix_len;
    a.gH = p.grid_h;
    a.gW = p.grid_w;
    a.cT = p.cube_t;
    a.cH = p.cube_h;
    a.cW = p.cube_w;
    a.ncx = D.cube ? p.grid_w / p.cube_w : 1;
    a.ncy = D.cube ? p.grid_h / p.cube_h : 1;
    dim3 grid(std::max(D.nQB, D.nKB), D.B, 3);
    count_launch();
    if (p.dtype == BSA_DT_BF16)
        pool_kernel<__nv_bfloat16, 8><<<grid, 128, 0, st>>>(a);
    else
        pool_kernel<float, 8><<<grid, 128, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace bsa
